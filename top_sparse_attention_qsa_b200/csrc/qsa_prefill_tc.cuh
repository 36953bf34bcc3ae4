// qsa_prefill_tc.cuh -- QSA top-K sparse-attention prefill, cp.async-gather +
// tcgen05 (TMEM) kernel for sm_100a.
//
// The operation (page "Qwen4-Exp QSA llega al Ascend de Huawei", section
// "Lo que realmente añade la pull request"; bullets "Formas de cabeza" and
// "Límites de tamaño"): for each (query token t, KV head g) unit, the G query
// heads of the group attend to the cache rows named by the token's list,
// softmax(scale q K_sel^T) V_sel, -1 / n_valid masking, zeros for empty rows.
//
// Persistent CTAs (one per SM) walk the units in KV-head-major order.
// Sixteen warps in four warpgroups with fixed roles, synchronised only
// through mbarriers; registers are rebalanced per warpgroup (setmaxnreg) so
// that the softmax keeps 176 per thread and each producer 120:
//   warps 4-11  eight producers: read each tile's 128 list entries one
//               tile ahead and gather the K and V rows (in the order K(0),
//               K(1), V(0), K(2), V(1), ... within a unit, so that a tile's
//               V rows land about when its probabilities are ready) with
//               16-byte cp.async copies written straight into the
//               128-byte-swizzled layout the tensor core reads, into a ring
//               of six 32 KB slots (one half, dims 0-127 or 128-255, of a
//               tile's K or V rows each); masked entries are zero-filled
//               without a global read.  Warp 4 also loads the 16 Q rows of
//               the unit (tiled TMA, double-buffered).  Each lane computes
//               where its copies land in a slot once, and where its rows
//               sit in the cache once per tile (for the K and the V copies
//               of both halves): per copy only an add and the copy remain.
//   warp 12     one thread issues the score MMAs (tcgen05.mma, kind::f16):
//               S^T[128 keys x 16 heads] = K_tile . Q^T (M=128, N=16, K-major
//               operands) into a TMEM double buffer.
//   warp 13     one thread issues the PV MMAs: O^T[256 x 16] += V_tile^T . P^T
//               (two M=128 halves, V read MN-major from the same slots) into
//               TMEM.  Two issuers keep PV of tile i from queueing behind the
//               scores of tile i+1.
//   warps 0-3   softmax: thread k owns TMEM lane k = key k of the tile;
//               exponentials in base 2 from the running max; P^T written
//               MN-major to shared memory; the running max is only raised
//               (with an O rescale in TMEM) when a head's max grows by more
//               than 2^8, which keeps every p <= 256 and the result exact up
//               to rounding.  A warp vote per tile detects that case; only
//               then is the tile max per head formed (a transposing shuffle
//               reduction and a 4-warp exchange).
//               Epilogue: lse = m + ln l, O / l -> BF16 rows, zeros for empty rows.
// The consumers of the ring take only their own slots (the score MMAs the K
// slots, PV the V slots) and skip the others without waiting.  That is safe
// because every lane's cp.async copies complete in issue order and, in this
// gather order, the previous fill of the slot a consumer waits on was always
// issued before the last slot that consumer waited on: when that one is
// full, so is the older fill, and a parity wait can never take an older
// phase of the slot for the one it waits for.  (Running the K rows two or
// more tiles ahead breaks this at unit boundaries, where the V rows of the
// last tiles follow each other.)
// Every wait (all on mbarriers, including the exchanges inside the softmax
// group) is bounded by 2 s of %globaltimer; on expiry the kernel raises status
// bit 1, every role stops, in-flight copies and MMAs are drained and the TMEM
// is released.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "qsa_ptx.cuh"
#include "qsa_tc_ptx.cuh"

namespace qsa {
namespace tc {

constexpr int kKeys = 128;                 // list entries per tile (M of the score MMA)
constexpr int kGp = 16;                    // query heads per group, padded (N)
constexpr int kSlotBytes = 32768;          // 128 rows x 128 dims x 2 B
constexpr int kSlots = 6;
constexpr int kBlockBytes = 16384;         // 128 rows x 64 dims (one 128-byte swizzle column block)
constexpr int kQBytes = kGp * 512;         // 16 rows x 256 dims x 2 B
constexpr int kPBytes = kKeys * kGp * 2;   // 128 keys x 16 heads x 2 B
// Eight producer warps, each lane with its copies' addresses computed once:
// more warps with fewer copies each in flight move random rows faster (the
// gather probe's finding), up to where their instructions crowd the issue
// slots of the softmax and MMA warps.
constexpr int kProducerWarps = 8;          // 16 rows of every tile each
static_assert(kKeys % (2 * kProducerWarps) == 0 && kKeys / kProducerWarps <= 32,
              "each producer lane holds at most one row id; rows per warp must be even");
// Warp roles, in warpgroups of four (registers are rebalanced per warpgroup):
//   warps 0-3     softmax (TMEM lane quadrants 0-3)
//   warps 4-11    producers
//   warp 12       score MMA issuer, warp 13 PV MMA issuer, warps 14-15 idle
constexpr int kWarpSoftmax0 = 0, kWarpProducer0 = 4;
constexpr int kWarpQK = kWarpProducer0 + kProducerWarps, kWarpPV = kWarpQK + 1;
constexpr int kProducerGroups = kProducerWarps / 4;   // warpgroups of producers
constexpr int kThreads = 32 * (kProducerWarps + 8);
// Registers per thread after setmaxnreg: softmax / producers / MMA warpgroup.
// Their sum over the four warpgroups (x 128 threads) must stay within what the
// block is launched with, 512 threads x 128 registers: 176 + 2 * 120 + 64 =
// 480 <= 4 * 128.
constexpr int kRegsSoftmax = 176, kRegsProducer = 120, kRegsMma = 64, kRegsLaunch = 128;
static_assert(kProducerWarps % 4 == 0 &&
                  kRegsSoftmax + kProducerGroups * kRegsProducer + kRegsMma <= (kProducerGroups + 2) * kRegsLaunch,
              "the register split exceeds the launch allocation");
constexpr int kTmemCols = 64;              // S double buffer (2 x 16) + O (2 halves x 16)
constexpr float kRescaleLog2 = 8.f;        // lazy-rescale threshold (p <= 2^8)

constexpr int OFF_RING = 0;
constexpr int OFF_Q = OFF_RING + kSlots * kSlotBytes;
constexpr int OFF_P = OFF_Q + 2 * kQBytes;
constexpr int OFF_RED = OFF_P + 2 * kPBytes;     // max[4][16], votes[2][4], sum[2][4][16]
constexpr int OFF_BAR = OFF_RED + 1024;
// barrier indices
constexpr int B_FULL = 0, B_EMPTY = 6, B_SFULL = 12, B_SFREE = 14, B_PFULL = 16, B_PEMPTY = 18,
              B_QFULL = 20, B_QEMPTY = 22, B_OFULL = 24, B_OEMPTY = 25, B_RMAX = 26, B_RSUM = 28,
              B_DONE = 30, B_RMX2 = 32, NUM_BARS = 33;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem base, abort flag
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment


struct TcParams {
  CUtensorMap tm_q;                 // Q as [T][Hq][256], box 16 heads x 64 dims
  const int32_t* idx;
  const int32_t* n_valid;
  const void* kraw;                 // K and V cache base pointers
  const void* vraw;
  __nv_bfloat16* out;
  float* lse;
  int32_t* status;
  int32_t* gathered;                // debug dump [T][Hkv][K << block_shift] or nullptr
  int64_t T;
  int64_t idx_st, idx_sh, o_st, o_sh, lse_st, kv_ss, kv_sh;
  int32_t Hkv, G, K, S;
  float scale_log2;
  // split-K: each list is cut into `splits` chunks of `chunk` entries (a
  // multiple of 128); with part_o set, every (token, KV head, chunk) unit
  // writes its normalised partial O (FP32 [T*Hq][splits][256]) and partial
  // lse ([T*Hq][splits]) there instead of out/lse, for a merge pass.
  int32_t splits, chunk;
  float* part_o;
  float* part_lse;
  // microblock lists: entry e names slots (idx[e] << block_shift) + r, r <
  // 2^block_shift, each one key (0: token lists); last_slot [T] bounds the
  // slots a token sees (nullptr: no bound).  K and n_valid count entries;
  // chunk counts keys.
  int32_t block_shift;
  const int32_t* last_slot;
  // output scale applied with the 1/l normalisation (the V dequantisation
  // scale of an FP8 cache, in the FP8 kernel; 1 otherwise)
  float o_scale;
  // Q in global memory (the FP8 kernel reads it directly; strides in elements)
  const void* q_ptr;
  int64_t q_st, q_sh;
};

// Instruction descriptors (kind::f16): FP32 accumulator, BF16 A and B,
// N = 16 (bits 17-22 hold N/8), M = 128 (bits 24-28 hold M/16).
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | (2u << 17) | (8u << 24);
// PV: both operands MN-major (bits 15 and 16).
constexpr uint32_t kIdescPV = kIdescQK | (1u << 15) | (1u << 16);


struct Unit {
  int64_t t;
  int g;
  int s;       // chunk of the list (split-K), 0 without splitting
  int j0;      // first list entry of the chunk
  int n_eff;   // live-range length inside the chunk
  int n_tiles;
};

__device__ __forceinline__ int64_t num_units(const TcParams& p) { return p.T * p.Hkv * p.splits; }

// Unit u -> (KV head, token, chunk), KV head outermost so that concurrent
// CTAs share one head's cache rows.
__device__ __forceinline__ Unit decode_unit(const TcParams& p, int64_t u) {
  Unit r;
  const int64_t per_head = p.T * p.splits;
  r.g = static_cast<int>(u / per_head);
  const int64_t rem = u - static_cast<int64_t>(r.g) * per_head;
  r.t = rem / p.splits;
  r.s = static_cast<int>(rem - r.t * p.splits);
  int n = p.K;
  if (p.n_valid != nullptr) n = min(n, max(__ldg(p.n_valid + r.t * p.Hkv + r.g), 0));
  const int n_keys = n << p.block_shift;
  r.j0 = r.s * p.chunk;
  r.n_eff = max(0, min(n_keys - r.j0, p.chunk));
  r.n_tiles = (r.n_eff + kKeys - 1) / kKeys;
  return r;
}

// List entry behind key `local` (counted from the unit's first key), or -1
// past the unit's live range.  A plain load with no use of its value, so it
// can be issued a tile ahead and resolved (key_slot) when needed.
template <bool kBlocks>
__device__ __forceinline__ int32_t key_entry(const TcParams& p, const int32_t* list, const Unit& un,
                                             int local) {
  const int key = un.j0 + local;
  return local < un.n_eff ? __ldg(list + (kBlocks ? key >> p.block_shift : key)) : -1;
}

// Cache slot of key `local` given its list entry: -1 when the key is masked
// (negative entry, past the cache end or the token's last visible slot), -2
// when the entry names a block that starts beyond the cache (reported
// through the status word).
template <bool kBlocks>
__device__ __forceinline__ int32_t key_slot(const TcParams& p, const Unit& un, int local,
                                            int32_t entry, int32_t last) {
  if (entry < 0) return -1;
  if (!kBlocks) return entry >= p.S ? -2 : entry;
  const int64_t start = static_cast<int64_t>(entry) << p.block_shift;
  if (start >= p.S) return -2;
  const int64_t slot = start + ((un.j0 + local) & ((1 << p.block_shift) - 1));
  if (slot >= p.S || slot > last) return -1;
  return static_cast<int32_t>(slot);
}

__device__ __forceinline__ int32_t last_visible(const TcParams& p, int64_t t) {
  return p.last_slot != nullptr ? __ldg(p.last_slot + t) : 0x7fffffff;
}

// Reduce 16 per-lane values across the 32 lanes of a warp by exchanging
// halves (16 shuffles instead of 80).  Lane l ends with the result for head
// (l >> 1) & 15.
template <bool kMax>
__device__ __forceinline__ float xreduce16(const float (&v)[16], int lane) {
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[8], b[4], c[2];
  bool up = (lane & 16) != 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float send = up ? v[j] : v[8 + j];
    const float keep = up ? v[8 + j] : v[j];
    a[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
  up = (lane & 8) != 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float send = up ? a[j] : a[4 + j];
    const float keep = up ? a[4 + j] : a[j];
    b[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
  up = (lane & 4) != 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float send = up ? b[j] : b[2 + j];
    const float keep = up ? b[2 + j] : b[j];
    c[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
  up = (lane & 2) != 0;
  float d = op(up ? c[1] : c[0], __shfl_xor_sync(0xffffffffu, up ? c[0] : c[1], 2));
  d = op(d, __shfl_xor_sync(0xffffffffu, d, 1));
  return d;
}

// ------------------------------------------------------------------ producer

// kProducerWarps warps gather the K and V rows of each tile with 16-byte
// cp.async copies written straight into the 128-byte-swizzled K-major layout
// the tensor core reads.  Warp w owns rows_w = 128 / kProducerWarps rows of
// every tile; one warp instruction moves the 256-byte half rows of two keys
// (16 lanes each).
// Masked entries are zero-filled without a global read.  Every lane signals
// the slot's full barrier when its own copies land (cp.async.mbarrier.arrive).
// kStall (test hook): withhold the completion signal of the first ring slot,
// so that every wait must expire and the kernel must stop with kStatusTimeout.
template <bool kDump, bool kStall, bool kBlocks>
__device__ void producer_role(const TcParams& p, const Sync& sy, uint32_t sb, int pw, int lane) {
  uint32_t c_slot = 0, c_unit = 0;
  const int64_t units = num_units(p);
  uint32_t q_issued = 0, q_par = 0;                  // per Q buffer: load issued, its phase parity
  const int cc = lane & 15;                          // 16-byte chunk of the half row
  const int rsel = lane >> 4;                        // which of the two rows of an instruction
  const uint32_t dchunk = static_cast<uint32_t>((cc >> 3) * kBlockBytes);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    if (pw == 0) {
      const uint32_t qb = c_unit & 1u;
      if (lane == 0) {
        ok = sy.wait(B_QEMPTY + qb, ((c_unit >> 1) & 1u) ^ 1u);
        if (ok) {
          mbar_arrive_expect_tx(sy.bar(B_QFULL + qb), kQBytes);
#pragma unroll
          for (int b = 0; b < 4; ++b)
            tma_load_3d(sb + OFF_Q + qb * kQBytes + b * (kQBytes / 4), &p.tm_q, b * 64, un.g * p.G,
                        static_cast<int32_t>(un.t), sy.bar(B_QFULL + qb));
          q_issued |= 1u << qb;
          q_par = (q_par & ~(1u << qb)) | (((c_unit >> 1) & 1u) << qb);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    ++c_unit;
    if (!ok) break;
    const int32_t* list = p.idx + un.t * p.idx_st + static_cast<int64_t>(un.g) * p.idx_sh;
    const int32_t last = kBlocks ? last_visible(p, un.t) : 0x7fffffff;
    const char* kbase = reinterpret_cast<const char*>(p.kraw) + static_cast<int64_t>(un.g) * p.kv_sh * 2 + cc * 16;
    const char* vbase = reinterpret_cast<const char*>(p.vraw) + static_cast<int64_t>(un.g) * p.kv_sh * 2 + cc * 16;
    const int64_t row_bytes = p.kv_ss * 2;
    // list entry of this lane's row (rows_w rows per warp; lanes >= rows_w idle), one tile ahead
    constexpr int rows_w = kKeys / kProducerWarps;
    const int jr = rows_w * pw + lane;
    const bool own = lane < rows_w;
    // this lane's copies: one 16-byte chunk of rows_w / 2 rows per half tile;
    // their places in a slot never change, their sources change per tile
    constexpr int kCopies = rows_w / 2;
    uint32_t dofs[kCopies];
#pragma unroll
    for (int k = 0; k < kCopies; ++k) {
      const int r = rows_w * pw + 2 * k + rsel;                   // row of the tile
      dofs[k] = dchunk + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
    }
    // byte offsets in the cache of the rows this lane copies for one tile,
    // from the row slots the owning lanes resolved (-1: masked, zero-filled)
    auto row_offsets = [&](int32_t id, int64_t (&off)[kCopies]) {
#pragma unroll
      for (int k = 0; k < kCopies; ++k) {
        const int32_t rid = __shfl_sync(0xffffffffu, id, 2 * k + rsel);
        off[k] = rid >= 0 ? static_cast<int64_t>(rid) * row_bytes : int64_t(-1);
      }
    };
    // the tile's two K or V ring slots (dims 0-127, 128-255) for this lane's
    // share of the rows
    auto issue = [&](int i, bool v, const int64_t (&off)[kCopies]) {
      const char* base = v ? vbase : kbase;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const uint32_t slot = c_slot % kSlots;
        const uint32_t round = c_slot / kSlots;
        ok = sy.wait_warp(B_EMPTY + slot, (round & 1u) ^ 1u);
        if (!ok) return;
        const char* src0 = base + h * 256;
        const uint32_t dst0 = sb + OFF_RING + slot * kSlotBytes;
#pragma unroll
        for (int k = 0; k < kCopies; ++k) {
          const int r = rows_w * pw + 2 * k + rsel;               // row of the tile
          const bool live = off[k] >= 0;
          const char* src = src0 + (live ? off[k] : int64_t(0));
          cp_async_16(dst0 + dofs[k], src, live ? 16 : 0);
          if (kDump && cc == 0 && h == 0) {
            // debug dump: the slot this copy read, recovered from its source
            // address (-1 for a zero-filled row); the V copy of a key (by the
            // same lane, after the K copy) must agree, else -2 is recorded
            const int32_t from = live ? static_cast<int32_t>((src - src0) / row_bytes) : -1;
            const int64_t key = un.j0 + static_cast<int64_t>(i) * kKeys + r;
            const int64_t n_keys = static_cast<int64_t>(p.K) << p.block_shift;
            if (key < n_keys) {
              int32_t* d = p.gathered + (un.t * p.Hkv + un.g) * n_keys + key;
              if (!v)
                *d = from;
              else if (*d != from)
                *d = -2;
            }
          }
        }
        if (!(kStall && c_slot == 0)) cp_async_mbar_arrive(sy.bar(B_FULL + slot));
        ++c_slot;
      }
    };
    // slot of this lane's row of tile i from its entry (loaded a tile ahead)
    auto resolve = [&](int i, int32_t e) {
      int32_t id = key_slot<kBlocks>(p, un, i * kKeys + jr, e, last);
      if (id == -2) {
        id = -1;
        if (p.status != nullptr) atomicOr(p.status, static_cast<int32_t>(kStatusOob));
      }
      return id;
    };
    // Order within a unit: K(0), K(1), V(0), K(2), V(1), ..., V(n-1): a
    // tile's V rows follow the next tile's K rows, so that they land about
    // when the tile's probabilities are ready.
    int32_t entry_next = own ? key_entry<kBlocks>(p, list, un, jr) : -1;
    int64_t off0[kCopies], off1[kCopies];
    row_offsets(resolve(0, entry_next), off0);
    entry_next = (own && 1 < un.n_tiles) ? key_entry<kBlocks>(p, list, un, kKeys + jr) : -1;
    if (un.n_tiles > 0) issue(0, false, off0);
    for (int i = 0; i < un.n_tiles && ok; ++i) {
      if (i + 1 < un.n_tiles) {
        row_offsets(resolve(i + 1, entry_next), off1);
        entry_next = (own && i + 2 < un.n_tiles) ? key_entry<kBlocks>(p, list, un, (i + 2) * kKeys + jr) : -1;
        issue(i + 1, false, off1);
        if (!ok) break;
      }
      issue(i, true, off0);
#pragma unroll
      for (int k = 0; k < kCopies; ++k) off0[k] = off1[k];
    }
  }
  // every copy this lane issued has landed before the CTA can exit
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  if (pw == 0 && lane == 0)
    for (int b = 0; b < 2; ++b)
      if (q_issued & (1u << b)) sy.drain(B_QFULL + b, (q_par >> b) & 1u);
}

// ------------------------------------------------------------------ MMA issuers

// Scores: S^T[c & 1] = K_tile(c) . Q^T for every tile c of the CTA.
__device__ void qk_role(const TcParams& p, const Sync& sy, uint32_t sb, uint32_t tmem) {
  uint32_t c_tile = 0, c_unit = 0;
  const int64_t units = num_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t qb = c_unit & 1u;
    ok = sy.wait(B_QFULL + qb, (c_unit >> 1) & 1u);
    if (!ok) break;
    ++c_unit;
    if (un.n_tiles == 0) {
      mbar_arrive(sy.bar(B_QEMPTY + qb));
      continue;
    }
    const uint32_t qaddr = sb + OFF_Q + qb * kQBytes;
    for (int i = 0; i < un.n_tiles && ok; ++i, ++c_tile) {
      const uint32_t c = c_tile;
      const uint32_t sbuf = c & 1u;
      ok = sy.wait(B_SFREE + sbuf, ((c >> 1) & 1u) ^ 1u);
      // the unit's items in the producers' order: K(0), K(1), V(0), K(2), ...
      const uint32_t item = 2u * (c - i) + (i == 0 ? 0u : 2u * i - 1u);
      for (int h = 0; h < 2 && ok; ++h) {
        const uint32_t ck = 2u * item + h;
        const uint32_t slot = ck % kSlots;
        ok = sy.wait(B_FULL + slot, (ck / kSlots) & 1u);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int ks = h * 8 + kk;
          // A = K tile, B = Q: K-major, 128-byte swizzle, 8-row groups 1 KB
          // apart; a 16-dim step advances 32 B inside the swizzle atom.
          const uint64_t a = smem_desc(
              sb + OFF_RING + slot * kSlotBytes + (kk >> 2) * kBlockBytes + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t b = smem_desc(qaddr + (ks >> 2) * (kQBytes / 4) + (ks & 3) * 32, 16, 1024, 2);
          umma_f16_ss(tmem + sbuf * 16, a, b, kIdescQK, ks > 0 ? 1u : 0u);
        }
        umma_commit(sy.bar(B_EMPTY + slot));
      }
      if (!ok) break;
      umma_commit(sy.bar(B_SFULL + sbuf));
      if (i == un.n_tiles - 1) umma_commit(sy.bar(B_QEMPTY + qb));
    }
  }
  // no tensor-core operation of this thread may still run when TMEM is released
  umma_commit(sy.bar(B_DONE));
  sy.drain(B_DONE, 0);
}

// PV: O^T (two M=128 halves) += V_tile(c)^T . P^T(c) for every tile c.
__device__ void pv_role(const TcParams& p, const Sync& sy, uint32_t sb, uint32_t tmem) {
  uint32_t c_tile = 0, c_unit = 0;
  const int64_t units = num_units(p);
  const uint32_t t_o = tmem + 32;  // O halves: columns 32-47 and 48-63
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t ue = c_unit++;
    // the previous unit's epilogue has read O
    ok = sy.wait(B_OEMPTY, (ue & 1u) ^ 1u);
    if (!ok) break;
    if (un.n_tiles == 0) {
      mbar_arrive(sy.bar(B_OFULL));
      continue;
    }
    for (int i = 0; i < un.n_tiles && ok; ++i, ++c_tile) {
      const uint32_t c = c_tile;
      const uint32_t pb = c & 1u;
      ok = sy.wait(B_PFULL + pb, (c >> 1) & 1u);
      const uint32_t item = 2u * (c - i) + (i + 1 < un.n_tiles ? 2u * i + 2u : 2u * un.n_tiles - 1u);
      for (int mh = 0; mh < 2 && ok; ++mh) {
        const uint32_t cv = 2u * item + mh;
        const uint32_t slot = cv % kSlots;
        ok = sy.wait(B_FULL + slot, (cv / kSlots) & 1u);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = V^T: MN-major, 128-byte swizzle; the two 64-dim blocks of the
          // half are 16 KB apart (LBO), groups of 8 keys 1 KB apart (SBO).
          const uint64_t a = smem_desc(sb + OFF_RING + slot * kSlotBytes + kk * 2048, kBlockBytes, 1024, 2);
          // B = P^T: MN-major, no swizzle; 8x8 core matrices, key groups 128 B
          // apart (LBO), head groups 2 KB apart (SBO).
          const uint64_t b = smem_desc(sb + OFF_P + pb * kPBytes + kk * 256, 128, 2048, 0);
          umma_f16_ss(t_o + mh * 16, a, b, kIdescPV, (i == 0 && kk == 0) ? 0u : 1u);
        }
        umma_commit(sy.bar(B_EMPTY + slot));
      }
      if (!ok) break;
      umma_commit(sy.bar(B_PEMPTY + pb));
    }
    if (ok) umma_commit(sy.bar(B_OFULL));
  }
  umma_commit(sy.bar(B_DONE + 1));
  sy.drain(B_DONE + 1, 0);
}

// ------------------------------------------------------------------ softmax

// p = 2^(s - m) for this thread's key and 16 heads, as BF16 pairs; pv gets
// the unrounded p for the running sums.
__device__ __forceinline__ void form_p16(const float (&s)[kGp], const float (&m)[kGp], uint32_t (&pk)[8],
                                         float (&pv)[kGp]) {
#pragma unroll
  for (int h = 0; h < kGp; h += 2) {
    pv[h] = ex2(s[h] - (m[h] == -INFINITY ? 0.f : m[h]));
    pv[h + 1] = ex2(s[h + 1] - (m[h + 1] == -INFINITY ? 0.f : m[h + 1]));
    pk[h >> 1] = pack_bf16x2(pv[h], pv[h + 1]);
  }
}

template <bool kBlocks>
__device__ void softmax_role(const TcParams& p, const Sync& sy, uint32_t sb, uint8_t* sp,
                             uint32_t tmem, int warp, int lane) {
  const int wq = warp & 3;                       // TMEM lane quadrant of this warp
  const int key = wq * 32 + lane;                // TMEM lane = key row of the tile
  const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  float* red_max = reinterpret_cast<float*>(sp + OFF_RED);        // [4][16]
  uint8_t* votes = sp + OFF_RED + 256;                             // [2][4]
  float* red_sum = red_max + 128;                                  // [2][4][16]
  uint32_t c_tile = 0, c_unit = 0, c_exact = 0;
  const int64_t units = num_units(p);
  const int G = p.G;
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const int32_t* list = p.idx + un.t * p.idx_st + static_cast<int64_t>(un.g) * p.idx_sh;
    const int32_t last = kBlocks ? last_visible(p, un.t) : 0x7fffffff;
    float m_run[kGp], l_part[kGp];
#pragma unroll
    for (int h = 0; h < kGp; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    // list entry of this thread's key, read one tile ahead
    int32_t entry_next = un.n_tiles > 0 ? key_entry<kBlocks>(p, list, un, key) : -1;
    for (int i = 0; i < un.n_tiles; ++i) {
      const uint32_t c = c_tile + i;
      const uint32_t buf = c & 1u;
      // this tile's entry was loaded a tile ago: resolve it before waiting for S
      const bool valid = key_slot<kBlocks>(p, un, i * kKeys + key, entry_next, last) >= 0;
      entry_next = i + 1 < un.n_tiles ? key_entry<kBlocks>(p, list, un, (i + 1) * kKeys + key) : -1;
      ok = sy.wait_warp(B_SFULL + buf, (c >> 1) & 1u);
      if (!ok) break;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tl + buf * 16, r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(B_SFREE + buf));
      float s[kGp];
      bool over = false;
#pragma unroll
      for (int h = 0; h < kGp; ++h) {
        s[h] = (valid && h < G) ? __uint_as_float(r[h]) * p.scale_log2 : -INFINITY;
        over |= s[h] > m_run[h] + kRescaleLog2;
      }
      // Most tiles hold no score above the running max plus the lazy-rescale
      // bound.  Each warp votes on that and forms P from the running max
      // while the other votes arrive; only a yes anywhere (the first tile of
      // a unit, a real rescale) makes the warps exchange exact tile maxima
      // and form P again.  P always uses the running max, so the result is
      // the same either way.
      const bool wover = __any_sync(0xffffffffu, over);
      uint8_t* vt = votes + buf * 4;
      if (lane == 0) vt[wq] = wover ? 1 : 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(B_RMAX + buf));
      uint32_t pk[8];
      float pv[kGp];
      if (!wover) form_p16(s, m_run, pk, pv);
      ok = sy.wait_warp(B_RMAX + buf, (c >> 1) & 1u);  // all four votes are in
      if (!ok) break;
      if (*reinterpret_cast<const uint32_t*>(vt) != 0u) {
        // tile max per head over the 128 keys
        const float wmax = xreduce16<true>(s, lane);
        float* rm = red_max;
        if ((lane & 1) == 0) rm[wq * 16 + ((lane >> 1) & 15)] = wmax;
        __syncwarp();
        if (lane == 0) mbar_arrive(sy.bar(B_RMX2));
        ok = sy.wait_warp(B_RMX2, c_exact & 1u);  // all four warps' maxima are in
        ++c_exact;
        if (!ok) break;
        float tmax[kGp];
#pragma unroll
        for (int h = 0; h < kGp; ++h)
          tmax[h] = fmaxf(fmaxf(rm[h], rm[16 + h]), fmaxf(rm[32 + h], rm[48 + h]));
        bool need = false;
#pragma unroll
        for (int h = 0; h < kGp; ++h)
          need |= (m_run[h] != -INFINITY) && (tmax[h] > m_run[h] + kRescaleLog2);
        if (need) {
          // raise the running max: O (TMEM) and the partial sums scale by 2^(m_old - m_new)
          if (i > 0) {
            const uint32_t cp = c - 1;
            ok = sy.wait_warp(B_PEMPTY + (cp & 1u), (cp >> 1) & 1u);  // the previous PV has finished
            if (!ok) break;
          }
          tc_fence_after();
          float alpha[kGp];
#pragma unroll
          for (int h = 0; h < kGp; ++h) {
            const float mn = fmaxf(m_run[h], tmax[h]);
            alpha[h] = m_run[h] == -INFINITY ? 1.f : ex2(m_run[h] - mn);
            m_run[h] = mn;
            l_part[h] *= alpha[h];
          }
          if (i > 0) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t o[16];
              tmem_ld16(tl + 32 + half * 16, o);
              tmem_wait_ld();
#pragma unroll
              for (int h = 0; h < kGp; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
              tmem_st16(tl + 32 + half * 16, o);
            }
            tmem_wait_st();
          }
        } else {
#pragma unroll
          for (int h = 0; h < kGp; ++h)
            if (m_run[h] == -INFINITY) m_run[h] = tmax[h];
        }
        form_p16(s, m_run, pk, pv);
      }
#pragma unroll
      for (int h = 0; h < kGp; ++h) l_part[h] += pv[h];
      ok = sy.wait_warp(B_PEMPTY + buf, ((c >> 1) & 1u) ^ 1u);
      if (!ok) break;
      // P^T row of this key: heads 0-7 in the first 8x8 core-matrix column,
      // heads 8-15 in the second (2 KB further)
      const uint32_t pa = sb + OFF_P + buf * kPBytes + (key >> 3) * 128 + (key & 7) * 16;
      st_shared_v4(pa, pk[0], pk[1], pk[2], pk[3]);
      st_shared_v4(pa + 2048, pk[4], pk[5], pk[6], pk[7]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(B_PFULL + buf));
    }
    if (!ok) break;
    // epilogue: l per head over the 128 threads
    const float wsum = xreduce16<false>(l_part, lane);
    float* rs = red_sum + (c_unit & 1u) * 64;
    if ((lane & 1) == 0) rs[wq * 16 + ((lane >> 1) & 15)] = wsum;
    __syncwarp();
    if (lane == 0) mbar_arrive(sy.bar(B_RSUM + (c_unit & 1u)));
    ok = sy.wait_warp(B_RSUM + (c_unit & 1u), (c_unit >> 1) & 1u);
    if (!ok) break;
    float l_tot[kGp];
#pragma unroll
    for (int h = 0; h < kGp; ++h) l_tot[h] = (rs[h] + rs[16 + h]) + (rs[32 + h] + rs[48 + h]);
    ok = sy.wait_warp(B_OFULL, c_unit & 1u);
    if (!ok) break;
    tc_fence_after();
    uint32_t o0[16] = {}, o1[16] = {};
    if (un.n_tiles > 0) {
      tmem_ld16(tl + 32, o0);
      tmem_ld16(tl + 48, o1);
      tmem_wait_ld();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sy.bar(B_OEMPTY));
    const int64_t row0 = un.t * static_cast<int64_t>(p.Hkv) * G + static_cast<int64_t>(un.g) * G;
    __nv_bfloat16* orow = p.out + un.t * p.o_st + static_cast<int64_t>(un.g) * G * p.o_sh;
#pragma unroll
    for (int h = 0; h < kGp; ++h) {
      if (h < G) {
        const bool live = l_tot[h] > 0.f;
        const float inv = live ? 1.f / l_tot[h] : 0.f;
        const float v0 = live ? __uint_as_float(o0[h]) * inv : 0.f;
        const float v1 = live ? __uint_as_float(o1[h]) * inv : 0.f;
        if (p.part_o != nullptr) {
          float* po = p.part_o + ((row0 + h) * p.splits + un.s) * 256;
          po[key] = v0;
          po[128 + key] = v1;
        } else {
          orow[h * p.o_sh + key] = __float2bfloat16_rn(v0);
          orow[h * p.o_sh + 128 + key] = __float2bfloat16_rn(v1);
        }
      }
    }
    if (key < G && (p.lse != nullptr || p.part_lse != nullptr)) {
      float mk = 0.f, lk = 0.f;
#pragma unroll
      for (int h = 0; h < kGp; ++h)
        if (h == key) {
          mk = m_run[h];
          lk = l_tot[h];
        }
      const float lv = lk > 0.f ? (mk + lg2(lk)) * 0.69314718055994531f : -INFINITY;
      if (p.part_lse != nullptr)
        p.part_lse[(row0 + key) * p.splits + un.s] = lv;
      else
        p.lse[un.t * p.lse_st + static_cast<int64_t>(un.g) * G + key] = lv;
    }
    c_tile += un.n_tiles;
    ++c_unit;
  }
}

// ------------------------------------------------------------------ kernel

template <bool kDump, bool kStall = false, bool kBlocks = false>
__global__ void __launch_bounds__(kThreads, 1) qsa_prefill_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sp = smem_raw + (sb - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Sync sy;
  sy.bars = sb + OFF_BAR;
  sy.abort_flag = reinterpret_cast<volatile uint32_t*>(sp + OFF_MISC + 4);
  sy.status = p.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(sy.bar(B_FULL + s), 32 * kProducerWarps);
      mbar_init(sy.bar(B_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sy.bar(B_SFULL + b), 1);
      mbar_init(sy.bar(B_SFREE + b), 4);
      mbar_init(sy.bar(B_PFULL + b), 4);
      mbar_init(sy.bar(B_PEMPTY + b), 1);
      mbar_init(sy.bar(B_QFULL + b), 1);
      mbar_init(sy.bar(B_QEMPTY + b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sy.bar(B_RMAX + b), 4);
      mbar_init(sy.bar(B_RSUM + b), 4);
      if (b == 0) mbar_init(sy.bar(B_RMX2), 4);
    }
    mbar_init(sy.bar(B_OFULL), 1);
    mbar_init(sy.bar(B_OEMPTY), 4);
    mbar_init(sy.bar(B_DONE), 1);
    mbar_init(sy.bar(B_DONE + 1), 1);
    *sy.abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == kWarpProducer0 && lane == 0) prefetch_tensormap(&p.tm_q);
  if (warp == kWarpQK) {
    tmem_alloc(sb + OFF_MISC, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sp + OFF_MISC);

  if (warp < kWarpProducer0) {
    setmaxnreg_inc<kRegsSoftmax>();
    softmax_role<kBlocks>(p, sy, sb, sp, tmem, warp, lane);
  } else if (warp < kWarpQK) {
    setmaxnreg_dec<kRegsProducer>();
    producer_role<kDump, kStall, kBlocks>(p, sy, sb, warp - kWarpProducer0, lane);
  } else {
    setmaxnreg_dec<kRegsMma>();
    if (warp == kWarpQK) {
      if (lane == 0) qk_role(p, sy, sb, tmem);
    } else if (warp == kWarpPV) {
      if (lane == 0) pv_role(p, sy, sb, tmem);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpQK) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace qsa
