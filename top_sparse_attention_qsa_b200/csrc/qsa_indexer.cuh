// qsa_indexer.cuh -- QSA indexer scores (tcgen05) and top-K microblock
// selection for sm_100a.
//
// The operation (page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Por
// qué QSA es la parte incómoda, en cifras"): a multi-query indexer, H query
// heads per token (4 in the published configuration) sharing one key head of
// dim 128, over a key cache compressed 4x (one key per microblock of 4
// slots), picks a budget of microblocks (2048) per query token.  The page
// fixes the shapes only; this file computes
//   score(t, b) = sum_h <q_idx[t, h, :], k_idx[b, :]>        (FP32)
// for the complete causal microblocks b in [seq_start/bs, (pos+1)/bs) of
// token t, and selects the `budget` highest scores (ties to the smaller block
// index, -0.0 equal to +0.0) in ascending block order, optionally followed by
// the token's own incomplete block.
//
// Score kernel: persistent CTAs, one per SM, over units (64 tokens x up to 16
// block tiles of 128 blocks).  Swap-AB so that one TMEM lane is one block and
// the head sum stays inside a thread: D^T[128 blocks x 256 token-heads] =
// K_tile[128 x 128] . Q_tile[256 x 128]^T, kind::f16, M=128, N=256.
//   warp 0      TMA: the unit's Q tile once (3-d map, 64 KB, two buffers so
//               that the next unit's Q loads while this one's last MMAs
//               run), K tiles through a 2-stage ring (2-d map, 32 KB each;
//               the 8 MB key table stays in L2), 128-byte swizzle
//   warp 1      one thread issues the MMAs into a TMEM double buffer (2 x 256
//               FP32 columns)
//   warps 2-9   epilogue: thread = block row, two warps per TMEM lane quarter
//               (one per half of the token-head columns); 16-column TMEM loads,
//               head sums in FP32, coalesced stores into the tokens' rows,
//               masked only in tiles that straddle a token's candidate range
// Every mbarrier wait is bounded (2 s of %globaltimer, status bit 1).
//
// Top-K kernel: persistent CTAs; each row's candidate scores arrive in shared
// memory by a bulk copy issued while the previous row is processed, then sit
// in registers as order-preserving 32-bit keys; a 12/12/8-bit radix select
// over one shared histogram finds the threshold key and how many keys equal
// to it are taken; bitmaps and one packed block-wide scan give every chosen
// block its place in ascending order.
#pragma once

#include <cuda.h>

#include <climits>
#include <cstdint>

#include "qsa_ptx.cuh"
#include "qsa_tc_ptx.cuh"

namespace qsa {
namespace ix {

using namespace tc;

constexpr int kBlk = 128;                    // microblocks per tile (M)
constexpr int kRows = 256;                   // token-head rows per tile (N)
constexpr int kDh = 128;                     // indexer head dim
constexpr int kStages = 2;
constexpr int kTilesPerUnit = 16;            // block tiles per unit
constexpr int kKBytes = kBlk * kDh * 2;      // 32 KB
constexpr int kKHalf = kKBytes / 2;          // 128 rows x 64 dims
constexpr int kQBytes = kRows * kDh * 2;     // 64 KB
constexpr int kQHalf = kQBytes / 2;          // 256 rows x 64 dims
constexpr int kEpiWarps = 8;                 // two per TMEM lane quarter
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kTmemCols = 512;

constexpr int OFF_K = 0;
constexpr int OFF_Q = OFF_K + kStages * kKBytes;
constexpr int OFF_BAR = OFF_Q + 2 * kQBytes;            // two Q buffers
constexpr int B_KFULL = 0, B_KEMPTY = 4, B_QFULL = 8, B_TFULL = 10, B_TEMPTY = 12, B_DONE = 14,
              B_QEMPTY = 16, NUM_BARS = 18;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;       // tmem base, abort flag
constexpr int OFF_TOK = OFF_MISC + 16;                 // [8 warps][2][256] int32
constexpr int SMEM_BYTES = OFF_TOK + kEpiWarps * 2 * kRows * 4 + 1024;

// N = 256 (bits 17-22 hold N/8), M = 128 (bits 24-28 hold M/16), FP32
// accumulator, BF16 A and B, both K-major.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (32u << 17) | (8u << 24);

struct IxParams {
  CUtensorMap tm_k;        // k_idx [NB][128], box 64 dims x 128 blocks
  CUtensorMap tm_q;        // q_idx [T][H][128], box 64 dims x H heads x tpt tokens
  const int32_t* positions;
  const int32_t* seq_start;
  float* scores;           // [T][ld]
  int32_t* status;
  int64_t T, ld;
  int32_t NB, H, tpt, bs, n_chunks;
};

// Candidate blocks [lo, hi) of a token from its position and sequence
// start: the complete causal microblocks of its sequence (integer division
// truncating like C, clamped to [0, NB]).  Non-negative inputs take 32-bit
// unsigned divisions (pos + 1 <= 2^31).
__device__ __forceinline__ void range_of(int32_t pos, int32_t s0, int32_t NB, int32_t bs, int& lo, int& hi) {
  int64_t l, h;
  if ((pos | s0) >= 0) {
    l = static_cast<uint32_t>(s0) / static_cast<uint32_t>(bs);
    h = (static_cast<uint32_t>(pos) + 1u) / static_cast<uint32_t>(bs);
  } else {
    l = static_cast<int64_t>(s0) / bs;
    h = (static_cast<int64_t>(pos) + 1) / bs;
  }
  if (l < 0) l = 0;
  if (h > NB) h = NB;
  if (h < l) h = l;
  lo = static_cast<int>(l);
  hi = static_cast<int>(h);
}

// Shared-memory add of 1 at `addr` when a == b, without a branch.
__device__ __forceinline__ void red_add_if_eq(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, %1, %2;\n\t@p red.shared.add.u32 [%0], 1;\n\t}\n" ::"r"(addr),
      "r"(a), "r"(b)
      : "memory");
}

struct IxUnit {
  int64_t tok0;
  int tile0;
  int n_tiles;
  int full_lo, full_hi;  // blocks every token of the tile sees: [max lo, min hi)
};

// Unit u (token tile outer, chunk of block tiles inner) as seen by one warp:
// every lane returns the same tile range; with `lo_s` set, the candidate range
// of each of the tile's tokens is written there (tokens past T: empty).
// Every role calls this at each unit start, so it is kept short: a lane
// loads the positions and sequence starts of all its tokens (at most
// kRows / 32) before any arithmetic, paying one global-memory latency per
// unit, and the divisions are 32-bit wherever the values allow.
__device__ IxUnit ix_unit(const IxParams& p, int64_t u, int lane, int* lo_s, int* hi_s) {
  constexpr int kIt = kRows / 32;                  // tokens per lane at most (tpt <= kRows)
  IxUnit r;
  int64_t tt;
  int c;
  if (u <= 0xffffffffLL) {
    const uint32_t uu = static_cast<uint32_t>(u), nc = static_cast<uint32_t>(p.n_chunks);
    const uint32_t q = uu / nc;
    tt = q;
    c = static_cast<int>(uu - q * nc);
  } else {
    tt = u / p.n_chunks;
    c = static_cast<int>(u - tt * p.n_chunks);
  }
  r.tok0 = tt * p.tpt;
  int32_t pos[kIt], s0[kIt];
#pragma unroll
  for (int k = 0; k < kIt; ++k) {
    const int i = lane + 32 * k;
    const bool in = i < p.tpt && r.tok0 + i < p.T;
    pos[k] = in ? __ldg(p.positions + r.tok0 + i) : 0;
    s0[k] = in ? __ldg(p.seq_start + r.tok0 + i) : 0;
  }
  int mn = INT_MAX, mx = -1, flo = 0, fhi = INT_MAX;
#pragma unroll
  for (int k = 0; k < kIt; ++k) {
    const int i = lane + 32 * k;
    if (i >= p.tpt) break;
    int lo = 0, hi = 0;
    if (r.tok0 + i < p.T) range_of(pos[k], s0[k], p.NB, p.bs, lo, hi);
    if (lo_s != nullptr) {
      lo_s[i] = lo;
      hi_s[i] = hi;
    }
    if (hi > lo) {
      mn = min(mn, lo);
      mx = max(mx, hi);
    }
    flo = max(flo, lo);
    fhi = min(fhi, hi);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    flo = max(flo, __shfl_xor_sync(0xffffffffu, flo, o));
    fhi = min(fhi, __shfl_xor_sync(0xffffffffu, fhi, o));
  }
  r.full_lo = flo;
  r.full_hi = fhi;
  r.tile0 = 0;
  r.n_tiles = 0;
  if (mx > 0) {
    const int t_lo = max(mn / kBlk, c * kTilesPerUnit);
    const int t_hi = min((mx + kBlk - 1) / kBlk, (c + 1) * kTilesPerUnit);
    r.tile0 = t_lo;
    r.n_tiles = max(0, t_hi - t_lo);
  }
  return r;
}

__device__ __forceinline__ int64_t ix_units(const IxParams& p) {
  return ((p.T + p.tpt - 1) / p.tpt) * p.n_chunks;
}

__device__ void ix_producer(const IxParams& p, const Sync& sy, uint32_t sb, int lane) {
  uint32_t c_tile = 0, c_q = 0;
  const int64_t units = ix_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const IxUnit un = ix_unit(p, u, lane, nullptr, nullptr);
    if (un.n_tiles == 0) continue;
    if (lane == 0) {
      const uint32_t qb = c_q & 1u;
      ok = sy.wait(B_QEMPTY + qb, ((c_q >> 1) & 1u) ^ 1u);
      if (ok) {
        mbar_arrive_expect_tx(sy.bar(B_QFULL + qb), kQBytes);
        const int32_t t0 = static_cast<int32_t>(un.tok0);
        tc::tma_load_3d(sb + OFF_Q + qb * kQBytes, &p.tm_q, 0, 0, t0, sy.bar(B_QFULL + qb));
        tc::tma_load_3d(sb + OFF_Q + qb * kQBytes + kQHalf, &p.tm_q, 64, 0, t0, sy.bar(B_QFULL + qb));
        ++c_q;
      }
      for (int i = 0; i < un.n_tiles && ok; ++i, ++c_tile) {
        const uint32_t st = c_tile % kStages;
        ok = sy.wait(B_KEMPTY + st, ((c_tile / kStages) & 1u) ^ 1u);
        if (!ok) break;
        mbar_arrive_expect_tx(sy.bar(B_KFULL + st), kKBytes);
        const int32_t b0 = (un.tile0 + i) * kBlk;
        tc::tma_load_2d(sb + OFF_K + st * kKBytes, &p.tm_k, 0, b0, sy.bar(B_KFULL + st));
        tc::tma_load_2d(sb + OFF_K + st * kKBytes + kKHalf, &p.tm_k, 64, b0, sy.bar(B_KFULL + st));
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  }
  // no copy may still land in shared memory after the CTA ends: wait (bounded,
  // ignoring the abort flag) for the last load issued into every stage and Q
  if (lane == 0) {
    for (uint32_t c = c_tile > kStages ? c_tile - kStages : 0; c < c_tile; ++c)
      sy.drain(B_KFULL + c % kStages, (c / kStages) & 1u);
    for (uint32_t c = c_q > 2 ? c_q - 2 : 0; c < c_q; ++c) sy.drain(B_QFULL + (c & 1u), (c >> 1) & 1u);
  }
  __syncwarp();
}

__device__ void ix_mma(const IxParams& p, const Sync& sy, uint32_t sb, uint32_t tmem, int lane) {
  uint32_t c_tile = 0, c_q = 0;
  const int64_t units = ix_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const IxUnit un = ix_unit(p, u, lane, nullptr, nullptr);
    if (un.n_tiles == 0) continue;
    if (lane == 0) {
      const uint32_t qb = c_q & 1u;
      ok = sy.wait(B_QFULL + qb, (c_q >> 1) & 1u);
      ++c_q;
      for (int i = 0; i < un.n_tiles && ok; ++i, ++c_tile) {
        const uint32_t buf = c_tile & 1u;
        ok = sy.wait(B_TEMPTY + buf, ((c_tile >> 1) & 1u) ^ 1u);
        const uint32_t st = c_tile % kStages;
        if (ok) ok = sy.wait(B_KFULL + st, (c_tile / kStages) & 1u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t ka = sb + OFF_K + st * kKBytes;
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk) {
          // K-major, 128-byte swizzle, 8-row groups 1 KB apart; a 16-dim step
          // advances 32 B inside the swizzle atom, dims 64-127 in the second half
          const uint64_t a = smem_desc(ka + (kk >> 2) * kKHalf + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t b = smem_desc(sb + OFF_Q + qb * kQBytes + (kk >> 2) * kQHalf + (kk & 3) * 32, 16, 1024, 2);
          umma_f16_ss(tmem + buf * kRows, a, b, kIdesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(sy.bar(B_KEMPTY + st));
        umma_commit(sy.bar(B_TFULL + buf));
      }
      if (ok) umma_commit(sy.bar(B_QEMPTY + qb));
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  }
  if (lane == 0) {
    umma_commit(sy.bar(B_DONE));
    sy.drain(B_DONE, 0);
  }
  __syncwarp();
}

// Epilogue warp w (2..9): TMEM lanes 32*(w%4).. (blocks of the tile) and
// accumulator columns [128*h, 128*h + 128) with h = (w-2)/4 (token-heads).
template <int kH>
__device__ void ix_epilogue(const IxParams& p, const Sync& sy, uint8_t* sp, uint32_t tmem, int warp,
                            int lane) {
  constexpr int kCols = kRows / 2;                 // columns per warp
  constexpr int kTokPerLd = 16 / kH;               // tokens per 16-column load
  const int ew = warp - 2;
  const int quarter = warp & 3;
  const int half = ew >> 2;
  int* lo_s = reinterpret_cast<int*>(sp + OFF_TOK) + ew * 2 * kRows;
  int* hi_s = lo_s + kRows;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + half * kCols;
  const int tl0 = half * (kCols / kH);
  const int32_t ld32 = static_cast<int32_t>(p.ld);   // < 2^31 (checked by the host)
  uint32_t c_tile = 0;
  const int64_t units = ix_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    __syncwarp();
    const IxUnit un = ix_unit(p, u, lane, lo_s, hi_s);
    __syncwarp();
    for (int i = 0; i < un.n_tiles; ++i, ++c_tile) {
      const uint32_t buf = c_tile & 1u;
      ok = sy.wait(B_TFULL + buf, (c_tile >> 1) & 1u);
      if (!ok) break;
      tc_fence_after();
      const int b0 = (un.tile0 + i) * kBlk;
      const int b = b0 + quarter * 32 + lane;
      // every token of the tile sees every block of this tile: no masks
      const bool full = b0 >= un.full_lo && b0 + kBlk <= un.full_hi;
      float* d = p.scores + (un.tok0 + tl0) * p.ld + b;
#pragma unroll 1
      for (int j0 = 0; j0 < kCols / 16; j0 += 4) {
        uint32_t v[4][16];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) tmem_ld16(t_lane + buf * kRows + (j0 + jj) * 16, v[jj]);
        tmem_wait_ld();
        float* dj = d + static_cast<int64_t>(j0 * kTokPerLd) * ld32;
        if (full) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int tk = 0; tk < kTokPerLd; ++tk) {
              float s = __uint_as_float(v[jj][tk * kH]);
#pragma unroll
              for (int h = 1; h < kH; ++h) s += __uint_as_float(v[jj][tk * kH + h]);
              dj[static_cast<int64_t>(jj * kTokPerLd + tk) * ld32] = s;
            }
        } else {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int tk = 0; tk < kTokPerLd; ++tk) {
              float s = __uint_as_float(v[jj][tk * kH]);
#pragma unroll
              for (int h = 1; h < kH; ++h) s += __uint_as_float(v[jj][tk * kH + h]);
              const int tl = tl0 + (j0 + jj) * kTokPerLd + tk;
              const bool live = b >= lo_s[tl] && b < hi_s[tl];
              if (live) dj[static_cast<int64_t>(jj * kTokPerLd + tk) * ld32] = s;
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(B_TEMPTY + buf));
    }
  }
}

template <int kH>
__global__ void __launch_bounds__(kThreads, 1) qsa_indexer_scores_kernel(const __grid_constant__ IxParams p) {
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
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sy.bar(B_KFULL + s), 1);
      mbar_init(sy.bar(B_KEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sy.bar(B_QFULL + b), 1);
      mbar_init(sy.bar(B_QEMPTY + b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sy.bar(B_TFULL + b), 1);
      mbar_init(sy.bar(B_TEMPTY + b), kEpiWarps);
    }
    mbar_init(sy.bar(B_DONE), 1);
    *sy.abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_q);
  }
  if (warp == 1) {
    tmem_alloc(sb + OFF_MISC, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sp + OFF_MISC);

  if (warp == 0)
    ix_producer(p, sy, sb, lane);
  else if (warp == 1)
    ix_mma(p, sy, sb, tmem, lane);
  else
    ix_epilogue<kH>(p, sy, sp, tmem, warp, lane);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------ head folding

// The score is linear in the query, sum_h <q[t,h], k[b]> = <sum_h q[t,h], k[b]>,
// so the H indexer heads of a token can be summed once per token instead of
// once per (token, block).  The FP32 head sum s of each dim (heads added in
// order 0..H-1) is stored as two BF16 terms, hi = bf16(s) and
// lo = bf16(s - hi) (round to nearest; s - hi is exact in FP32; BF16 keeps
// 8 significant bits, so each rounding is within 2^-8), so
// |s - hi - lo| <= 2^-16 |s|; the score kernel then takes (hi, lo) as a
// query of two heads, which halves its tensor-core work and its accumulator
// reads.  One thread per (token, 8-dim chunk): H 16-byte loads, two 16-byte
// stores into folded[t][0..1][128].
struct FoldParams {
  const __nv_bfloat16* q;     // [T][H][128], strides in elements (multiples of 8)
  __nv_bfloat16* folded;      // [T][2][128] contiguous
  int64_t T, q_st, q_sh;
};

template <int kH>
__global__ void __launch_bounds__(256) qsa_indexer_fold_kernel(const __grid_constant__ FoldParams p) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= p.T * 16) return;
  const int64_t t = i >> 4;
  const int c = static_cast<int>(i & 15);
  float s[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] = 0.f;
#pragma unroll
  for (int h = 0; h < kH; ++h) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.q + t * p.q_st + h * p.q_sh + c * 8));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s[2 * e] += __uint_as_float(w[e] << 16);
      s[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
    }
  }
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(s[2 * e], s[2 * e + 1]);
    const float2 hf = __bfloat1622float2(h2);
    const __nv_bfloat162 l2 = __floats2bfloat162_rn(s[2 * e] - hf.x, s[2 * e + 1] - hf.y);
    hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
    lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
  }
  uint4* dst = reinterpret_cast<uint4*>(p.folded + t * 256 + c * 8);
  dst[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  dst[16] = make_uint4(lo[0], lo[1], lo[2], lo[3]);        // 128 elements further
}

// ------------------------------------------------------------------ top-K

struct TopkParams {
  const float* scores;       // [T][ld], 16-byte aligned, ld % 4 == 0
  const int32_t* positions;
  const int32_t* seq_start;
  int32_t* lists;            // [T][list_st], `width` entries written per row
  int32_t* n_valid;          // [T][copies] or nullptr
  int32_t* status;           // bit 1 on a timed-out row copy, or nullptr
  int64_t T, ld, list_st;
  int32_t NB, bs, budget, width, copies, append_tail;
};

// Order-preserving key: a > b as floats  <=>  key(a) > key(b) as unsigned,
// with -0.0 and +0.0 on the same key.  A negative float u maps to ~u, a
// positive one to (u | 2^31) - 1: both zeros land on 0x7fffffff and every
// other order is kept; -inf maps to 0x007fffff and only the negative NaN
// 0xffffffff to 0.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  const uint32_t sgn = static_cast<uint32_t>(static_cast<int32_t>(u) >> 31);   // 0 or ~0
  return (u ^ (sgn | 0x80000000u)) + ~sgn;
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

constexpr int kTkThreads = 512;
constexpr int kTkMax = 32768;                      // candidates per row
constexpr int kTkSlots = 16;                       // threshold-bin list entries per thread
constexpr int TK_OFF_ROW = 0;                      // row copy, 16-byte aligned span
constexpr int TK_OFF_HIST = ((kTkMax + 4) * 4 + 127) / 128 * 128;
constexpr int TK_OFF_GT = TK_OFF_HIST + 2 * 4096 * 4;  // two histograms, then the bitmaps
constexpr int TK_OFF_EQ = TK_OFF_GT + kTkMax / 8;
constexpr int TK_OFF_LK = TK_OFF_EQ + kTkMax / 8;  // per-thread lists: keys, then candidate ids
constexpr int TK_OFF_LE = TK_OFF_LK + kTkSlots * kTkThreads * 4;
constexpr int TK_OFF_MISC = TK_OFF_LE + kTkSlots * kTkThreads * 2;  // warp totals[16], results[4], mbarrier
constexpr int TK_SMEM = TK_OFF_MISC + 256;

// Persistent CTAs (one per SM) walk the rows t = blockIdx.x + i * gridDim.x.
// Thread 0 copies the next row's candidate scores into shared memory with
// one bulk copy (cp.async.bulk, completion on an mbarrier) while the CTA
// works on the current row from registers: candidate e = j * 512 + tid
// (j < kR) sits in a register of thread tid as its order-preserving key.
// Radix select over key bits 31-20, 19-8 and 7-0 with 4096-bin shared
// histograms (12 bits spread the few exponent values of real scores over
// many bins, which keeps the shared atomics nearly conflict-free); after
// each pass `prefix` and `mask` name the bin that holds the budget-th
// largest key and `need` how many keys of that bin are still to take; a pass
// that finds the whole bin taken ends the search.  The first pass counts
// the keys as they come out of the row copy.
// One sweep over the keys then writes the bitmap of the keys above the
// threshold bin (one warp ballot is one word) and appends the few keys in
// that bin (a few percent of the row for any smooth score distribution) to
// a per-thread list in shared memory, so that the remaining passes and the
// in-bin decisions touch only the list; each chosen list entry then sets its
// bit in the "above" or the "tied" bitmap.  A row whose bin does not fit the
// lists (heavy ties) finishes the same passes over the register keys
// instead.  Keys above the final bin are all taken, keys in it in block
// order until `need` runs out: one packed scan of the two bitmaps' word
// popcounts places every chosen block in ascending order.
template <int kR>
__global__ void __launch_bounds__(kTkThreads, 1) qsa_topk_kernel(const __grid_constant__ TopkParams p) {
  constexpr int kNT = kTkThreads, kW = kNT / 32;
  static_assert(kR % 32 == 0 && kR * kNT <= kTkMax, "bitmap words per thread = kR / 32");
  static_assert(kR * kNT <= 65536, "list candidate ids are 16-bit");
  constexpr int kWords = kR * kW;                   // bitmap words in use
  constexpr int kWPer = kWords / kNT;               // words per thread
  constexpr int kBins = 4096, kBinsPer = kBins / kNT;
  constexpr int kCap = kTkSlots;
  extern __shared__ __align__(128) uint8_t tk_smem[];
  const float* row_s = reinterpret_cast<const float*>(tk_smem + TK_OFF_ROW);
  uint32_t* hist = reinterpret_cast<uint32_t*>(tk_smem + TK_OFF_HIST);
  uint32_t* gtw = reinterpret_cast<uint32_t*>(tk_smem + TK_OFF_GT);
  uint32_t* eqw = reinterpret_cast<uint32_t*>(tk_smem + TK_OFF_EQ);
  uint32_t* wtot = reinterpret_cast<uint32_t*>(tk_smem + TK_OFF_MISC);
  volatile uint32_t* shv = reinterpret_cast<volatile uint32_t*>(tk_smem + TK_OFF_MISC + 64);
  const uint32_t row_addr = smem_u32(tk_smem + TK_OFF_ROW);
  const uint32_t bar = smem_u32(tk_smem + TK_OFF_MISC + 128);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this thread's list: entry i at [i * kNT] (consecutive threads, consecutive words)
  uint32_t* lk = reinterpret_cast<uint32_t*>(tk_smem + TK_OFF_LK) + tid;
  uint16_t* le = reinterpret_cast<uint16_t*>(tk_smem + TK_OFF_LE) + tid;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();

  // thread 0: start the copy of row t's candidate span [lo, hi) widened to
  // 16-byte boundaries, or complete the phase at once when nothing is read
  auto issue = [&](int64_t t, int lo, int hi) {
    if (min(hi - lo, p.budget) <= 0) {
      mbar_arrive(bar);
      return;
    }
    const int64_t a0 = (t * p.ld + lo) & ~int64_t(3), a1 = (t * p.ld + hi + 3) & ~int64_t(3);
    const uint32_t bytes = static_cast<uint32_t>(a1 - a0) * 4u;
    mbar_arrive_expect_tx(bar, bytes);
    for (uint32_t off = 0; off < bytes; off += 32768u)
      bulk_copy_g2s(row_addr + off, p.scores + a0 + off / 4, min(32768u, bytes - off), bar);
  };

  // The bin of histogram hb (bins high to low) that holds the need-th
  // largest counted key: its index, the count above it and its own count.
  // Thread i owns bins 4095 - i*kBinsPer .. ; warps in thread order cover the
  // bins from the top.  Two CTA barriers; hb may be cleared after it.
  auto find_bin = [&](const uint32_t* hb, int need, uint32_t& d, uint32_t& above, uint32_t& cnt) {
    uint32_t c[kBinsPer], own = 0u;
#pragma unroll
    for (int i = 0; i < kBinsPer; ++i) {
      c[i] = hb[kBins - 1 - tid * kBinsPer - i];
      own += c[i];
    }
    uint32_t x = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wtot[warp] = x;
    __syncthreads();
    uint32_t before = 0u;
    for (int w = 0; w < warp; ++w) before += wtot[w];
    const uint32_t incl = before + x, excl = incl - own;
    if (excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl) {
      uint32_t cum = excl;
#pragma unroll
      for (int i = 0; i < kBinsPer; ++i) {
        if (cum + c[i] >= static_cast<uint32_t>(need)) {
          shv[0] = kBins - 1u - tid * kBinsPer - i;
          shv[1] = cum;
          shv[3] = c[i];
          break;
        }
        cum += c[i];
      }
    }
    __syncthreads();
    d = shv[0];
    above = shv[1];
    cnt = shv[3];
  };

  uint32_t it = 0;
  bool pending = false;
  // position and sequence start of the next row, loaded a row ahead so that
  // their latency hides behind the current row
  int32_t npos = 0, ns0 = 0;
  if (blockIdx.x < p.T) {
    npos = __ldg(p.positions + blockIdx.x);
    ns0 = __ldg(p.seq_start + blockIdx.x);
    if (tid == 0) {
      int l0, h0;
      range_of(npos, ns0, p.NB, p.bs, l0, h0);
      issue(blockIdx.x, l0, h0);
      pending = true;
    }
  }
  for (int64_t t = blockIdx.x; t < p.T; t += gridDim.x, ++it) {
    const int32_t pos_t = npos;
    int lo, hi;
    range_of(npos, ns0, p.NB, p.bs, lo, hi);
    const int n = hi - lo;
    const int k = min(n, p.budget);
    const int64_t tn = t + gridDim.x;
    if (tn < p.T) {
      npos = __ldg(p.positions + tn);
      ns0 = __ldg(p.seq_start + tn);
    }
    if (tid == 0) {
      bool done = mbar_try_wait(bar, it & 1u);
      const uint64_t t0 = globaltimer_ns();
      while (!done && globaltimer_ns() - t0 < 2000000000ull) done = mbar_try_wait(bar, it & 1u);
      if (done) pending = false;
      else if (p.status != nullptr) atomicOr(p.status, 2);
      shv[2] = done ? 1u : 0u;
    }
#pragma unroll
    for (int i = 0; i < kBinsPer; ++i) hist[i * kNT + tid] = 0u;   // first pass's histogram
    __syncthreads();
    if (shv[2] == 0u) break;
    int32_t* out = p.lists + t * p.list_st;
    const int off = static_cast<int>((t * p.ld + lo) & 3);
    const int jn = n > tid ? (n - tid + kNT - 1) / kNT : 0;
    // key 0 marks "no candidate": a real score's key is at least 0x007fffff
    // (-inf), so 0 shares histogram bin 0 only with negative NaNs and never
    // reaches the selection threshold while n > k (it also sorts after every
    // real candidate in block order)
    // (reads past n stay inside the buffer, which holds kTkMax + 4 floats)
    const int jv = k > 0 ? jn : 0;
    const bool select = n > k;                         // else every candidate is taken
    uint32_t key[kR];
    if (select) {
      // the first radix pass counts bits 31-20 as the keys come in
#pragma unroll
      for (int j = 0; j < kR; ++j) {
        const uint32_t kk = order_key(row_s[off + j * kNT + tid]);
        key[j] = j < jv ? kk : 0u;
        atomicAdd(&hist[key[j] >> 20], 1u);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kR; ++j) {
        const uint32_t kk = order_key(row_s[off + j * kNT + tid]);
        key[j] = j < jv ? kk : 0u;
      }
    }
#pragma unroll
    for (int i = 0; i < kBinsPer; ++i) hist[kBins + i * kNT + tid] = 0u;   // the second pass's
    __syncthreads();                                   // the row buffer is free again
    if (tid == 0 && tn < p.T) {
      int l1, h1;
      range_of(npos, ns0, p.NB, p.bs, l1, h1);
      fence_proxy_async_smem();
      issue(tn, l1, h1);
      pending = true;
    }

    // bitmaps from the register keys: word j*kW + warp, bit lane =
    // candidate j*kNT + warp*32 + lane (each path below that still holds the
    // keys calls it last, so that no key outlives it)
    auto key_bitmaps = [&](uint32_t mask, uint32_t prefix) {
#pragma unroll
      for (int j = 0; j < kR; ++j) {
        const uint32_t km = key[j] & mask;
        const uint32_t bg = __ballot_sync(0xffffffffu, km > prefix);
        const uint32_t be = __ballot_sync(0xffffffffu, km == prefix);
        if (lane == 0) {
          gtw[j * kW + warp] = bg;
          eqw[j * kW + warp] = be;
        }
      }
    };

    if (k > 0) {
      // every candidate is taken when n <= k: all keys > 1, none equal
      uint32_t prefix = 1u, mask = 0xffffffffu;
      int need = 0;
      if (!select) {
        key_bitmaps(mask, prefix);
      } else {
        uint32_t d, above, cnt;
        find_bin(hist, k, d, above, cnt);
        need = k - static_cast<int>(above);
        prefix = d << 20;
        mask = 0xfff00000u;
        if (static_cast<uint32_t>(need) != cnt) {
          // one sweep: the "above" bitmap, and the bin's keys into the lists
          // (an entry past the last slot overwrites it; such a row takes the
          // fallback below)
          uint32_t nl = 0u;                            // this thread's list length
#pragma unroll
          for (int j = 0; j < kR; ++j) {
            const uint32_t b = key[j] >> 20;
            const uint32_t bg = __ballot_sync(0xffffffffu, b > d);
            if (lane == 0) gtw[j * kW + warp] = bg;
            if (b == d) {
              const uint32_t slot = min(nl, static_cast<uint32_t>(kCap - 1));
              lk[slot * kNT] = key[j];
              le[slot * kNT] = static_cast<uint16_t>(j * kNT + warp * 32 + lane);
              ++nl;
            }
          }
#pragma unroll
          for (int i = 0; i < kWPer; ++i) eqw[tid * kWPer + i] = 0u;
#pragma unroll
          for (int i = 0; i < kBinsPer; ++i) hist[i * kNT + tid] = 0u;   // the third pass's
          if (!__syncthreads_or(nl > static_cast<uint32_t>(kCap))) {
            // bits 19-8, then 7-0, of the listed keys
            for (uint32_t i = 0; i < nl; ++i) atomicAdd(&hist[kBins + ((lk[i * kNT] >> 8) & 0xfffu)], 1u);
            __syncthreads();
            find_bin(hist + kBins, need, d, above, cnt);
            need -= static_cast<int>(above);
            prefix |= d << 8;
            mask |= 0xfffu << 8;
            if (static_cast<uint32_t>(need) != cnt) {
              const uint32_t hbase = smem_u32(hist);
              for (uint32_t i = 0; i < nl; ++i) {
                const uint32_t kk = lk[i * kNT];
                red_add_if_eq(hbase + 4u * (kk & 0xffu), kk & mask, prefix);
              }
              __syncthreads();
              find_bin(hist, need, d, above, cnt);
              need -= static_cast<int>(above);
              prefix |= d;
              mask = 0xffffffffu;
            }
            // chosen list entries into the two bitmaps
            for (uint32_t i = 0; i < nl; ++i) {
              const uint32_t km = lk[i * kNT] & mask;
              const uint32_t e = le[i * kNT];
              if (km > prefix) atomicOr(&gtw[e >> 5], 1u << (e & 31u));
              else if (km == prefix) atomicOr(&eqw[e >> 5], 1u << (e & 31u));
            }
          } else {
            // heavy ties: the last two passes and the bitmaps over the
            // row's keys read again from global memory (the registers are
            // free by now, and the row has just been read, so it sits in L2)
            const float* srow = p.scores + t * p.ld + lo;
            auto gkey = [&](int j) -> uint32_t {
              const int e = j * kNT + tid;
              return e < n ? order_key(__ldg(srow + e)) : 0u;
            };
#pragma unroll 1
            for (int pass = 1; pass < 3; ++pass) {
              const int shift = pass == 1 ? 8 : 0;
              const uint32_t dmask = pass == 2 ? 0xffu : 0xfffu;
              uint32_t* hb = hist + (pass & 1) * kBins;   // both cleared before the sweep's barrier
              const uint32_t hbase = smem_u32(hb);
#pragma unroll 4
              for (int j = 0; j < kR; ++j) {
                const uint32_t kk = gkey(j);
                red_add_if_eq(hbase + 4u * ((kk >> shift) & dmask), kk & mask, prefix);
              }
              __syncthreads();
              find_bin(hb, need, d, above, cnt);
              need -= static_cast<int>(above);
              prefix |= d << shift;
              mask |= dmask << shift;
              if (static_cast<uint32_t>(need) == cnt) break;   // the whole bin is taken
            }
#pragma unroll 4
            for (int j = 0; j < kR; ++j) {
              const uint32_t km = gkey(j) & mask;
              const uint32_t bg = __ballot_sync(0xffffffffu, km > prefix);
              const uint32_t be = __ballot_sync(0xffffffffu, km == prefix);
              if (lane == 0) {
                gtw[j * kW + warp] = bg;
                eqw[j * kW + warp] = be;
              }
            }
          }
        } else {
          key_bitmaps(mask, prefix);                   // the whole bin is taken
        }
      }
      __syncthreads();
      // packed (above, in-bin) counts of the words before each word (each
      // half stays below 2^16: at most 32768 candidates)
      uint32_t loc[kWPer], run = 0u;
#pragma unroll
      for (int i = 0; i < kWPer; ++i) {
        const int w = tid * kWPer + i;
        loc[i] = run;
        run += (static_cast<uint32_t>(__popc(gtw[w])) << 16) | __popc(eqw[w]);
      }
      uint32_t x = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) wtot[warp] = x;
      __syncthreads();
      uint32_t base = x - run;
      for (int w = 0; w < warp; ++w) base += wtot[w];
#pragma unroll
      for (int i = 0; i < kWPer; ++i) {
        const int w = tid * kWPer + i;
        const uint32_t before = base + loc[i];
        const int gb = static_cast<int>(before >> 16), eb = static_cast<int>(before & 0xffffu);
        const uint32_t g = gtw[w], e = eqw[w];
        // in-bin candidates are taken in block order while need lasts
        uint32_t esel = 0u;
        const int take = need - eb;
        if (take > 0) {
          esel = e;
          while (__popc(esel) > take) esel &= ~(1u << (31 - __clz(esel)));
        }
        uint32_t sel = g | esel;
        while (sel != 0u) {
          const int bit = __ffs(sel) - 1;
          const uint32_t below = (1u << bit) - 1u;
          const int pos = gb + __popc(g & below) + min(eb + __popc(e & below), need);
          out[pos] = lo + w * 32 + bit;
          sel &= sel - 1u;
        }
      }
    }
    // causal tail, padding, counts
    int cnt = k;
    bool tail;
    int32_t tail_blk;
    if (pos_t >= 0) {
      // pos / bs == (pos + 1) / bs whenever bs does not divide pos + 1
      const uint32_t p1 = static_cast<uint32_t>(pos_t) + 1u, q1 = p1 / static_cast<uint32_t>(p.bs);
      tail = p.append_tail != 0 && q1 * static_cast<uint32_t>(p.bs) != p1;
      tail_blk = static_cast<int32_t>(q1);
    } else {
      const int64_t pos = pos_t;
      tail = p.append_tail != 0 && (pos + 1) % p.bs != 0;
      tail_blk = static_cast<int32_t>(pos / p.bs);
    }
    if (tail) {
      if (tid == 0) out[k] = tail_blk;
      ++cnt;
    }
    for (int j = cnt + tid; j < p.width; j += kNT) out[j] = -1;
    if (p.n_valid != nullptr && tid < p.copies) p.n_valid[t * p.copies + tid] = cnt;
  }
  // after a timed-out wait, give the copy in flight a bounded chance to land
  if (tid == 0 && pending) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, it & 1u) && globaltimer_ns() - t0 < 2000000000ull) {
    }
  }
}

}  // namespace ix
}  // namespace qsa
