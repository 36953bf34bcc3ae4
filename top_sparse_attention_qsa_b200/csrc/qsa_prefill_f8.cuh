// qsa_prefill_f8.cuh -- QSA top-K sparse-attention prefill over an FP8 E4M3
// KV cache: tcgen05 kind::f8f6f4 kernel for sm_100a.
//
// The operation is the one of qsa_prefill_tc.cuh (page "Qwen4-Exp QSA llega
// al Ascend de Huawei", section "Lo que realmente añade la pull request"),
// with the cache elements stored as OCP FP8 E4M3 times a per-tensor scale
// (same page, the observations on the NVIDIA side: an fp8_e4m3 KV cache).
//
// The tensor cores read the cache tiles as they were gathered: one 32 KB ring
// slot holds a whole K or V tile (128 keys x 256 dims x 1 B), so six slots
// keep three tiles in flight, twice the BF16 kernel's 1.5.  Both MMA operands
// of kind::f8f6f4 are FP8, so the BF16 query and the FP32 probabilities are
// each written as a pair of E4M3 terms:
//   q * 2^a_h = q_hi + q_lo / 16     (a_h puts the head's largest |q| in
//                                     [128, 256); a BF16 value has 8
//                                     significant bits, each E4M3 term 4, so
//                                     the pair is exact for every element
//                                     of magnitude >= 2^-6 after scaling,
//                                     i.e. within about 2^13 of the head's
//                                     largest; smaller ones lose low bits to
//                                     E4M3's subnormal floor, an error below
//                                     2^-14 after scaling, 2^-21 of the
//                                     largest)
//   p         = p_hi + p_lo / 16     (8 significant bits, like the BF16 P of
//                                     the BF16 kernel; p <= 2^8 by the lazy
//                                     rescale)
// with separate TMEM accumulators for the two terms: S_hi, S_lo per score
// buffer and O_hi, O_lo per output half (two O buffers, by unit parity).  s = (S_hi + S_lo / 16) * 2^-a_h and
// o = (O_hi + O_lo / 16) * v_scale / l.  The N dimension of Q, S, P and O runs
// [hi of heads 0-7, lo of heads 0-7, hi of heads 8-15, lo of heads 8-15], so
// that a softmax thread's 8 heads of both terms are 16 adjacent TMEM columns
// and 16 adjacent bytes of P.
//
// Warps (persistent CTAs, one per SM):
//   warps 0-3   producers: list entries one tile ahead, 16-byte cp.async of
//               the 256-byte K and V rows into the 128-byte-swizzled K-major
//               layout (K slot, then V slot per tile)
//   warp 4      all lanes: the unit's Q (BF16, from global memory) split into
//               q_hi / q_lo rows of one E4M3 tile with per-head scale, one
//               unit ahead (double-buffered)
//   warp 5      lane 0 issues the score MMAs (A = K tile, B = [q_hi; q_lo];
//               M=128, N=32, K=32)
//   warp 6      lane 0 issues PV: [O_hi O_lo]^T += V^T (MN-major) .
//               [P_hi P_lo]^T (MN-major, N=32) for the two 128-dim halves,
//               into the O buffer of the unit's parity
//   warp 7      idle (keeps the softmax warpgroups aligned)
//   warps 8-15  softmax as in the BF16 kernel, two warps per TMEM lane
//               quadrant (8 heads each), reading both score terms and
//               writing p_hi / p_lo; at the end of a unit they hand l and m
//               to the epilogue warps through shared memory and go on
//   warps 16-19 epilogue: once the unit's last PV is done, O from TMEM
//               (the buffer then goes back to warp 6), normalised, stored
//               with lse -- the next unit's scores and softmax overlap it
// The warpgroups take their registers with setmaxnreg (kRegs*8 below).
// Every wait is bounded (2 s of %globaltimer) as in the BF16 kernel.
#pragma once

#include "qsa_prefill_tc.cuh"

namespace qsa {
namespace f8 {

using namespace tc;

constexpr int kSlots8 = 6;                    // 32 KB: one K or V tile
constexpr int kProducerWarps8 = 4;            // 32 rows of every tile each
constexpr int kQ8Bytes = kGp * 256;           // one E4M3 Q term: 16 heads x 256 dims
constexpr int kQ8Block = 2 * kGp * 128;       // one 128-dim block of both terms: 32 rows x 128 B
constexpr int kP8Bytes = kKeys * kGp;         // one E4M3 P term: 128 keys x 16 heads
constexpr int kTmemCols8 = 256;               // S: 2 buffers x {hi, lo} x 16; O: 2 units x 2 halves x {hi, lo} x 16
constexpr int kTS = 0, kTO = 64;              // TMEM column bases (O of unit parity b at kTO + 64 b)

constexpr int F_RING = 0;
constexpr int F_Q8 = F_RING + kSlots8 * kSlotBytes;   // 2 buffers x {hi, lo}
constexpr int F_P8 = F_Q8 + 2 * 2 * kQ8Bytes;         // 2 buffers x {hi, lo}
constexpr int F_QSC = F_P8 + 2 * 2 * kP8Bytes;        // 2 buffers x 16 per-head score factors
constexpr int F_RED = F_QSC + 2 * kGp * 4;            // max[4][16], votes[2][8], sum[2][4][16]
constexpr int F_LM = F_RED + 1024;                    // per unit parity: l[16], m[16] for the epilogue warps
constexpr int F_BAR = F_LM + 256;
constexpr int G_FULL = 0, G_EMPTY = 6, G_SFULL = 12, G_SFREE = 14, G_PFULL = 16, G_PEMPTY = 18,
              G_QFULL = 20, G_QEMPTY = 22, G_RMAX = 24, G_RSUM = 26, G_DONE = 28, G_RMX2 = 30,
              G_OFULL2 = 32, G_OEMPTY2 = 34, G_LFULL = 36, G_LEMPTY = 38, G_NUM = 40;
constexpr int F_MISC = F_BAR + G_NUM * 8;             // tmem base, abort flag
constexpr int F_SMEM = F_MISC + 16 + 1024;

// kind::f8f6f4: FP32 accumulator, E4M3 A and B (format 0), M = 128, N = 32:
// the hi and lo terms share one MMA (B rows / columns 0-15 hi, 16-31 lo).
constexpr uint32_t kIdescQK8 = (1u << 4) | (4u << 17) | (8u << 24);
// PV: both operands MN-major.
constexpr uint32_t kIdescPV8 = kIdescQK8 | (1u << 15) | (1u << 16);

// ------------------------------------------------------------------ producers

// kDump: also write, per key, the slot its K and V copies read (see the BF16
// kernel's producer).
template <bool kBlocks, bool kDump = false>
__device__ void producer8(const TcParams& p, const Sync& sy, uint32_t sb, int pw, int lane) {
  uint32_t c_slot = 0;
  const int64_t units = num_units(p);
  const int cc = lane & 15;                          // 16-byte chunk of the 256-byte row
  const int rsel = lane >> 4;                        // which of the two rows of an instruction
  const uint32_t dchunk = static_cast<uint32_t>((cc >> 3) * kBlockBytes);
  constexpr int rows_w = kKeys / kProducerWarps8;
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const int32_t* list = p.idx + un.t * p.idx_st + static_cast<int64_t>(un.g) * p.idx_sh;
    const int32_t last = kBlocks ? last_visible(p, un.t) : 0x7fffffff;
    const char* kbase = reinterpret_cast<const char*>(p.kraw) + static_cast<int64_t>(un.g) * p.kv_sh + cc * 16;
    const char* vbase = reinterpret_cast<const char*>(p.vraw) + static_cast<int64_t>(un.g) * p.kv_sh + cc * 16;
    const int64_t row_bytes = p.kv_ss;
    const int jr = rows_w * pw + lane;
    const bool own = lane < rows_w;
    int32_t entry_next = own ? key_entry<kBlocks>(p, list, un, jr) : -1;
    for (int i = 0; i < un.n_tiles && ok; ++i) {
      int32_t id = key_slot<kBlocks>(p, un, i * kKeys + jr, entry_next, last);
      entry_next = (own && i + 1 < un.n_tiles) ? key_entry<kBlocks>(p, list, un, (i + 1) * kKeys + jr) : -1;
      if (id == -2) {
        id = -1;
        if (p.status != nullptr) atomicOr(p.status, static_cast<int32_t>(kStatusOob));
      }
      int32_t from_k[kDump ? rows_w / 2 : 1];
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {                  // K tile, then V tile
        const uint32_t slot = c_slot % kSlots8;
        ok = sy.wait_warp(G_EMPTY + slot, ((c_slot / kSlots8) & 1u) ^ 1u);
        if (!ok) break;
        const char* src0 = h == 0 ? kbase : vbase;
        const uint32_t dst0 = sb + F_RING + slot * kSlotBytes + dchunk;
#pragma unroll
        for (int k = 0; k < rows_w / 2; ++k) {
          const int r = rows_w * pw + 2 * k + rsel;
          const int32_t rid = __shfl_sync(0xffffffffu, id, 2 * k + rsel);
          const bool live = rid >= 0;
          const char* src = live ? src0 + static_cast<int64_t>(rid) * row_bytes : src0;
          cp_async_16(dst0 + r * 128 + (((cc & 7) ^ (r & 7)) << 4), src, live ? 16 : 0);
          if (kDump && cc == 0) {
            const int32_t from = live ? static_cast<int32_t>((src - src0) / row_bytes) : -1;
            if (h == 0) {
              from_k[kDump ? k : 0] = from;
            } else {
              const int64_t key = un.j0 + static_cast<int64_t>(i) * kKeys + r;
              const int64_t n_keys = static_cast<int64_t>(p.K) << p.block_shift;
              if (key < n_keys)
                p.gathered[(un.t * p.Hkv + un.g) * n_keys + key] = from == from_k[kDump ? k : 0] ? from : -2;
            }
          }
        }
        cp_async_mbar_arrive(sy.bar(G_FULL + slot));
        ++c_slot;
      }
    }
  }
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// ------------------------------------------------------------------ Q split

// Lane l of warp 4 takes head l/2, dims [128*(l&1), +128): loads them from
// global memory, finds the head's largest |q| (with its partner lane), and
// writes q * 2^a = q_hi + q_lo / 16 as one E4M3 tile of 32 rows (K-major,
// 128-byte swizzle: two 128-dim blocks of 32 rows x 128 B; head h has its hi
// term in row 16 (h / 8) + h % 8 and its lo term 8 rows further) and
// 2^-a * scale_log2 into the
// score factors.  Heads past the group are zero.
__device__ __forceinline__ void q_split(const TcParams& p, const Unit& un, uint32_t qt, float* qsc, int lane) {
  const int h = lane >> 1, half = lane & 1;
  const bool live = h < p.G;
  const uint4* src = reinterpret_cast<const uint4*>(
      reinterpret_cast<const char*>(p.q_ptr) +
      (un.t * p.q_st + (static_cast<int64_t>(un.g) * p.G + (live ? h : 0)) * p.q_sh + half * 128) * 2);
  // first read: the head's largest |q| (BF16 bits widened; order = magnitude)
  uint32_t mx = 0u;
  if (live) {
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) mx = max(mx, max((w[j] << 16) & 0x7fffffffu, w[j] & 0x7fff0000u));
    }
  }
  mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  // a = 7 - floor(log2 max): the largest |q| * 2^a lands in [128, 256)
  int a = 0;
  if (mx != 0u) a = 7 - (static_cast<int>(mx >> 23) - 127);
  a = max(-126, min(a, 126));
  const float up = __int_as_float((127 + a) << 23);
  if (half == 0) qsc[h] = p.scale_log2 * __int_as_float((127 - a) << 23);
  // second read (cached): the two E4M3 terms, 16 dims per 16-byte chunk
#pragma unroll 2
  for (int c8 = 0; c8 < 8; ++c8) {
    const uint4 va = live ? __ldg(src + 2 * c8) : make_uint4(0u, 0u, 0u, 0u);
    const uint4 vb = live ? __ldg(src + 2 * c8 + 1) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t wv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // dims 4j..4j+3 of the chunk: BF16 words wv[2j], wv[2j+1]
      const uint32_t w0 = wv[2 * j], w1 = wv[2 * j + 1];
      const float x0 = __uint_as_float(w0 << 16) * up, x1 = __uint_as_float(w0 & 0xffff0000u) * up;
      const float x2 = __uint_as_float(w1 << 16) * up, x3 = __uint_as_float(w1 & 0xffff0000u) * up;
      const uint32_t h01 = pack_e4m3x2(x0, x1), h23 = pack_e4m3x2(x2, x3);
      float y0, y1, y2, y3;
      f16x2_to_f32(e4m3x2_to_f16x2(h01), y0, y1);
      f16x2_to_f32(e4m3x2_to_f16x2(h23), y2, y3);
      const uint32_t l01 = pack_e4m3x2((x0 - y0) * 16.f, (x1 - y1) * 16.f);
      const uint32_t l23 = pack_e4m3x2((x2 - y2) * 16.f, (x3 - y3) * 16.f);
      hw[j] = h01 | (h23 << 16);
      lw[j] = l01 | (l23 << 16);
    }
    // hi row 16 (h / 8) + h % 8 and lo row 8 further share the swizzle phase h % 8
    const uint32_t off = half * kQ8Block + ((h >> 3) * 16 + (h & 7)) * 128 + ((c8 ^ (h & 7)) << 4);
    st_shared_v4(qt + off, hw[0], hw[1], hw[2], hw[3]);
    st_shared_v4(qt + off + 8 * 128, lw[0], lw[1], lw[2], lw[3]);
  }
}

// ------------------------------------------------------------------ MMA issuers

// Warp 4: per unit all lanes split Q into buffer (unit & 1) once the MMAs of
// two units ago have released it; lane 0 then issues S_hi += K q_hi^T and
// S_lo += K q_lo^T for every tile.
// Warp 4: each unit's Q tile and score factors, one unit ahead of the MMAs
// (double-buffered), so that no unit waits for its Q to be read and split.
__device__ void q8(const TcParams& p, const Sync& sy, uint32_t sb, uint8_t* sp, int lane) {
  uint32_t c_unit = 0;
  const int64_t units = num_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t qb = c_unit & 1u;
    ok = sy.wait_warp(G_QEMPTY + qb, ((c_unit >> 1) & 1u) ^ 1u);
    if (!ok) break;
    ++c_unit;
    const uint32_t qt = sb + F_Q8 + qb * 2 * kQ8Bytes;
    if (un.n_tiles > 0) q_split(p, un, qt, reinterpret_cast<float*>(sp + F_QSC) + qb * kGp, lane);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(sy.bar(G_QFULL + qb));             // the MMAs and the softmax read it
      if (un.n_tiles == 0) mbar_arrive(sy.bar(G_QEMPTY + qb));
    }
  }
}

// Warp 5, lane 0: the score MMAs of every tile.
__device__ void qk8(const TcParams& p, const Sync& sy, uint32_t sb, uint32_t tmem) {
  uint32_t c_tile = 0, c_unit = 0;
  const int64_t units = num_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t qb = c_unit & 1u;
    if (un.n_tiles > 0) ok = sy.wait(G_QFULL + qb, (c_unit >> 1) & 1u);
    if (!ok) break;
    ++c_unit;
    const uint32_t qt = sb + F_Q8 + qb * 2 * kQ8Bytes;
    {
      for (int i = 0; i < un.n_tiles && ok; ++i, ++c_tile) {
        const uint32_t c = c_tile;
        const uint32_t sbuf = c & 1u;
        ok = sy.wait(G_SFREE + sbuf, ((c >> 1) & 1u) ^ 1u);
        const uint32_t ck = 2u * c;
        const uint32_t slot = ck % kSlots8;
        if (ok) ok = sy.wait(G_FULL + slot, (ck / kSlots8) & 1u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kt = sb + F_RING + slot * kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // K-major, 128-byte swizzle: a 32-dim step advances 32 B inside the
          // atom; dims 128-255 sit 16 KB (K) / 4 KB (Q) further.  N = 32,
          // columns in the interleaved hi / lo head order of the Q rows.
          const uint64_t a = smem_desc(kt + (kk >> 2) * kBlockBytes + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t b = smem_desc(qt + (kk >> 2) * kQ8Block + (kk & 3) * 32, 16, 1024, 2);
          umma_f8_ss(tmem + kTS + sbuf * 32, a, b, kIdescQK8, kk > 0 ? 1u : 0u);
        }
        umma_commit(sy.bar(G_EMPTY + slot));
        umma_commit(sy.bar(G_SFULL + sbuf));
        if (i == un.n_tiles - 1) umma_commit(sy.bar(G_QEMPTY + qb));
      }
    }
  }
  umma_commit(sy.bar(G_DONE));
  sy.drain(G_DONE, 0);
}

// Warp 5, lane 0: O_{hi,lo}[mh] += V_half(mh)^T . P_{hi,lo}^T per tile.
__device__ void pv8(const TcParams& p, const Sync& sy, uint32_t sb, uint32_t tmem) {
  uint32_t c_tile = 0, c_unit = 0;
  const int64_t units = num_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t ue = c_unit++;
    const uint32_t ob = ue & 1u;                     // O buffer of this unit
    ok = sy.wait(G_OEMPTY2 + ob, ((ue >> 1) & 1u) ^ 1u);
    if (!ok) break;
    if (un.n_tiles == 0) {
      mbar_arrive(sy.bar(G_OFULL2 + ob));
      continue;
    }
    for (int i = 0; i < un.n_tiles && ok; ++i, ++c_tile) {
      const uint32_t c = c_tile;
      const uint32_t pb = c & 1u;
      ok = sy.wait(G_PFULL + pb, (c >> 1) & 1u);
      const uint32_t cv = 2u * c + 1u;
      const uint32_t slot = cv % kSlots8;
      if (ok) ok = sy.wait(G_FULL + slot, (cv / kSlots8) & 1u);
      if (!ok) break;
      tc_fence_after();
      const uint32_t vt = sb + F_RING + slot * kSlotBytes;
      const uint32_t pt = sb + F_P8 + pb * 2 * kP8Bytes;
#pragma unroll
      for (int mh = 0; mh < 2; ++mh)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // A = V^T: MN-major, 128-byte swizzle; the 128 dims of a half are
          // one atom row, groups of 8 keys 1 KB apart, 32 keys per step
          const uint64_t a = smem_desc(vt + mh * kBlockBytes + kk * 4096, kBlockBytes, 1024, 2);
          // B = P^T: MN-major, no swizzle; per key one 16-byte core row
          // (hi then lo of heads 0-7), key groups of 8 128 B apart (LBO), and
          // one core-matrix column (SBO = 2 KB) further the same for heads
          // 8-15: O of the half lands in the same interleaved column order
          const uint64_t b = smem_desc(pt + kk * 512, 128, kP8Bytes, 0);
          umma_f8_ss(tmem + kTO + ob * 64 + mh * 32, a, b, kIdescPV8, (i == 0 && kk == 0) ? 0u : 1u);
        }
      umma_commit(sy.bar(G_EMPTY + slot));
      umma_commit(sy.bar(G_PEMPTY + pb));
    }
    if (ok) umma_commit(sy.bar(G_OFULL2 + ob));
  }
  umma_commit(sy.bar(G_DONE + 1));
  sy.drain(G_DONE + 1, 0);
}

// ------------------------------------------------------------------ softmax

constexpr int kSmWarps = 8;     // two per TMEM lane quadrant, 8 heads each
constexpr int kHpw = kGp / 2;   // heads per softmax warp
// warpgroups: producers, {Q, score MMA, PV MMA, idle}, softmax (two), epilogue
constexpr int kWarpQ8 = kProducerWarps8, kWarpQK8 = kProducerWarps8 + 1, kWarpPV8 = kProducerWarps8 + 2,
              kWarpSm8 = kProducerWarps8 + 4, kWarpEpi8 = kWarpSm8 + kSmWarps;
constexpr int kThreads8 = 32 * (kWarpEpi8 + 4);
// Registers per thread after setmaxnreg (the block is launched with 640 x 96):
// producers 80, Q / MMA warpgroup 64, softmax 128, epilogue 80:
// 80 + 64 + 2*128 + 80 = 480 = 5 * 96.
constexpr int kRegsProd8 = 80, kRegsMisc8 = 64, kRegsSm8 = 128, kRegsEpi8 = 80, kRegsLaunch8 = 96;
static_assert(kRegsProd8 + kRegsMisc8 + 2 * kRegsSm8 + kRegsEpi8 <= 5 * kRegsLaunch8, "register split");

// Reduce 8 per-lane values across the 32 lanes of a warp by exchanging halves
// (7 shuffles for the exchange, 2 for the rest).  Lane l ends with the result
// for value (l >> 2) & 7.
template <bool kMax>
__device__ __forceinline__ float xreduce8(const float (&v)[8], int lane) {
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[4], b[2];
  bool up = (lane & 16) != 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float send = up ? v[j] : v[4 + j];
    const float keep = up ? v[4 + j] : v[j];
    a[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
  up = (lane & 8) != 0;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float send = up ? a[j] : a[2 + j];
    const float keep = up ? a[2 + j] : a[j];
    b[j] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
  up = (lane & 4) != 0;
  float c = op(up ? b[1] : b[0], __shfl_xor_sync(0xffffffffu, up ? b[0] : b[1], 4));
  c = op(c, __shfl_xor_sync(0xffffffffu, c, 2));
  c = op(c, __shfl_xor_sync(0xffffffffu, c, 1));
  return c;
}

// p = 2^(s - m) for this thread's key and 8 heads as p = p_hi + p_lo / 16,
// both E4M3 (p <= 2^8), packed 4 heads per word; pv gets the p themselves.
__device__ __forceinline__ void form_p(const float (&s)[kHpw], const float (&m)[kHpw], uint32_t (&ph)[2],
                                       uint32_t (&plo)[2], float (&pv)[kHpw]) {
#pragma unroll
  for (int h4 = 0; h4 < 2; ++h4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int h = 4 * h4 + j;
      pv[h] = ex2(s[h] - (m[h] == -INFINITY ? 0.f : m[h]));
    }
    const float* x = pv + 4 * h4;
    const uint32_t h01 = pack_e4m3x2(x[0], x[1]), h23 = pack_e4m3x2(x[2], x[3]);
    float y0, y1, y2, y3;
    f16x2_to_f32(e4m3x2_to_f16x2(h01), y0, y1);
    f16x2_to_f32(e4m3x2_to_f16x2(h23), y2, y3);
    const uint32_t l01 = pack_e4m3x2((x[0] - y0) * 16.f, (x[1] - y1) * 16.f);
    const uint32_t l23 = pack_e4m3x2((x[2] - y2) * 16.f, (x[3] - y3) * 16.f);
    ph[h4] = h01 | (h23 << 16);
    plo[h4] = l01 | (l23 << 16);
  }
}

// Softmax warp w (8..15): TMEM lane quadrant q = w & 3 (thread = key of the
// tile), heads [8 hh, 8 hh + 8) with hh = (w-8)/4.
template <bool kBlocks>
__device__ void softmax8(const TcParams& p, const Sync& sy, uint32_t sb, uint8_t* sp, uint32_t tmem, int warp,
                         int lane) {
  const int wq = warp & 3;
  const int hh = (warp - kWarpSm8) >> 2;
  const int h0 = hh * kHpw;
  const int key = wq * 32 + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  float* red_max = reinterpret_cast<float*>(sp + F_RED);
  uint8_t* votes = sp + F_RED + 256;
  float* red_sum = red_max + 128;
  const float* qsc_all = reinterpret_cast<const float*>(sp + F_QSC);
  uint32_t c_tile = 0, c_unit = 0, c_exact = 0;
  uint32_t vote_par = 0u;                            // bit b: parity of the votes taken on score buffer b
  const int64_t units = num_units(p);
  const int G = p.G;
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const int32_t* list = p.idx + un.t * p.idx_st + static_cast<int64_t>(un.g) * p.idx_sh;
    const int32_t last = kBlocks ? last_visible(p, un.t) : 0x7fffffff;
    const uint32_t qb = c_unit & 1u;
    ok = sy.wait_warp(G_QFULL + qb, (c_unit >> 1) & 1u);
    if (!ok) break;
    float qs[kHpw];
#pragma unroll
    for (int h = 0; h < kHpw; ++h) qs[h] = qsc_all[qb * kGp + h0 + h];
    // the score factors are read: the Q buffer may be refilled once the MMAs
    // are done too (without this release, warp 4 could run two units ahead
    // through empty units and complete a G_QFULL phase this warp never saw)
    __syncwarp();
    if (lane == 0) mbar_arrive(sy.bar(G_QEMPTY + qb));
    float m_run[kHpw], l_part[kHpw];
#pragma unroll
    for (int h = 0; h < kHpw; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    int32_t entry_next = un.n_tiles > 0 ? key_entry<kBlocks>(p, list, un, key) : -1;
    for (int i = 0; i < un.n_tiles; ++i) {
      const uint32_t c = c_tile + i;
      const uint32_t buf = c & 1u;
      const bool valid = key_slot<kBlocks>(p, un, i * kKeys + key, entry_next, last) >= 0;
      entry_next = i + 1 < un.n_tiles ? key_entry<kBlocks>(p, list, un, (i + 1) * kKeys + key) : -1;
      ok = sy.wait_warp(G_SFULL + buf, (c >> 1) & 1u);
      if (!ok) break;
      tc_fence_after();
      uint32_t r16[16];                              // hi of this warp's 8 heads, then lo
      tmem_ld16(tl + kTS + buf * 32 + 16 * hh, r16);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(G_SFREE + buf));
      float s[kHpw];
      bool over = false;
#pragma unroll
      for (int h = 0; h < kHpw; ++h) {
        s[h] = (valid && h0 + h < G) ? fmaf(__uint_as_float(r16[8 + h]), 0.0625f, __uint_as_float(r16[h])) * qs[h]
                                     : -INFINITY;
        over |= s[h] > m_run[h] + kRescaleLog2;
      }
      // Most tiles hold no score above the running max plus the lazy-rescale
      // bound.  Each warp votes on that, then forms P from the running max
      // while the other warps' votes arrive; only a yes anywhere (a real
      // rescale) makes the warps combine the exact tile max and form P
      // again.  The first tile of a unit always takes that path (the
      // running max is -inf), without a vote; the votes of each score buffer
      // are counted apart, as the barrier's phases are.
      uint32_t ph[2], plo[2];
      float pv[kHpw];
      bool exact = true;
      if (i > 0) {
        const bool wover = __any_sync(0xffffffffu, over);
        uint8_t* vt = votes + buf * 8;
        if (lane == 0) vt[warp - kWarpSm8] = wover ? 1 : 0;
        __syncwarp();
        if (lane == 0) mbar_arrive(sy.bar(G_RMAX + buf));
        if (!wover) form_p(s, m_run, ph, plo, pv);
        ok = sy.wait_warp(G_RMAX + buf, (vote_par >> buf) & 1u);
        vote_par ^= 1u << buf;
        if (!ok) break;
        const uint2 vw = *reinterpret_cast<const uint2*>(vt);
        exact = (vw.x | vw.y) != 0u;
      }
      if (exact) {
        const float wmax = xreduce8<true>(s, lane);
        float* rm = red_max;
        if ((lane & 3) == 0) rm[wq * 16 + h0 + ((lane >> 2) & 7)] = wmax;
        __syncwarp();
        if (lane == 0) mbar_arrive(sy.bar(G_RMX2));
        ok = sy.wait_warp(G_RMX2, c_exact & 1u);
        ++c_exact;
        if (!ok) break;
        float tmax[kHpw];
#pragma unroll
        for (int h = 0; h < kHpw; ++h)
          tmax[h] = fmaxf(fmaxf(rm[h0 + h], rm[16 + h0 + h]), fmaxf(rm[32 + h0 + h], rm[48 + h0 + h]));
        bool need = false;
#pragma unroll
        for (int h = 0; h < kHpw; ++h)
          need |= (m_run[h] != -INFINITY) && (tmax[h] > m_run[h] + kRescaleLog2);
        if (need) {
          if (i > 0) {
            const uint32_t cp = c - 1;
            ok = sy.wait_warp(G_PEMPTY + (cp & 1u), (cp >> 1) & 1u);
            if (!ok) break;
          }
          tc_fence_after();
          float alpha[kHpw];
#pragma unroll
          for (int h = 0; h < kHpw; ++h) {
            const float mn = fmaxf(m_run[h], tmax[h]);
            alpha[h] = m_run[h] == -INFINITY ? 1.f : ex2(m_run[h] - mn);
            m_run[h] = mn;
            l_part[h] *= alpha[h];
          }
          if (i > 0) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {          // O_hi, O_lo x two halves, this warp's heads
              uint32_t o[8];
              const uint32_t col = kTO + (c_unit & 1u) * 64 + (q4 >> 1) * 32 + 16 * hh + (q4 & 1) * 8;
              tmem_ld8(tl + col, o);
              tmem_wait_ld();
#pragma unroll
              for (int h = 0; h < kHpw; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
              tmem_st8(tl + col, o);
            }
            tmem_wait_st();
          }
        } else {
#pragma unroll
          for (int h = 0; h < kHpw; ++h)
            if (m_run[h] == -INFINITY) m_run[h] = tmax[h];
        }
        form_p(s, m_run, ph, plo, pv);
      }
#pragma unroll
      for (int h = 0; h < kHpw; ++h) l_part[h] += pv[h];
      ok = sy.wait_warp(G_PEMPTY + buf, ((c >> 1) & 1u) ^ 1u);
      if (!ok) break;
      // P^T row of this key for this warp's 8 heads: p_hi then p_lo, 16 bytes
      // at 16 key in core-matrix column hh
      const uint32_t pa = sb + F_P8 + buf * 2 * kP8Bytes + hh * kP8Bytes + key * 16;
      st_shared_v4(pa, ph[0], ph[1], plo[0], plo[1]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(G_PFULL + buf));
    }
    if (!ok) break;
    const float wsum = xreduce8<false>(l_part, lane);
    float* rs = red_sum + (c_unit & 1u) * 64;
    if ((lane & 3) == 0) rs[wq * 16 + h0 + ((lane >> 2) & 7)] = wsum;
    __syncwarp();
    if (lane == 0) mbar_arrive(sy.bar(G_RSUM + (c_unit & 1u)));
    ok = sy.wait_warp(G_RSUM + (c_unit & 1u), (c_unit >> 1) & 1u);
    if (!ok) break;
    float l_tot[kHpw];
#pragma unroll
    for (int h = 0; h < kHpw; ++h)
      l_tot[h] = (rs[h0 + h] + rs[16 + h0 + h]) + (rs[32 + h0 + h] + rs[48 + h0 + h]);
    // hand l and m of the unit to the epilogue warps, which write the output
    // once the last PV is done, while these warps go on to the next unit
    const uint32_t lb = c_unit & 1u;
    if (wq == 0) {
      ok = sy.wait_warp(G_LEMPTY + lb, ((c_unit >> 1) & 1u) ^ 1u);
      if (!ok) break;
      float* lm = reinterpret_cast<float*>(sp + F_LM) + lb * 32;
      if (lane < kHpw) {
        float mk = 0.f, lk = 0.f;
#pragma unroll
        for (int h = 0; h < kHpw; ++h)
          if (h == lane) {
            mk = m_run[h];
            lk = l_tot[h];
          }
        lm[h0 + lane] = lk;
        lm[16 + h0 + lane] = mk;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(sy.bar(G_LFULL + lb));
    }
    c_tile += un.n_tiles;
    ++c_unit;
  }
}

// Epilogue warp w (16..19, TMEM lane quadrant w & 3: thread = dim of an
// output half): for every unit, l and m from the softmax warps, O from TMEM
// once the unit's last PV is done (the O buffer then goes back to the PV
// issuer), then o = (O_hi + O_lo / 16) * v_scale / l as BF16 rows (or the
// normalised partial output of a split-K chunk) and lse.
__device__ void epilogue8(const TcParams& p, const Sync& sy, uint8_t* sp, uint32_t tmem, int warp, int lane) {
  const int wq = warp & 3;
  const int key = wq * 32 + lane;
  const uint32_t tl = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  uint32_t c_unit = 0;
  const int64_t units = num_units(p);
  const int G = p.G;
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t ub = c_unit & 1u, par = (c_unit >> 1) & 1u;
    ++c_unit;
    ok = sy.wait_warp(G_LFULL + ub, par);
    if (!ok) break;
    const float* lm = reinterpret_cast<const float*>(sp + F_LM) + ub * 32;
    const int64_t row0 = un.t * static_cast<int64_t>(p.Hkv) * G + static_cast<int64_t>(un.g) * G;
    if (wq == 0 && lane < G && (p.lse != nullptr || p.part_lse != nullptr)) {
      const float lk = lm[lane], mk = lm[16 + lane];
      const float lv = lk > 0.f ? (mk + lg2(lk)) * 0.69314718055994531f : -INFINITY;
      if (p.part_lse != nullptr)
        p.part_lse[(row0 + lane) * p.splits + un.s] = lv;
      else
        p.lse[un.t * p.lse_st + static_cast<int64_t>(un.g) * G + lane] = lv;
    }
    float inv[kGp];
#pragma unroll
    for (int h = 0; h < kGp; ++h) inv[h] = lm[h] > 0.f ? p.o_scale / lm[h] : 0.f;
    __syncwarp();
    if (lane == 0) mbar_arrive(sy.bar(G_LEMPTY + ub));
    ok = sy.wait_warp(G_OFULL2 + ub, par);
    if (!ok) break;
    tc_fence_after();
    __nv_bfloat16* orow = p.out + un.t * p.o_st + static_cast<int64_t>(un.g) * G * p.o_sh;
#pragma unroll
    for (int q = 0; q < 4; ++q) {                   // O columns: half (q >> 1), heads 8 (q & 1) ..
      uint32_t o[16] = {};                          // hi of 8 heads, then lo of the same 8
      if (un.n_tiles > 0) {
        tmem_ld16(tl + kTO + ub * 64 + q * 16, o);
        tmem_wait_ld();
      }
      if (q == 3) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sy.bar(G_OEMPTY2 + ub));
      }
      const int dim = (q >> 1) * 128 + key;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int h = (q & 1) * 8 + j;
        if (h < G) {
          const float oh = fmaf(__uint_as_float(o[8 + j]), 0.0625f, __uint_as_float(o[j]));
          const float v = inv[h] != 0.f ? oh * inv[h] : 0.f;
          if (p.part_o != nullptr)
            p.part_o[((row0 + h) * p.splits + un.s) * 256 + dim] = v;
          else
            orow[h * p.o_sh + dim] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ kernel

template <bool kBlocks, bool kDump = false>
__global__ void __launch_bounds__(kThreads8, 1) qsa_prefill_f8_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* sp = smem_raw + (sb - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Sync sy;
  sy.bars = sb + F_BAR;
  sy.abort_flag = reinterpret_cast<volatile uint32_t*>(sp + F_MISC + 4);
  sy.status = p.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots8; ++s) {
      mbar_init(sy.bar(G_FULL + s), 32 * kProducerWarps8);
      mbar_init(sy.bar(G_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sy.bar(G_SFULL + b), 1);
      mbar_init(sy.bar(G_SFREE + b), kSmWarps);
      mbar_init(sy.bar(G_PFULL + b), kSmWarps);
      mbar_init(sy.bar(G_PEMPTY + b), 1);
      mbar_init(sy.bar(G_QFULL + b), 1);
      mbar_init(sy.bar(G_QEMPTY + b), 1 + kSmWarps);   // the MMAs, and each softmax warp
      mbar_init(sy.bar(G_RMAX + b), kSmWarps);
      mbar_init(sy.bar(G_RSUM + b), kSmWarps);
    }
    mbar_init(sy.bar(G_RMX2), kSmWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sy.bar(G_OFULL2 + b), 1);
      mbar_init(sy.bar(G_OEMPTY2 + b), 4);          // the epilogue warps
      mbar_init(sy.bar(G_LFULL + b), 2);            // the quadrant-0 softmax warps
      mbar_init(sy.bar(G_LEMPTY + b), 4);
    }
    mbar_init(sy.bar(G_DONE), 1);
    mbar_init(sy.bar(G_DONE + 1), 1);
    *sy.abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == kWarpQK8) {
    tmem_alloc(sb + F_MISC, kTmemCols8);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sp + F_MISC);

  if (warp < kProducerWarps8) {
    setmaxnreg_dec<kRegsProd8>();
    producer8<kBlocks, kDump>(p, sy, sb, warp, lane);
  } else if (warp < kWarpSm8) {
    setmaxnreg_dec<kRegsMisc8>();
    if (warp == kWarpQ8) {
      q8(p, sy, sb, sp, lane);
    } else if (warp == kWarpQK8) {
      if (lane == 0) qk8(p, sy, sb, tmem);
      __syncwarp();
    } else if (warp == kWarpPV8) {
      if (lane == 0) pv8(p, sy, sb, tmem);
      __syncwarp();
    }
  } else if (warp < kWarpEpi8) {
    setmaxnreg_inc<kRegsSm8>();
    softmax8<kBlocks>(p, sy, sb, sp, tmem, warp, lane);
  } else {
    setmaxnreg_dec<kRegsEpi8>();
    epilogue8(p, sy, sp, tmem, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpQK8) tmem_dealloc(tmem, kTmemCols8);
}

}  // namespace f8
}  // namespace qsa
