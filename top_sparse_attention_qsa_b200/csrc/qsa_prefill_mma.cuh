// qsa_prefill_mma.cuh -- QSA top-K sparse-attention prefill, warp-MMA kernel.
//
// Computes, for one (query token t, KV head g) per CTA, attention of the G
// query heads of that group over the cache rows named by the token's
// selected-slot list (page "Qwen4-Exp QSA llega al Ascend de Huawei",
// section "Lo que realmente añade la pull request": softmax(scale Q K_sel^T)
// V_sel with the D256 scale; bullet "Límites de tamaño": -1 padding, fully
// masked rows give zeros).
//
// Per 64-entry tile of the list:
//   gather   64 K rows + 64 V rows (512 B each) with 16-byte cp.async, one
//            row per warp instruction, into a 3-stage XOR-swizzled ring;
//            masked entries are zero-filled without a global read.
//   scores   S^T[64 keys x Gp heads] = K_tile . Q^T on mma.sync m16n8k16
//            (keys in M so that a small head group only pads N to 8 or 16).
//   softmax  running max / sum per head in the log2 domain; the tile max
//            is combined across the 4 warps through shared memory.
//   PV       O^T[256 x Gp] += V_tile^T . P^T, each warp owning 64 rows of D.
// Epilogue: O / l rounded to BF16, lse = m + ln l, exact zeros for empty rows.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "qsa_ptx.cuh"

namespace qsa {

struct PrefillParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* idx;
  const int32_t* n_valid;
  __nv_bfloat16* out;
  float* lse;
  int32_t* status;
  int32_t* gathered;  // debug dump [T, Hkv, K] or nullptr
  int64_t T;
  int32_t Hkv, G, K;
  int64_t S;
  int64_t q_st, q_sh, kv_ss, kv_sh, idx_st, idx_sh, o_st, o_sh, lse_st;
  float scale_log2;  // softmax scale * log2(e)
};

constexpr int kHeadDim = 256;
constexpr int kRowBytes = kHeadDim * 2;  // one cache row, BF16
constexpr int kRowChunks = kRowBytes / 16;

template <int NT>  // padded group size Gp = 8 * NT
struct MmaCfg {
  static constexpr int BK = 64;       // list entries per tile
  static constexpr int STAGES = 3;    // gather ring depth
  static constexpr int WARPS = 4;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int GP = 8 * NT;
  static constexpr int P_STRIDE = BK + 8;  // P row pitch in BF16 (144 B: ldmatrix conflict-free)
  static constexpr int KV_TILE = BK * kRowBytes;
  static constexpr int STAGE_BYTES = 2 * KV_TILE;
  static constexpr int OFF_Q = STAGES * STAGE_BYTES;
  static constexpr int OFF_P = OFF_Q + GP * kRowBytes;
  static constexpr int OFF_RED = OFF_P + GP * P_STRIDE * 2;
  static constexpr int OFF_IDS = OFF_RED + WARPS * GP * 4;
  static constexpr int SMEM = OFF_IDS + STAGES * BK * 4;
  static_assert(GP * kRowBytes <= STAGE_BYTES, "epilogue staging must fit in stage 0");
};

// Byte offset of 16-byte chunk c of row r in a swizzled [rows x 512 B] tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

template <int NT, bool kDump>
__global__ void __launch_bounds__(MmaCfg<NT>::THREADS, 1)
    qsa_prefill_mma_kernel(const PrefillParams p) {
  using C = MmaCfg<NT>;
  constexpr int BK = C::BK;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t = blockIdx.x;
  const int g = blockIdx.y;
  const int G = p.G;
  const uint32_t sbase = smem_u32(smem);
  int32_t* ids_s = reinterpret_cast<int32_t*>(smem + C::OFF_IDS);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  __nv_bfloat16* p_s = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_P);

  // Step a1: list length and base pointers.
  int n_eff = p.K;
  if (p.n_valid != nullptr) n_eff = min(n_eff, max(p.n_valid[t * p.Hkv + g], 0));
  const int n_tiles = (n_eff + BK - 1) / BK;
  const int32_t* list = p.idx + t * p.idx_st + static_cast<int64_t>(g) * p.idx_sh;
  const __nv_bfloat16* kbase = p.k + static_cast<int64_t>(g) * p.kv_sh;
  const __nv_bfloat16* vbase = p.v + static_cast<int64_t>(g) * p.kv_sh;

  // Q rows of this group -> shared (padded heads zero-filled).
  {
    const __nv_bfloat16* q0 = p.q + t * p.q_st + static_cast<int64_t>(g) * G * p.q_sh;
    for (int i = tid; i < C::GP * kRowChunks; i += C::THREADS) {
      const int r = i / kRowChunks, c = i % kRowChunks;
      const bool real = r < G;
      cp_async_16(sbase + C::OFF_Q + swz(r, c), real ? q0 + r * p.q_sh + c * 8 : q0, real ? 16 : 0);
    }
  }

  // Each lane holds list entries (base + lane) and (base + 32 + lane) of a tile.
  auto load_ids = [&](int it, int& id0, int& id1) {
    const int j0 = it * BK + lane, j1 = j0 + 32;
    id0 = j0 < n_eff ? __ldg(list + j0) : -1;
    id1 = j1 < n_eff ? __ldg(list + j1) : -1;
  };
  auto check_ids = [&](int& id0, int& id1) {
    const bool bad0 = id0 >= p.S, bad1 = id1 >= p.S;
    if (bad0) id0 = -1;
    if (bad1) id1 = -1;
    if (warp == 0 && (bad0 || bad1) && p.status != nullptr) atomicOr(p.status, 1);
  };

  // Step a2: gather one tile into ring stage `st`.
  auto issue_tile = [&](int it, int st, int id0, int id1) {
    const uint32_t kdst = sbase + st * C::STAGE_BYTES;
    const uint32_t vdst = kdst + C::KV_TILE;
#pragma unroll
    for (int r = 0; r < BK / C::WARPS; ++r) {
      const int row = r * C::WARPS + warp;
      const int id = __shfl_sync(0xffffffffu, row < 32 ? id0 : id1, row & 31);
      const bool ok = id >= 0;
      const __nv_bfloat16* ks = ok ? kbase + static_cast<int64_t>(id) * p.kv_ss + lane * 8 : kbase;
      const __nv_bfloat16* vs = ok ? vbase + static_cast<int64_t>(id) * p.kv_ss + lane * 8 : vbase;
      const uint32_t off = swz(row, lane);
      cp_async_16(kdst + off, ks, ok ? 16 : 0);
      cp_async_16(vdst + off, vs, ok ? 16 : 0);
      if (kDump && lane == 0) {
        const int j = it * BK + row;
        if (j < p.K)
          p.gathered[(t * p.Hkv + g) * static_cast<int64_t>(p.K) + j] =
              ok ? static_cast<int32_t>((ks - kbase) / p.kv_ss) : -1;
      }
    }
    if (warp == 0) {
      ids_s[st * BK + lane] = id0;
      ids_s[st * BK + 32 + lane] = id1;
    }
  };

  int nid0 = -1, nid1 = -1;
  if (n_tiles > 0) load_ids(0, nid0, nid1);
#pragma unroll
  for (int s = 0; s < C::STAGES - 1; ++s) {
    if (s < n_tiles) {
      check_ids(nid0, nid1);
      issue_tile(s, s, nid0, nid1);
      if (s + 1 < n_tiles) load_ids(s + 1, nid0, nid1);
    }
    cp_async_commit();
  }

  uint32_t qf[NT][16][2];
  float m_run[NT][2], l_run[NT][2];
  float o_acc[4][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_run[nt][e] = -INFINITY;
      l_run[nt][e] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) o_acc[mt][nt][c] = 0.f;
  }

  for (int i = 0; i < n_tiles; ++i) {
    cp_async_wait<C::STAGES - 2>();
    __syncthreads();
    if (i == 0) {
      // Q^T fragments (B operand of the score MMA), kept in registers.
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) {
          const int row = nt * 8 + (lane & 7);
          const int chunk = k2 * 4 + (lane >> 3);
          ldmatrix_x4(sbase + C::OFF_Q + swz(row, chunk), qf[nt][2 * k2][0], qf[nt][2 * k2][1],
                      qf[nt][2 * k2 + 1][0], qf[nt][2 * k2 + 1][1]);
        }
    }
    {
      const int it = i + C::STAGES - 1;
      if (it < n_tiles) {
        check_ids(nid0, nid1);
        issue_tile(it, it % C::STAGES, nid0, nid1);
        if (it + 1 < n_tiles) load_ids(it + 1, nid0, nid1);
      }
      cp_async_commit();
    }
    const int st = i % C::STAGES;
    const uint32_t kaddr = sbase + st * C::STAGE_BYTES;
    const uint32_t vaddr = kaddr + C::KV_TILE;

    // Step a3: scores for this warp's 16 keys.
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[nt][c] = 0.f;
    {
      const int krow = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(kaddr + swz(krow, ks * 2 + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
      }
    }

    // Step a4: mask, tile max across warps, exponentials, running sums.
    const int key0 = warp * 16 + (lane >> 2), key1 = key0 + 8;
    const bool v0 = ids_s[st * BK + key0] >= 0, v1 = ids_s[st * BK + key1] >= 0;
    float mx[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[nt][e] = v0 ? s[nt][e] * p.scale_log2 : -INFINITY;
        s[nt][2 + e] = v1 ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
        float m = fmaxf(s[nt][e], s[nt][2 + e]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        mx[nt][e] = m;
      }
    if (lane < 4) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) red[warp * C::GP + nt * 8 + lane * 2 + e] = mx[nt][e];
    }
    __syncthreads();
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = nt * 8 + (lane & 3) * 2 + e;
        float tm = red[h];
#pragma unroll
        for (int w = 1; w < C::WARPS; ++w) tm = fmaxf(tm, red[w * C::GP + h]);
        const float m_new = fmaxf(m_run[nt][e], tm);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        alpha[nt][e] = ex2(m_run[nt][e] - m_use);
        m_run[nt][e] = m_new;
        const float p0 = ex2(s[nt][e] - m_use);
        const float p1 = ex2(s[nt][2 + e] - m_use);
        // the row sum keeps FP32 precision (it sets lse); P enters PV as BF16
        l_run[nt][e] = l_run[nt][e] * alpha[nt][e] + p0 + p1;
        p_s[h * C::P_STRIDE + key0] = __float2bfloat16_rn(p0);
        p_s[h * C::P_STRIDE + key1] = __float2bfloat16_rn(p1);
      }
    __syncthreads();

    // Step a5: O^T += V^T P^T for this warp's 64 rows of D.
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        o_acc[mt][nt][0] *= alpha[nt][0];
        o_acc[mt][nt][1] *= alpha[nt][1];
        o_acc[mt][nt][2] *= alpha[nt][0];
        o_acc[mt][nt][3] *= alpha[nt][1];
      }
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int prow = nt * 8 + (lane & 7);
        const int pcol = kk * 16 + ((lane >> 3) & 1) * 8;
        ldmatrix_x2(sbase + C::OFF_P + (prow * C::P_STRIDE + pcol) * 2, pb[nt][0], pb[nt][1]);
      }
      const int vrow = kk * 16 + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int vchunk = (warp * 64 + mt * 16) / 8 + ((lane >> 3) & 1);
        uint32_t a[4];
        ldmatrix_x4_trans(vaddr + swz(vrow, vchunk), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o_acc[mt][nt], a, pb[nt][0], pb[nt][1]);
      }
    }
  }

  // Step a6: epilogue.
  cp_async_wait<0>();
  __syncthreads();
  float inv[NT][2], lsum[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      lsum[nt][e] = l;
    }
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) red[warp * C::GP + nt * 8 + lane * 2 + e] = lsum[nt][e];
  }
  __syncthreads();
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = nt * 8 + (lane & 3) * 2 + e;
      float l = red[h];
#pragma unroll
      for (int w = 1; w < C::WARPS; ++w) l += red[w * C::GP + h];
      lsum[nt][e] = l;
      inv[nt][e] = l > 0.f ? 1.f / l : 0.f;
    }
  // O^T fragments -> [h][d] BF16 staging in stage 0 (all copies have landed).
  __nv_bfloat16* o_s = reinterpret_cast<__nv_bfloat16*>(smem);
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int d = warp * 64 + mt * 16 + (lane >> 2);
      const int h = nt * 8 + (lane & 3) * 2;
      const bool z0 = !(lsum[nt][0] > 0.f), z1 = !(lsum[nt][1] > 0.f);
      o_s[h * kHeadDim + d] = __float2bfloat16_rn(z0 ? 0.f : o_acc[mt][nt][0] * inv[nt][0]);
      o_s[(h + 1) * kHeadDim + d] = __float2bfloat16_rn(z1 ? 0.f : o_acc[mt][nt][1] * inv[nt][1]);
      o_s[h * kHeadDim + d + 8] = __float2bfloat16_rn(z0 ? 0.f : o_acc[mt][nt][2] * inv[nt][0]);
      o_s[(h + 1) * kHeadDim + d + 8] = __float2bfloat16_rn(z1 ? 0.f : o_acc[mt][nt][3] * inv[nt][1]);
    }
  if (p.lse != nullptr && warp == 0 && lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = nt * 8 + lane * 2 + e;
        if (h < G) {
          const float l = lsum[nt][e];
          p.lse[t * p.lse_st + static_cast<int64_t>(g) * G + h] =
              l > 0.f ? (m_run[nt][e] + lg2(l)) * 0.69314718055994531f : -INFINITY;
        }
      }
  }
  __syncthreads();
  __nv_bfloat16* orow0 = p.out + t * p.o_st + static_cast<int64_t>(g) * G * p.o_sh;
  for (int i = tid; i < G * kRowChunks; i += C::THREADS) {
    const int h = i / kRowChunks, c = i % kRowChunks;
    *reinterpret_cast<uint4*>(orow0 + h * p.o_sh + c * 8) =
        *reinterpret_cast<const uint4*>(o_s + h * kHeadDim + c * 8);
  }
}

}  // namespace qsa
