// qsa_merge.cuh -- combine split-K partial attention results.
//
// Each chunk s of a token's list yields a normalised partial output o_s and
// its log-sum-exp lse_s (natural log, scale included).  Attention over the
// whole list is the lse-weighted mix of the chunks:
//   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) o_s,
// which is exact (it is the same softmax with the normaliser split into
// per-chunk sums).  This is the combine step of decode context parallelism
// for QSA named on page "Qwen4-Exp QSA llega al Ascend de Huawei", section
// "Dónde encaja esto en el despliegue del servicio de Qwen4Exp" (vLLM #59279);
// a chunk with no live entry has lse_s = -inf and weight 0, and a row whose
// chunks are all empty gets out = +0.0 and lse = -inf.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace qsa {

struct MergeParams {
  const float* part_o;    // [rows][splits][256]
  const float* part_lse;  // [rows][splits]
  __nv_bfloat16* out;
  float* lse;             // may be nullptr
  int64_t rows;           // T * Hq
  int32_t Hq, splits;
  int64_t o_st, o_sh, lse_st;
};

// One CTA of 64 threads per (token, query head) row; thread i owns dims 4i..4i+3.
__global__ void __launch_bounds__(64) qsa_merge_splits_kernel(const MergeParams p) {
  const int64_t r = blockIdx.x;
  if (r >= p.rows) return;
  const float* pl = p.part_lse + r * p.splits;
  float m = -INFINITY;
  for (int s = 0; s < p.splits; ++s) m = fmaxf(m, pl[s]);
  const int64_t t = r / p.Hq;
  const int h = static_cast<int>(r - t * p.Hq);
  __nv_bfloat16* orow = p.out + t * p.o_st + static_cast<int64_t>(h) * p.o_sh;
  const int d = 4 * threadIdx.x;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float w = expf(pl[s] - m);  // 0 for an empty chunk
      wsum += w;
      const float4 o = *reinterpret_cast<const float4*>(p.part_o + (r * p.splits + s) * 256 + d);
      acc[0] += w * o.x;
      acc[1] += w * o.y;
      acc[2] += w * o.z;
      acc[3] += w * o.w;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  __nv_bfloat162 b = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&a);
  pk.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(orow + d) = pk;
  if (p.lse != nullptr && threadIdx.x == 0)
    p.lse[t * p.lse_st + h] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace qsa
