// qsa_gather_only.cuh -- the KV gather of the tcgen05 prefill kernel alone,
// for measuring how fast that step can run.
//
// The gather (page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Lo
// que realmente añade la pull request": the attention reads only the cache
// rows named by each token's list) is the step that bounds the prefill on
// B200.  This kernel runs the prefill kernel's own producer warps
// (producer_role: the same list reads, masking, 16-byte cp.async copies and
// six-slot shared-memory ring, the same Q loads) and replaces the MMA and
// softmax warps with one warp that hands every slot back as soon as it is
// full.  It writes nothing to global memory.  Its time over a workload is
// the floor the full kernel could reach with free compute, and the ratio of
// the two times is the full kernel's efficiency against its own gather.
// qsa_gather_only_f8_kernel does the same for the FP8-cache kernel.
#pragma once

#include "qsa_prefill_f8.cuh"
#include "qsa_prefill_tc.cuh"

namespace qsa {
namespace tc {

constexpr int kGatherOnlyThreads = 32 * (kProducerWarps + 1);

// The consumer: for every unit take the Q buffer and give it back, for every
// tile take its four slots (K halves, V halves) and give them back.  Waits
// and phases mirror the score and PV issuers of the full kernel.
__device__ void release_role(const TcParams& p, const Sync& sy) {
  uint32_t c_slot = 0, c_unit = 0;
  const int64_t units = num_units(p);
  bool ok = true;
  for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const Unit un = decode_unit(p, u);
    const uint32_t qb = c_unit & 1u;
    ok = sy.wait(B_QFULL + qb, (c_unit >> 1) & 1u);
    if (!ok) break;
    ++c_unit;
    mbar_arrive(sy.bar(B_QEMPTY + qb));
    for (int i = 0; i < un.n_tiles && ok; ++i) {
      for (int h = 0; h < 4 && ok; ++h, ++c_slot) {
        const uint32_t slot = c_slot % kSlots;
        ok = sy.wait(B_FULL + slot, (c_slot / kSlots) & 1u);
        if (ok) mbar_arrive(sy.bar(B_EMPTY + slot));
      }
    }
  }
}

__global__ void __launch_bounds__(kGatherOnlyThreads, 1)
    qsa_gather_only_kernel(const __grid_constant__ TcParams p) {
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
      mbar_init(sy.bar(B_QFULL + b), 1);
      mbar_init(sy.bar(B_QEMPTY + b), 1);
    }
    *sy.abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp < kProducerWarps)
    producer_role<false, false, false>(p, sy, sb, warp, lane);
  else if (lane == 0)
    release_role(p, sy);
  __syncwarp();
  __syncthreads();
}

}  // namespace tc

namespace f8 {

// The same for the FP8 kernel's gather: its producer warps (one 32 KB slot
// per K or V tile of 256-byte rows), token lists; Q is not loaded, since the
// FP8 kernel reads it from global memory in its own warp.
__global__ void __launch_bounds__(32 * (kProducerWarps8 + 1), 1)
    qsa_gather_only_f8_kernel(const __grid_constant__ TcParams p) {
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
    *sy.abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp < kProducerWarps8) {
    producer8<false>(p, sy, sb, warp, lane);
  } else if (lane == 0) {
    uint32_t c_slot = 0;
    const int64_t units = num_units(p);
    bool ok = true;
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const Unit un = decode_unit(p, u);
      for (int i = 0; i < 2 * un.n_tiles && ok; ++i, ++c_slot) {   // K tile, V tile
        const uint32_t slot = c_slot % kSlots8;
        ok = sy.wait(G_FULL + slot, (c_slot / kSlots8) & 1u);
        if (ok) mbar_arrive(sy.bar(G_EMPTY + slot));
      }
    }
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace f8
}  // namespace qsa
