// qsa_gather_peak.cuh -- measurement kernels: how fast this GPU moves rows
// named by a random index list from global memory into its SMs.
//
// The sparse-attention prefill reads, for every list entry, one K row and one
// V row picked at random from the cache (page "Qwen4-Exp QSA llega al Ascend
// de Huawei", section "Lo que realmente añade la pull request": only the
// selected rows take part).  Its speed is therefore bounded by the rate of
// random row reads, not by the streaming copy rate of HBM.  These kernels
// measure that rate with no attention around it, written independently of
// the prefill kernels' producer code, so that the prefill can be judged
// against the hardware and not only against its own gather.
//
// Three ways to move a row, each with a depth of rows in flight:
//   kCpAsync  16-byte cp.async per lane into a per-warp shared-memory ring
//             (one warp instruction = 512 bytes: one 512-byte row or two
//             256-byte rows), commit groups of 8 instructions, at most
//             `depth` groups outstanding per warp;
//   kLdV4     16-byte ld.global.cg.v4 per lane into registers, `depth`
//             instructions issued before any is consumed (the values are
//             folded into one word per thread so the loads stay live);
//   kBulk     one cp.async.bulk (1-d, global -> shared) per row, 32 rows per
//             stage and warp, stages completed on mbarriers (bounded waits).
// Each CTA takes a contiguous share of the index list.  Row ids are clamped
// into the table, so every access stays inside it whatever the list holds.
#pragma once

#include <cstdint>

#include "qsa_ptx.cuh"
#include "qsa_tc_ptx.cuh"

namespace qsa {
namespace peak {

enum Method : int { kCpAsync = 0, kLdV4 = 1, kBulk = 2 };

constexpr int kInstrPerGroup = 8;       // cp.async: warp instructions per commit group
constexpr int kGroupBytes = kInstrPerGroup * 512;
constexpr int kBulkRows = 32;           // bulk: rows per stage (one per lane)

struct PeakParams {
  const char* table;      // rows of row_bytes, row_stride bytes apart
  const int32_t* ids;     // n_ids row ids
  int64_t n_ids;
  int64_t rows;           // rows in the table (ids are clamped into [0, rows))
  int64_t row_stride;     // bytes, multiple of 16
  uint32_t* sink;         // kLdV4: one word per thread
  int32_t* status;        // kBulk: bit 1 when a wait ran past its bound
};

__device__ __forceinline__ int64_t clamp_row(int32_t id, int64_t rows) {
  return (id >= 0 && id < rows) ? id : 0;
}

// [begin, end) of this CTA's share of n units.
__device__ __forceinline__ void cta_share(int64_t n, int64_t& begin, int64_t& end) {
  const int64_t per = (n + gridDim.x - 1) / gridDim.x;
  begin = min(n, static_cast<int64_t>(blockIdx.x) * per);
  end = min(n, begin + per);
}

// cp.async into a per-warp ring of kDepth groups (kDepth x 4 KB per warp).
template <int kRowBytes, int kDepth>
__global__ void __launch_bounds__(1024) gather_peak_cp_async(const __grid_constant__ PeakParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kRowsPerInstr = 512 / kRowBytes;
  constexpr int kRowsPerGroup = kInstrPerGroup * kRowsPerInstr;
  constexpr int kChunks = kRowBytes / 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int64_t g0, g1;
  cta_share(p.n_ids / kRowsPerGroup, g0, g1);
  const uint32_t ring = smem_u32(smem) + static_cast<uint32_t>(warp * kDepth * kGroupBytes);
  const int sub = lane / kChunks, cc = lane % kChunks;
  int k = 0;
  // the ids of a group are loaded one group ahead, off the copies' critical path
  auto ids_of = [&](int64_t g) { return (g < g1 && lane < kRowsPerGroup) ? __ldg(p.ids + g * kRowsPerGroup + lane) : 0; };
  int32_t next = ids_of(g0 + warp);
  for (int64_t g = g0 + warp; g < g1; g += nw) {
    const int32_t mine = next;
    next = ids_of(g + nw);
    const uint32_t dst = ring + static_cast<uint32_t>(k * kGroupBytes);
#pragma unroll
    for (int i = 0; i < kInstrPerGroup; ++i) {
      const int64_t row = clamp_row(__shfl_sync(0xffffffffu, mine, i * kRowsPerInstr + sub), p.rows);
      cp_async_16(dst + i * 512 + lane * 16, p.table + row * p.row_stride + cc * 16, 16);
    }
    cp_async_commit();
    cp_async_wait<kDepth - 1>();
    k = k + 1 == kDepth ? 0 : k + 1;
  }
  cp_async_wait<0>();
}

// ld.global.cg.v4: kDepth independent 16-byte loads per lane in flight
// (at most 512 threads per CTA for kDepth 16, else 1024).
template <int kRowBytes, int kDepth>
__global__ void __launch_bounds__(kDepth >= 16 ? 512 : 1024) gather_peak_ld_v4(const __grid_constant__ PeakParams p) {
  constexpr int kRowsPerInstr = 512 / kRowBytes;
  constexpr int kRowsPerGroup = kDepth * kRowsPerInstr;
  constexpr int kChunks = kRowBytes / 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  int64_t g0, g1;
  cta_share(p.n_ids / kRowsPerGroup, g0, g1);
  const int sub = lane / kChunks, cc = lane % kChunks;
  uint32_t acc = 0;
  constexpr int kIdWords = (kRowsPerGroup + 31) / 32;
  int32_t next[kIdWords];
  auto load_ids = [&](int64_t g, int32_t (&dst)[kIdWords]) {
#pragma unroll
    for (int j = 0; j < kIdWords; ++j) {
      const int r = j * 32 + lane;
      dst[j] = (g < g1 && r < kRowsPerGroup) ? __ldg(p.ids + g * kRowsPerGroup + r) : 0;
    }
  };
  load_ids(g0 + warp, next);
  for (int64_t g = g0 + warp; g < g1; g += nw) {
    int32_t mine[kIdWords];
#pragma unroll
    for (int j = 0; j < kIdWords; ++j) mine[j] = next[j];
    load_ids(g + nw, next);
    uint4 v[kDepth];
#pragma unroll
    for (int i = 0; i < kDepth; ++i) {
      const int r = i * kRowsPerInstr + sub;
      const int64_t row = clamp_row(__shfl_sync(0xffffffffu, mine[r / 32], r % 32), p.rows);
      v[i] = __ldcg(reinterpret_cast<const uint4*>(p.table + row * p.row_stride + cc * 16));
    }
#pragma unroll
    for (int i = 0; i < kDepth; ++i) acc ^= v[i].x ^ v[i].y ^ v[i].z ^ v[i].w;
  }
  p.sink[static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x] = acc;
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// One 1-d bulk copy per row: each warp owns kDepth stages of 32 rows and one
// mbarrier per stage.  Waits are bounded (2 s) and set status bit 1 on expiry.
template <int kRowBytes, int kDepth>
__global__ void __launch_bounds__(1024) gather_peak_bulk(const __grid_constant__ PeakParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kStageBytes = kBulkRows * kRowBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + static_cast<uint32_t>(nw * kDepth * kStageBytes) + warp * kDepth * 8;
  const uint32_t ring = base + static_cast<uint32_t>(warp * kDepth * kStageBytes);
  if (lane < kDepth) tc::mbar_init(bars + 8 * lane, 1);
  tc::mbar_fence_init();
  __syncwarp();
  int64_t g0, g1;
  cta_share(p.n_ids / kBulkRows, g0, g1);
  uint32_t n_issued = 0;
  bool ok = true;
  int32_t next = g0 + warp < g1 ? __ldg(p.ids + (g0 + warp) * kBulkRows + lane) : 0;
  for (int64_t g = g0 + warp; g < g1 && ok; g += nw, ++n_issued) {
    const int32_t mine = next;
    next = g + nw < g1 ? __ldg(p.ids + (g + nw) * kBulkRows + lane) : 0;
    const uint32_t st = n_issued % kDepth;
    const uint32_t bar = bars + 8 * st;
    if (n_issued >= static_cast<uint32_t>(kDepth)) {
      // the stage's previous copies have landed
      const uint32_t par = ((n_issued / kDepth) - 1) & 1u;
      const uint64_t t0 = tc::globaltimer_ns();
      while (!tc::mbar_try_wait(bar, par)) {
        if (tc::globaltimer_ns() - t0 > 2000000000ull) {
          ok = false;
          break;
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
    }
    if (lane == 0) tc::mbar_arrive_expect_tx(bar, kStageBytes);
    __syncwarp();
    const int64_t row = clamp_row(mine, p.rows);
    bulk_copy_g2s(ring + st * kStageBytes + lane * kRowBytes, p.table + row * p.row_stride, kRowBytes, bar);
  }
  // drain: every stage that received copies completes before the CTA exits
  const uint32_t live = n_issued < static_cast<uint32_t>(kDepth) ? n_issued : kDepth;
  for (uint32_t j = 0; j < live; ++j) {
    const uint32_t c = n_issued - 1 - j;           // the last issue on stage c % kDepth
    const uint32_t bar = bars + 8 * (c % kDepth);
    const uint32_t par = (c / kDepth) & 1u;
    const uint64_t t0 = tc::globaltimer_ns();
    while (!tc::mbar_try_wait(bar, par))
      if (tc::globaltimer_ns() - t0 > 2000000000ull) {
        ok = false;
        break;
      }
  }
  if (!ok && lane == 0 && p.status != nullptr) atomicOr(p.status, static_cast<int32_t>(tc::kStatusTimeout));
}

}  // namespace peak
}  // namespace qsa
