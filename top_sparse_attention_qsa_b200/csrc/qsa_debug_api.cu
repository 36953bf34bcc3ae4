// qsa_debug_api.cu -- C ABI of the measurement kernels and test hooks
// (include/qsa_debug.h).  Compiled only into libqsa_debug.so, with QSA_DEBUG
// defined; the production library libqsa.so does not contain this file.
#ifndef QSA_DEBUG
#error "qsa_debug_api.cu belongs to the debug library (build with -DQSA_DEBUG)"
#endif

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "qsa.h"
#include "qsa_debug.h"
#include "qsa_gather_only.cuh"
#include "qsa_gather_peak.cuh"
#include "qsa_launch.cuh"

namespace {

using namespace qsa::host;
using namespace qsa::launch;

// Fills the tcgen05 parameters of an unsplit token-list call, or returns an error.
qsa_status_t prepare(const qsa_shape_t* s, const void* q, const void* k, const void* v, const int32_t* idx,
                     const int32_t* n_valid, float scale, void* out, float* lse, int32_t* status,
                     qsa::tc::TcParams* tp) {
  qsa_status_t rc = validate(s, q, k, v, idx, out);
  if (rc != QSA_OK) return rc;
  if (s->num_tokens == 0) return QSA_OK;
  if (!make_tc_params(s, q, tp)) return QSA_ERR_UNSUPPORTED;
  fill_tc_params(tp, s, q, k, v, idx, n_valid, scale, 1.f, 1.f, out, lse, status, 0, nullptr);
  return QSA_OK;
}

template <typename Kernel>
cudaError_t launch_persistent(Kernel kernel, const qsa::tc::TcParams& tp, int threads, int smem,
                              std::atomic<int>* done, cudaStream_t stream) {
  cudaError_t e = set_smem_once(kernel, smem, done);
  if (e != cudaSuccess) return e;
  unsigned grid = 0;
  if ((e = persistent_grid(tp, &grid)) != cudaSuccess) return e;
  kernel<<<grid, threads, smem, stream>>>(tp);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- gather peak

struct PeakLaunch {
  qsa::peak::PeakParams p;
  int threads, smem, grid;
};

template <int kRowBytes, int kDepth>
cudaError_t run_peak_depth(int method, const PeakLaunch& L, cudaStream_t st) {
  using namespace qsa::peak;
  static std::atomic<int> done[3][kMaxDevices];
  cudaError_t e;
  switch (method) {
    case kCpAsync: {
      auto k = gather_peak_cp_async<kRowBytes, kDepth>;
      if ((e = set_smem_once(k, L.smem, done[0])) != cudaSuccess) return e;
      k<<<L.grid, L.threads, L.smem, st>>>(L.p);
      break;
    }
    case kLdV4: {
      auto k = gather_peak_ld_v4<kRowBytes, kDepth>;
      k<<<L.grid, L.threads, 0, st>>>(L.p);
      break;
    }
    default: {
      auto k = gather_peak_bulk<kRowBytes, kDepth>;
      if ((e = set_smem_once(k, L.smem, done[2])) != cudaSuccess) return e;
      k<<<L.grid, L.threads, L.smem, st>>>(L.p);
      break;
    }
  }
  return cudaGetLastError();
}

template <int kRowBytes>
cudaError_t run_peak(int method, int depth, const PeakLaunch& L, cudaStream_t st) {
  switch (depth) {
    case 1: return run_peak_depth<kRowBytes, 1>(method, L, st);
    case 2: return run_peak_depth<kRowBytes, 2>(method, L, st);
    case 3: return run_peak_depth<kRowBytes, 3>(method, L, st);
    case 4: return run_peak_depth<kRowBytes, 4>(method, L, st);
    case 8: return run_peak_depth<kRowBytes, 8>(method, L, st);
    default: return run_peak_depth<kRowBytes, 16>(method, L, st);
  }
}

bool peak_depth_ok(int method, int depth) {
  using namespace qsa::peak;
  switch (method) {
    case kCpAsync: return depth == 1 || depth == 2 || depth == 4 || depth == 8;
    case kLdV4: return depth == 4 || depth == 8 || depth == 16;
    case kBulk: return depth >= 1 && depth <= 4;
    default: return false;
  }
}

}  // namespace

extern "C" {

qsa_status_t qsa_debug_gather_only(const qsa_shape_t* shape, int32_t cache_fp8, const void* q,
                                   const void* k_cache, const void* v_cache, const int32_t* topk_idx,
                                   const int32_t* n_valid, int32_t* status, void* stream) {
  if (shape == nullptr) return QSA_ERR_NULL;
  // out is never written; q stands in for it in the checks
  if (cache_fp8 && shape->topk > 0 && (shape->kv_stride_slot % 16 != 0 || shape->kv_stride_head % 16 != 0))
    return QSA_ERR_ALIGN;
  static thread_local qsa::tc::TcParams tp;
  qsa_status_t rc = prepare(shape, q, k_cache, v_cache, topk_idx, n_valid, 0.f, const_cast<void*>(q), nullptr,
                            status, &tp);
  if (rc != QSA_OK || shape->num_tokens == 0) return rc;
  tp.out = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (cache_fp8) {
    static std::atomic<int> done[kMaxDevices];
    e = launch_persistent(qsa::f8::qsa_gather_only_f8_kernel, tp, 32 * (qsa::f8::kProducerWarps8 + 1),
                          qsa::f8::F_SMEM, done, st);
  } else {
    static std::atomic<int> done[kMaxDevices];
    e = launch_persistent(qsa::tc::qsa_gather_only_kernel, tp, qsa::tc::kGatherOnlyThreads,
                          qsa::tc::SMEM_BYTES, done, st);
  }
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

qsa_status_t qsa_debug_gather_peak(const void* table, int64_t rows, int64_t row_stride_bytes, int32_t row_bytes,
                                   const int32_t* ids, int64_t n_ids, int32_t method, int32_t depth,
                                   int32_t warps, int32_t ctas_per_sm, uint32_t* sink, int64_t sink_words,
                                   int32_t* status, void* stream) {
  using namespace qsa::peak;
  if (table == nullptr || ids == nullptr) return QSA_ERR_NULL;
  if (rows < 1 || rows > 0x7fffffffLL || n_ids < 0 || warps < 1 || warps > 32 || ctas_per_sm < 1 ||
      ctas_per_sm > 8)
    return QSA_ERR_SHAPE;
  if (row_bytes != 256 && row_bytes != 512) return QSA_ERR_UNSUPPORTED;
  if (!peak_depth_ok(method, depth)) return QSA_ERR_UNSUPPORTED;
  if (row_stride_bytes < row_bytes || row_stride_bytes % 16 != 0) return QSA_ERR_SHAPE;
  if (!aligned16(table) || (reinterpret_cast<uintptr_t>(ids) & 3u)) return QSA_ERR_ALIGN;
  const int nsm = sm_count();
  if (nsm <= 0) return QSA_ERR_CUDA;
  PeakLaunch L;
  L.threads = 32 * warps;
  L.grid = nsm * ctas_per_sm;
  switch (method) {
    case kCpAsync: L.smem = warps * depth * kGroupBytes; break;
    case kBulk: L.smem = warps * depth * (kBulkRows * row_bytes + 8); break;
    default: L.smem = 0; break;
  }
  if (L.smem > 227 * 1024 || static_cast<int64_t>(L.smem) * ctas_per_sm > 228 * 1024) return QSA_ERR_UNSUPPORTED;
  if (method == kLdV4 && warps > (depth >= 16 ? 16 : 32)) return QSA_ERR_UNSUPPORTED;
  // every kernel is built for at most 1024 threads per SM (64 registers each)
  if (warps * 32 * ctas_per_sm > 1024) return QSA_ERR_UNSUPPORTED;
  if (method == kLdV4 && (sink == nullptr || sink_words < static_cast<int64_t>(L.grid) * L.threads))
    return QSA_ERR_SHAPE;
  if (n_ids == 0) return QSA_OK;
  L.p.table = static_cast<const char*>(table);
  L.p.ids = ids;
  L.p.n_ids = n_ids;
  L.p.rows = rows;
  L.p.row_stride = row_stride_bytes;
  L.p.sink = sink;
  L.p.status = status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = row_bytes == 512 ? run_peak<512>(method, depth, L, st) : run_peak<256>(method, depth, L, st);
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

qsa_status_t qsa_test_stalled_pipeline(const qsa_shape_t* shape, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* topk_idx, const int32_t* n_valid,
                                       float scale, void* out, float* lse, int32_t* status, void* stream) {
  if (status == nullptr) return QSA_ERR_NULL;
  static thread_local qsa::tc::TcParams tp;
  qsa_status_t rc = prepare(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status, &tp);
  if (rc != QSA_OK || shape->num_tokens == 0) return rc;
  const cudaError_t e = launch_tc<false, true>(tp, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

int32_t qsa_debug_abi_version(void) { return QSA_DEBUG_ABI_VERSION; }

}  // extern "C"
