// qsa_api.cu -- C ABI of the QSA sparse-attention prefill library (sm_100a).
//
// Host-side argument validation, kernel selection and launch.  See
// include/qsa.h for the contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "qsa.h"
#include "qsa_launch.cuh"
#include "qsa_merge.cuh"

namespace {

using namespace qsa::host;
using namespace qsa::launch;

qsa_status_t run_forward(const qsa_shape_t* s, const void* q, const void* k, const void* v,
                         const int32_t* idx, const int32_t* n_valid, float scale, void* out,
                         float* lse, int32_t* status, int32_t* gathered, void* stream,
                         qsa_kernel_t which = QSA_KERNEL_AUTO) {
  if (which != QSA_KERNEL_AUTO && which != QSA_KERNEL_TCGEN05 && which != QSA_KERNEL_WARP_MMA)
    return QSA_ERR_UNSUPPORTED;
  qsa_status_t rc = validate(s, q, k, v, idx, out);
  if (rc != QSA_OK) return rc;
  if (gathered != nullptr && s->topk > 0 && (reinterpret_cast<uintptr_t>(gathered) & 3u))
    return QSA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s->num_tokens == 0) return QSA_OK;
  if (gathered != nullptr && s->topk > 0) {
    const size_t n = static_cast<size_t>(s->num_tokens) * s->num_kv_heads * s->topk;
    if (cudaMemsetAsync(gathered, 0xff, n * sizeof(int32_t), st) != cudaSuccess) return QSA_ERR_CUDA;
  }
  cudaError_t e;
  const bool dump = gathered != nullptr;
  static thread_local qsa::tc::TcParams tp;
  const bool use_tc = which != QSA_KERNEL_WARP_MMA && make_tc_params(s, q, &tp);
  if (which == QSA_KERNEL_TCGEN05 && !use_tc) return QSA_ERR_UNSUPPORTED;
  if (use_tc) {
    fill_tc_params(&tp, s, q, k, v, idx, n_valid, scale, 1.f, 1.f, out, lse, status, 0, nullptr);
    tp.gathered = gathered;
    e = dump ? launch_tc<true>(tp, st) : launch_tc<false>(tp, st);
    return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
  }
  qsa::PrefillParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.idx = idx;
  p.n_valid = n_valid;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = status;
  p.gathered = gathered;
  p.T = s->num_tokens;
  p.Hkv = s->num_kv_heads;
  p.G = s->num_q_heads / s->num_kv_heads;
  p.K = s->topk;
  p.S = s->num_slots;
  p.q_st = s->q_stride_tok;
  p.q_sh = s->q_stride_head;
  p.kv_ss = s->kv_stride_slot;
  p.kv_sh = s->kv_stride_head;
  p.idx_st = s->idx_stride_tok;
  p.idx_sh = s->idx_stride_head;
  p.o_st = s->o_stride_tok;
  p.o_sh = s->o_stride_head;
  p.lse_st = s->lse_stride_tok;
  const float sc = scale > 0.f ? scale : 0.0625f;  // 1/sqrt(256)
  p.scale_log2 = sc * 1.4426950408889634f;
  if (p.G <= 8)
    e = dump ? launch_mma<1, true>(p, st) : launch_mma<1, false>(p, st);
  else
    e = dump ? launch_mma<2, true>(p, st) : launch_mma<2, false>(p, st);
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

// ---------------------------------------------------------------- split-K decode

struct SplitPlan {
  int32_t splits;
  int32_t chunk;
  size_t part_o_bytes;   // [T*Hq][splits][256] FP32
  size_t lse_offset;     // 256-byte aligned
  size_t total_bytes;
};

// Chunk count for a decode-shaped call, never chunks shorter than one
// 128-entry tile.  With num_splits <= 0: floor(SMs / units) chunks per list
// for the (token, KV head) units, so that all chunks run in one wave of one
// persistent CTA per SM, but no chunk shorter than 256 entries.  Timed in
// CUDA graphs on 148 SMs (K = 2048, 8 to 128 units, BF16 and FP8 caches),
// that count was the fastest of 1, 2, 3, 4, 6 and 8 at every size: a
// second wave costs a whole unit's serial latency, while shorter chunks
// below one wave cost only the merge.  Deterministic for a given shape and
// device.
bool plan_splits(const qsa_shape_t* s, int32_t num_splits, SplitPlan* pl) {
  const int64_t K = s->topk;
  const int64_t max_splits = K > 0 ? (K + qsa::tc::kKeys - 1) / qsa::tc::kKeys : 1;
  int64_t splits = num_splits;
  if (num_splits <= 0) {
    const int nsm = sm_count();
    if (nsm <= 0) return false;
    const int64_t units = s->num_tokens * s->num_kv_heads;
    splits = 1;
    if (units > 0 && units * 2 <= nsm) {
      splits = nsm / units;
      const int64_t by_len = K / 256;
      if (splits > by_len) splits = by_len < 1 ? 1 : by_len;
    }
  }
  splits = splits < 1 ? 1 : (splits > max_splits ? max_splits : splits);
  int64_t chunk = K > 0 ? (K + splits - 1) / splits : 0;
  chunk = (chunk + qsa::tc::kKeys - 1) / qsa::tc::kKeys * qsa::tc::kKeys;
  if (chunk > 0) splits = (K + chunk - 1) / chunk;
  pl->splits = static_cast<int32_t>(splits);
  pl->chunk = static_cast<int32_t>(chunk);
  const size_t rows = static_cast<size_t>(s->num_tokens) * s->num_q_heads;
  pl->part_o_bytes = rows * pl->splits * 256 * sizeof(float);
  pl->lse_offset = (pl->part_o_bytes + 255) / 256 * 256;
  pl->total_bytes = pl->lse_offset + rows * pl->splits * sizeof(float);
  return true;
}

cudaError_t launch_merge(const qsa_shape_t* s, const float* part_o, const float* part_lse,
                         int32_t splits, void* out, float* lse, cudaStream_t stream) {
  qsa::MergeParams mp;
  mp.part_o = part_o;
  mp.part_lse = part_lse;
  mp.out = static_cast<__nv_bfloat16*>(out);
  mp.lse = lse;
  mp.rows = s->num_tokens * s->num_q_heads;
  mp.Hq = s->num_q_heads;
  mp.splits = splits;
  mp.o_st = s->o_stride_tok;
  mp.o_sh = s->o_stride_head;
  mp.lse_st = s->lse_stride_tok;
  if (mp.rows > 0x7fffffffLL) return cudaErrorInvalidValue;
  qsa::qsa_merge_splits_kernel<<<static_cast<unsigned>(mp.rows), 64, 0, stream>>>(mp);
  return cudaGetLastError();
}

// Split-K forward: partial results of every chunk go to `workspace` (laid
// out by plan_splits), then one merge launch writes out/lse.
qsa_status_t run_lists(const qsa_shape_t* shape, int32_t block_size, const int32_t* last_slot,
                       const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* topk_idx, const int32_t* n_valid, float scale,
                       float k_scale, float v_scale, bool fp8, void* out, float* lse,
                       int32_t* status, void* stream, int32_t* gathered = nullptr);

// The host-buffer entry point cuts the query tokens into chunks of about
// kHostChunkTokens (at most kHostMaxChunks) so that the copies of one chunk
// overlap the kernel of the previous one.  Its copy streams and events are
// made once per device and reused; a mutex serialises the calls that enqueue
// on them.
constexpr int64_t kHostChunkTokens = 1024;
constexpr int kHostMaxChunks = 8;

struct HostPipe {
  std::mutex lock;
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t ev[2 + 2 * kHostMaxChunks] = {};
};

HostPipe* host_pipe() {
  static HostPipe pipes[kMaxDevices];
  static std::atomic<int> made[kMaxDevices];
  static std::mutex make_lock;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (made[dev].load(std::memory_order_acquire) == 1) return &pipes[dev];
  std::lock_guard<std::mutex> g(make_lock);
  if (made[dev].load(std::memory_order_acquire) == 0) {
    HostPipe& hp = pipes[dev];
    bool ok = cudaStreamCreateWithFlags(&hp.up, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.down, cudaStreamNonBlocking) == cudaSuccess;
    for (auto& e : hp.ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    made[dev].store(ok ? 1 : -1, std::memory_order_release);
  }
  return made[dev].load(std::memory_order_acquire) == 1 ? &pipes[dev] : nullptr;
}

qsa_status_t run_decode(const qsa_shape_t* s, const void* q, const void* k, const void* v,
                        const int32_t* idx, const int32_t* n_valid, float scale, void* out,
                        float* lse, int32_t* status, int32_t num_splits, void* workspace,
                        size_t workspace_bytes, void* stream, bool fp8 = false, float k_scale = 1.f,
                        float v_scale = 1.f) {
  qsa_status_t rc = validate(s, q, k, v, idx, out);
  if (rc != QSA_OK) return rc;
  if (fp8 && s->topk > 0 && (s->kv_stride_slot % 16 != 0 || s->kv_stride_head % 16 != 0))
    return QSA_ERR_ALIGN;
  if (s->num_tokens == 0) return QSA_OK;
  SplitPlan pl;
  if (!plan_splits(s, num_splits, &pl)) return QSA_ERR_CUDA;
  static thread_local qsa::tc::TcParams tp;
  if (pl.splits <= 1 || !make_tc_params(s, q, &tp)) {
    if (fp8)
      return run_lists(s, 1, nullptr, q, k, v, idx, n_valid, scale, k_scale, v_scale, true, out, lse,
                       status, stream);
    return run_forward(s, q, k, v, idx, n_valid, scale, out, lse, status, nullptr, stream);
  }
  if (workspace == nullptr) return QSA_ERR_NULL;
  if (workspace_bytes < pl.total_bytes) return QSA_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return QSA_ERR_ALIGN;
  float* part_o = static_cast<float*>(workspace);
  float* part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.lse_offset);
  fill_tc_params(&tp, s, q, k, v, idx, n_valid, scale, fp8 ? k_scale : 1.f, fp8 ? v_scale : 1.f, out, lse,
                 status, 0, nullptr);
  tp.splits = pl.splits;
  tp.chunk = pl.chunk;
  tp.part_o = part_o;
  tp.part_lse = part_lse;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((fp8 ? launch_f8<false>(tp, st) : launch_tc<false>(tp, st)) != cudaSuccess) return QSA_ERR_CUDA;
  if (launch_merge(s, part_o, part_lse, pl.splits, out, lse, st) != cudaSuccess) return QSA_ERR_CUDA;
  return QSA_OK;
}

// Bytes spanned by a strided [n0, n1, inner] layout (first to last element).
size_t span_bytes(int64_t n0, int64_t s0, int64_t n1, int64_t s1, int64_t inner, size_t elem) {
  if (n0 <= 0 || n1 <= 0 || inner <= 0) return 0;
  return static_cast<size_t>((n0 - 1) * s0 + (n1 - 1) * s1 + inner) * elem;
}

// ---------------------------------------------------------------- allocation-free decode

// Scratch for qsa_sparse_decode_fwd_noalloc: lives in the library's device
// image, so it exists on every device the module is loaded on.  Host code
// must not pass `g_noalloc_scratch` itself to a kernel (in host code it is
// only a stand-in symbol); it passes the device address looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch in the current context.  The lookup
// (cudaGetSymbolAddress, which allocates nothing) is cached per device
// together with the context it was made in, and redone when the current
// context differs (after cudaDeviceReset, or under another context): the
// module, and with it the array, may then sit at another address.  A lookup
// that would have to happen while `stream` is being captured is refused
// (cudaErrorStreamCaptureUnsupported), since it may load the module.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

cudaError_t noalloc_scratch_address(cudaStream_t stream, void** ptr) {
  struct Entry {
    CUcontext ctx = nullptr;
    void* ptr = nullptr;
  };
  static Entry cache[kMaxDevices];
  static std::mutex lock;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return cudaErrorContextIsDestroyed;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
  std::lock_guard<std::mutex> g(lock);
  if (ctx == nullptr || cache[dev].ctx != ctx || cache[dev].ptr == nullptr) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if ((e = cudaStreamIsCapturing(stream, &cap)) != cudaSuccess) return e;
    if (cap != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
    void* p = nullptr;
    // (this also makes the device's primary context current if none was)
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return e;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorContextIsDestroyed;
    cache[dev].ctx = ctx;
    cache[dev].ptr = p;
  }
  *ptr = cache[dev].ptr;
  return cudaSuccess;
}

// Microblock (or token) lists on the tcgen05 kernel, BF16 or FP8 E4M3 cache.
qsa_status_t run_lists(const qsa_shape_t* shape, int32_t block_size, const int32_t* last_slot,
                       const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* topk_idx, const int32_t* n_valid, float scale,
                       float k_scale, float v_scale, bool fp8, void* out, float* lse,
                       int32_t* status, void* stream, int32_t* gathered) {
  qsa_status_t rc = validate(shape, q, k_cache, v_cache, topk_idx, out);
  if (rc != QSA_OK) return rc;
  if (fp8 && shape->topk > 0 && (shape->kv_stride_slot % 16 != 0 || shape->kv_stride_head % 16 != 0))
    return QSA_ERR_ALIGN;   // FP8 rows move in 16-byte pieces of 16 elements
  const int shift = block_shift_of(block_size);
  if (shift < 0) return QSA_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(shape->topk) << shift) > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  if (gathered != nullptr && shape->topk > 0 && (reinterpret_cast<uintptr_t>(gathered) & 3u))
    return QSA_ERR_ALIGN;
  if (shape->num_tokens == 0) return QSA_OK;
  static thread_local qsa::tc::TcParams tp;
  if (!make_tc_params(shape, q, &tp)) return QSA_ERR_UNSUPPORTED;
  fill_tc_params(&tp, shape, q, k_cache, v_cache, topk_idx, n_valid, scale, fp8 ? k_scale : 1.f,
                 fp8 ? v_scale : 1.f, out, lse, status, shift, last_slot);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (gathered != nullptr) {
    const size_t n = static_cast<size_t>(shape->num_tokens) * shape->num_kv_heads * (static_cast<size_t>(shape->topk) << shift);
    if (cudaMemsetAsync(gathered, 0xff, n * sizeof(int32_t), st) != cudaSuccess) return QSA_ERR_CUDA;
    tp.gathered = gathered;
  }
  const bool plain = shift == 0 && last_slot == nullptr;
  const bool dump = gathered != nullptr;
  cudaError_t e;
  if (fp8) {
    if (dump)
      e = plain ? launch_f8<false, true>(tp, st) : launch_f8<true, true>(tp, st);
    else
      e = plain ? launch_f8<false>(tp, st) : launch_f8<true>(tp, st);
  } else {
    if (dump)
      e = plain ? launch_tc<true>(tp, st) : launch_tc<true, false, true>(tp, st);
    else
      e = plain ? launch_tc<false>(tp, st) : launch_tc<false, false, true>(tp, st);
  }
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

}  // namespace

extern "C" {

qsa_status_t qsa_sparse_prefill_fwd(const qsa_shape_t* shape, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* topk_idx,
                                    const int32_t* n_valid, float scale, void* out, float* lse,
                                    int32_t* status, void* stream) {
  return run_forward(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status,
                     nullptr, stream);
}

qsa_status_t qsa_sparse_prefill_fwd_with(const qsa_shape_t* shape, const void* q,
                                         const void* k_cache, const void* v_cache,
                                         const int32_t* topk_idx, const int32_t* n_valid,
                                         float scale, void* out, float* lse, int32_t* status,
                                         qsa_kernel_t kernel, void* stream) {
  return run_forward(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status,
                     nullptr, stream, kernel);
}

qsa_status_t qsa_sparse_prefill_debug_gather(const qsa_shape_t* shape, const void* q,
                                             const void* k_cache, const void* v_cache,
                                             const int32_t* topk_idx, const int32_t* n_valid,
                                             float scale, void* out, float* lse, int32_t* status,
                                             int32_t* gathered_ids, void* stream) {
  if (gathered_ids == nullptr) return QSA_ERR_NULL;
  return run_forward(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status,
                     gathered_ids, stream);
}

qsa_status_t qsa_sparse_prefill_fwd_host(const qsa_shape_t* s, const void* q_host,
                                         const void* k_cache_host, const void* v_cache_host,
                                         const int32_t* topk_idx_host, const int32_t* n_valid_host,
                                         float scale, void* out_host, float* lse_host,
                                         const qsa_device_buffers_t* dev, void* stream) {
  if (s == nullptr || dev == nullptr) return QSA_ERR_NULL;
  qsa_status_t rc = validate(s, dev->q, dev->k_cache, dev->v_cache, dev->topk_idx, dev->out);
  if (rc != QSA_OK) return rc;
  if (s->num_tokens == 0) return QSA_OK;
  const int64_t T = s->num_tokens, Hq = s->num_q_heads, Hkv = s->num_kv_heads, D = s->head_dim;
  const int64_t K = s->topk, S = s->num_slots;
  if (q_host == nullptr || out_host == nullptr) return QSA_ERR_NULL;
  if (K > 0 && (k_cache_host == nullptr || v_cache_host == nullptr || topk_idx_host == nullptr))
    return QSA_ERR_NULL;
  if ((n_valid_host != nullptr) != (dev->n_valid != nullptr)) return QSA_ERR_NULL;
  if (lse_host != nullptr && dev->lse == nullptr) return QSA_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int chunks = static_cast<int>(std::min<int64_t>(std::max<int64_t>(T / kHostChunkTokens, 1), kHostMaxChunks));
  HostPipe* hp = chunks > 1 ? host_pipe() : nullptr;
  if (chunks > 1 && hp == nullptr) return QSA_ERR_CUDA;
  std::unique_lock<std::mutex> hold;
  if (hp != nullptr) hold = std::unique_lock<std::mutex>(hp->lock);
  // one stream does everything for a single chunk; otherwise inputs go up on
  // hp->up, the kernels run on `stream`, outputs come down on hp->down
  cudaStream_t up = hp ? hp->up : st, down = hp ? hp->down : st;
  auto copy = [](void* d, const void* h, size_t n, cudaMemcpyKind kind, cudaStream_t x) {
    return n == 0 || cudaMemcpyAsync(d, h, n, kind, x) == cudaSuccess;
  };
  auto at = [](const void* p, int64_t elems, int64_t bytes_per) {
    return static_cast<const char*>(p) + elems * bytes_per;
  };
  bool ok = true;
  if (hp != nullptr) {
    ok = cudaEventRecord(hp->ev[0], st) == cudaSuccess && cudaStreamWaitEvent(up, hp->ev[0], 0) == cudaSuccess &&
         cudaStreamWaitEvent(down, hp->ev[0], 0) == cudaSuccess;
  }
  if (ok && K > 0) {
    const size_t kv = span_bytes(S, s->kv_stride_slot, Hkv, s->kv_stride_head, D, 2);
    ok = copy(dev->k_cache, k_cache_host, kv, cudaMemcpyHostToDevice, up) &&
         copy(dev->v_cache, v_cache_host, kv, cudaMemcpyHostToDevice, up);
  }
  if (ok && dev->status != nullptr) ok = cudaMemsetAsync(dev->status, 0, 4, st) == cudaSuccess;
  for (int c = 0; c < chunks && ok; ++c) {
    const int64_t t0 = T * c / chunks, tc = T * (c + 1) / chunks - t0;
    // this chunk's inputs
    ok = copy(const_cast<char*>(at(dev->q, t0 * s->q_stride_tok, 2)), at(q_host, t0 * s->q_stride_tok, 2),
              span_bytes(tc, s->q_stride_tok, Hq, s->q_stride_head, D, 2), cudaMemcpyHostToDevice, up);
    if (ok && K > 0)
      ok = copy(const_cast<char*>(at(dev->topk_idx, t0 * s->idx_stride_tok, 4)),
                at(topk_idx_host, t0 * s->idx_stride_tok, 4),
                span_bytes(tc, s->idx_stride_tok, Hkv, s->idx_stride_head, K, 4), cudaMemcpyHostToDevice, up);
    if (ok && n_valid_host != nullptr)
      ok = copy(const_cast<char*>(at(dev->n_valid, t0 * Hkv, 4)), at(n_valid_host, t0 * Hkv, 4),
                static_cast<size_t>(tc * Hkv) * 4, cudaMemcpyHostToDevice, up);
    if (ok && hp != nullptr)
      ok = cudaEventRecord(hp->ev[2 + c], up) == cudaSuccess && cudaStreamWaitEvent(st, hp->ev[2 + c], 0) == cudaSuccess;
    if (!ok) break;
    // its kernel
    qsa_shape_t sc = *s;
    sc.num_tokens = tc;
    rc = run_forward(&sc, at(dev->q, t0 * s->q_stride_tok, 2), dev->k_cache, dev->v_cache,
                     reinterpret_cast<const int32_t*>(at(dev->topk_idx, t0 * s->idx_stride_tok, 4)),
                     dev->n_valid ? reinterpret_cast<const int32_t*>(at(dev->n_valid, t0 * Hkv, 4)) : nullptr,
                     scale, const_cast<char*>(at(dev->out, t0 * s->o_stride_tok, 2)),
                     lse_host != nullptr ? reinterpret_cast<float*>(const_cast<char*>(at(dev->lse, t0 * s->lse_stride_tok, 4)))
                                         : nullptr,
                     dev->status, nullptr, st);
    if (rc != QSA_OK) break;
    // its outputs
    if (hp != nullptr)
      ok = cudaEventRecord(hp->ev[2 + kHostMaxChunks + c], st) == cudaSuccess &&
           cudaStreamWaitEvent(down, hp->ev[2 + kHostMaxChunks + c], 0) == cudaSuccess;
    ok = ok && copy(const_cast<char*>(at(out_host, t0 * s->o_stride_tok, 2)), at(dev->out, t0 * s->o_stride_tok, 2),
                    span_bytes(tc, s->o_stride_tok, Hq, s->o_stride_head, D, 2), cudaMemcpyDeviceToHost, down);
    if (ok && lse_host != nullptr)
      ok = copy(const_cast<char*>(at(lse_host, t0 * s->lse_stride_tok, 4)), at(dev->lse, t0 * s->lse_stride_tok, 4),
                span_bytes(tc, s->lse_stride_tok, 1, 0, Hq, 4), cudaMemcpyDeviceToHost, down);
  }
  // `stream` ends after every copy enqueued on the two copy streams, on the
  // error paths too: the caller may free or reuse the host buffers as soon
  // as `stream` is done
  if (hp != nullptr) {
    const bool joined = cudaEventRecord(hp->ev[0], up) == cudaSuccess &&
                        cudaStreamWaitEvent(st, hp->ev[0], 0) == cudaSuccess &&
                        cudaEventRecord(hp->ev[1], down) == cudaSuccess &&
                        cudaStreamWaitEvent(st, hp->ev[1], 0) == cudaSuccess;
    ok = ok && joined;
  }
  if (rc != QSA_OK) return rc;
  return ok ? QSA_OK : QSA_ERR_CUDA;
}

size_t qsa_sparse_decode_workspace_bytes(const qsa_shape_t* shape, int32_t num_splits) {
  if (shape == nullptr || shape->num_tokens < 0 || shape->topk < 0 || shape->num_q_heads <= 0 ||
      shape->num_kv_heads <= 0)
    return 0;
  SplitPlan pl;
  if (!plan_splits(shape, num_splits, &pl) || pl.splits <= 1) return 0;
  return pl.total_bytes;
}

int32_t qsa_sparse_decode_num_splits(const qsa_shape_t* shape, int32_t num_splits) {
  if (shape == nullptr || shape->topk < 0 || shape->num_tokens < 0 || shape->num_kv_heads <= 0)
    return 0;
  SplitPlan pl;
  if (!plan_splits(shape, num_splits, &pl)) return 0;
  return pl.splits;
}

qsa_status_t qsa_sparse_decode_fwd(const qsa_shape_t* shape, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* topk_idx,
                                   const int32_t* n_valid, float scale, void* out, float* lse,
                                   int32_t* status, int32_t num_splits, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return run_decode(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status,
                    num_splits, workspace, workspace_bytes, stream);
}

qsa_status_t qsa_sparse_decode_fp8_fwd(const qsa_shape_t* shape, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* topk_idx,
                                       const int32_t* n_valid, float scale, float k_scale,
                                       float v_scale, void* out, float* lse, int32_t* status,
                                       int32_t num_splits, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  return run_decode(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status, num_splits,
                    workspace, workspace_bytes, stream, true, k_scale, v_scale);
}

qsa_status_t qsa_sparse_decode_fwd_noalloc(const qsa_shape_t* shape, const void* q,
                                           const void* k_cache, const void* v_cache,
                                           const int32_t* topk_idx, const int32_t* n_valid,
                                           float scale, void* out, float* lse, int32_t* status,
                                           int32_t num_splits, void* stream) {
  qsa_status_t rc = validate(shape, q, k_cache, v_cache, topk_idx, out);
  if (rc != QSA_OK) return rc;
  if (shape->num_tokens == 0) return QSA_OK;
  SplitPlan pl;
  if (!plan_splits(shape, num_splits, &pl)) return QSA_ERR_CUDA;
  const size_t need = pl.splits > 1 ? pl.total_bytes : 0;
  if (need > QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_SCRATCH;
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = noalloc_scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (e == cudaErrorStreamCaptureUnsupported) return QSA_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return QSA_ERR_CUDA;
  }
  return run_decode(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status,
                    num_splits, scratch, need, stream);
}

qsa_status_t qsa_sparse_prefill_block_fwd(const qsa_shape_t* shape, int32_t block_size,
                                          const int32_t* last_slot, const void* q,
                                          const void* k_cache, const void* v_cache,
                                          const int32_t* topk_idx, const int32_t* n_valid,
                                          float scale, void* out, float* lse, int32_t* status,
                                          void* stream) {
  return run_lists(shape, block_size, last_slot, q, k_cache, v_cache, topk_idx, n_valid, scale, 1.f,
                   1.f, false, out, lse, status, stream);
}

qsa_status_t qsa_sparse_prefill_fp8_fwd(const qsa_shape_t* shape, int32_t block_size,
                                        const int32_t* last_slot, const void* q,
                                        const void* k_cache, const void* v_cache,
                                        const int32_t* topk_idx, const int32_t* n_valid,
                                        float scale, float k_scale, float v_scale, void* out,
                                        float* lse, int32_t* status, void* stream) {
  return run_lists(shape, block_size, last_slot, q, k_cache, v_cache, topk_idx, n_valid, scale,
                   k_scale, v_scale, true, out, lse, status, stream);
}

qsa_status_t qsa_sparse_prefill_debug_gather_lists(const qsa_shape_t* shape, int32_t block_size,
                                                   const int32_t* last_slot, int32_t cache_fp8,
                                                   const void* q, const void* k_cache, const void* v_cache,
                                                   const int32_t* topk_idx, const int32_t* n_valid,
                                                   float scale, float k_scale, float v_scale, void* out,
                                                   float* lse, int32_t* status, int32_t* gathered_ids,
                                                   void* stream) {
  if (gathered_ids == nullptr) return QSA_ERR_NULL;
  return run_lists(shape, block_size, last_slot, q, k_cache, v_cache, topk_idx, n_valid, scale,
                   cache_fp8 ? k_scale : 1.f, cache_fp8 ? v_scale : 1.f, cache_fp8 != 0, out, lse, status,
                   stream, gathered_ids);
}

const char* qsa_status_string(qsa_status_t status) {
  switch (status) {
    case QSA_OK: return "ok";
    case QSA_ERR_NULL: return "a required pointer is NULL";
    case QSA_ERR_SHAPE: return "inconsistent sizes or strides";
    case QSA_ERR_UNSUPPORTED: return "unsupported configuration (attention: BF16, head_dim 256, G <= 16; indexer: head_dim 128, 1/2/4/8 heads, <= 32768 candidates)";
    case QSA_ERR_ALIGN: return "rows must start on 16-byte boundaries";
    case QSA_ERR_CUDA: return "a CUDA runtime call failed";
    case QSA_ERR_SCRATCH: return "the call needs more scratch than the built-in array holds (QSA_NOALLOC_SCRATCH_BYTES)";
  }
  return "unknown status";
}

int32_t qsa_abi_version(void) { return QSA_ABI_VERSION; }

}  // extern "C"
