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
#include "qsa_host.cuh"
#include "qsa_gather_only.cuh"
#include "qsa_merge.cuh"
#include "qsa_prefill_mma.cuh"
#include "qsa_prefill_tc.cuh"
#include "qsa_prefill_f8.cuh"

namespace {

using namespace qsa::host;

// Validates `s` and the pointers of a forward call.  Returns QSA_OK or the
// first error found; never touches device memory.
qsa_status_t validate(const qsa_shape_t* s, const void* q, const void* k, const void* v,
                      const int32_t* idx, const void* out) {
  if (s == nullptr) return QSA_ERR_NULL;
  if (s->num_tokens < 0 || s->topk < 0 || s->num_slots < 0 || s->num_q_heads <= 0 ||
      s->num_kv_heads <= 0)
    return QSA_ERR_SHAPE;
  if (s->num_q_heads % s->num_kv_heads != 0) return QSA_ERR_SHAPE;
  if (s->head_dim != qsa::kHeadDim) return QSA_ERR_UNSUPPORTED;
  const int G = s->num_q_heads / s->num_kv_heads;
  if (G > 16) return QSA_ERR_UNSUPPORTED;
  if (s->num_kv_heads > 65535 || s->num_tokens > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  if (s->num_tokens == 0) return QSA_OK;
  if (q == nullptr || out == nullptr) return QSA_ERR_NULL;
  const bool reads_cache = s->topk > 0;
  if (reads_cache && (k == nullptr || v == nullptr || idx == nullptr)) return QSA_ERR_NULL;
  // strides: non-negative, rows 16-byte aligned
  const int64_t st[] = {s->q_stride_tok, s->q_stride_head, s->o_stride_tok, s->o_stride_head,
                        s->kv_stride_slot, s->kv_stride_head};
  for (int64_t x : st)
    if (x < 0) return QSA_ERR_SHAPE;
  if (s->idx_stride_tok < 0 || s->idx_stride_head < 0 || s->lse_stride_tok < 0) return QSA_ERR_SHAPE;
  if (reads_cache && s->num_slots > 0 && s->kv_stride_slot == 0) return QSA_ERR_SHAPE;
  for (int64_t x : st)
    if (x % 8 != 0) return QSA_ERR_ALIGN;
  if (!aligned16(q) || !aligned16(out)) return QSA_ERR_ALIGN;
  if (reads_cache && (!aligned16(k) || !aligned16(v))) return QSA_ERR_ALIGN;
  if (reads_cache && (reinterpret_cast<uintptr_t>(idx) & 3u)) return QSA_ERR_ALIGN;
  if (s->num_slots > 0x80000000LL) return QSA_ERR_UNSUPPORTED;  // int32 slot ids
  return QSA_OK;
}

template <int NT, bool kDump>
cudaError_t launch_mma(const qsa::PrefillParams& p, cudaStream_t stream) {
  using C = qsa::MmaCfg<NT>;
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::qsa_prefill_mma_kernel<NT, kDump>;
  cudaError_t e = set_smem_once(kernel, C::SMEM, done);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.T), static_cast<unsigned>(p.Hkv));
  kernel<<<grid, C::THREADS, C::SMEM, stream>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- TMA path

// Fills the Q tensor map of the tcgen05 kernel.  Returns false when a TMA
// descriptor cannot express the Q layout or there is nothing to gather (the
// warp-MMA kernel takes those calls).
bool make_tc_params(const qsa_shape_t* s, const void* q, qsa::tc::TcParams* tp) {
  using namespace qsa::tc;
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  if (s->topk <= 0 || s->num_slots <= 0 || s->num_slots >= 0x7fffffffLL) return false;
  const cuuint32_t elem_str[3] = {1, 1, 1};
  const uint64_t hq = static_cast<uint64_t>(s->num_q_heads);
  uint64_t st_h = static_cast<uint64_t>(s->q_stride_head) * 2;
  if (hq == 1 || st_h < 512) {
    if (hq > 1) return false;
    st_h = 512;
  }
  uint64_t st_t = static_cast<uint64_t>(s->q_stride_tok) * 2;
  if (s->num_tokens == 1 || st_t < st_h * hq) {
    if (s->num_tokens > 1) return false;
    st_t = st_h * hq;
  }
  const cuuint64_t qdims[3] = {256, hq, static_cast<cuuint64_t>(s->num_tokens)};
  const cuuint64_t qstr[2] = {st_h, st_t};
  const cuuint32_t qbox[3] = {64, static_cast<cuuint32_t>(kGp), 1};
  return enc(&tp->tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), qdims, qstr, qbox,
             elem_str, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kBlocks>
cudaError_t launch_f8(const qsa::tc::TcParams& tp, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::f8::qsa_prefill_f8_kernel<kBlocks>;
  cudaError_t e = set_smem_once(kernel, qsa::f8::F_SMEM, done);
  if (e != cudaSuccess) return e;
  const int64_t units = tp.T * tp.Hkv;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
  kernel<<<grid, qsa::f8::kThreads8, qsa::f8::F_SMEM, stream>>>(tp);
  return cudaGetLastError();
}

cudaError_t launch_gather_only(const qsa::tc::TcParams& tp, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::tc::qsa_gather_only_kernel;
  cudaError_t e = set_smem_once(kernel, qsa::tc::SMEM_BYTES, done);
  if (e != cudaSuccess) return e;
  const int64_t units = tp.T * tp.Hkv;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
  kernel<<<grid, qsa::tc::kGatherOnlyThreads, qsa::tc::SMEM_BYTES, stream>>>(tp);
  return cudaGetLastError();
}

cudaError_t launch_f8_gather_only(const qsa::tc::TcParams& tp, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::f8::qsa_gather_only_f8_kernel;
  cudaError_t e = set_smem_once(kernel, qsa::f8::F_SMEM, done);
  if (e != cudaSuccess) return e;
  const int64_t units = tp.T * tp.Hkv;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
  kernel<<<grid, 32 * (qsa::tc::kProducerWarps + 1), qsa::f8::F_SMEM, stream>>>(tp);
  return cudaGetLastError();
}

template <bool kDump, bool kStall = false, bool kBlocks = false>
cudaError_t launch_tc(const qsa::tc::TcParams& tp, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::tc::qsa_prefill_tc_kernel<kDump, kStall, kBlocks>;
  cudaError_t e = set_smem_once(kernel, qsa::tc::SMEM_BYTES, done);
  if (e != cudaSuccess) return e;
  const int64_t units = tp.T * tp.Hkv;
  int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
  kernel<<<grid, qsa::tc::kThreads, qsa::tc::SMEM_BYTES, stream>>>(tp);
  return cudaGetLastError();
}

qsa_status_t run_forward(const qsa_shape_t* s, const void* q, const void* k, const void* v,
                         const int32_t* idx, const int32_t* n_valid, float scale, void* out,
                         float* lse, int32_t* status, int32_t* gathered, void* stream,
                         qsa_kernel_t which = QSA_KERNEL_AUTO, bool stall_test = false) {
  if (which != QSA_KERNEL_AUTO && which != QSA_KERNEL_TCGEN05 && which != QSA_KERNEL_WARP_MMA &&
      which != QSA_KERNEL_GATHER_ONLY)
    return QSA_ERR_UNSUPPORTED;
  if (which == QSA_KERNEL_GATHER_ONLY && (gathered != nullptr || stall_test)) return QSA_ERR_UNSUPPORTED;
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
  cudaError_t e;
  const bool dump = gathered != nullptr;
  static thread_local qsa::tc::TcParams tp;
  const bool use_tc = which != QSA_KERNEL_WARP_MMA && make_tc_params(s, q, &tp);
  if ((which == QSA_KERNEL_TCGEN05 || which == QSA_KERNEL_GATHER_ONLY) && !use_tc) return QSA_ERR_UNSUPPORTED;
  if (use_tc) {
    tp.idx = idx;
    tp.n_valid = n_valid;
    tp.kraw = k;
    tp.vraw = v;
    tp.kv_ss = s->kv_stride_slot;
    tp.kv_sh = s->kv_stride_head;
    tp.out = p.out;
    tp.lse = lse;
    tp.status = status;
    tp.gathered = gathered;
    tp.T = p.T;
    tp.idx_st = p.idx_st;
    tp.idx_sh = p.idx_sh;
    tp.o_st = p.o_st;
    tp.o_sh = p.o_sh;
    tp.lse_st = p.lse_st;
    tp.Hkv = p.Hkv;
    tp.G = p.G;
    tp.K = p.K;
    tp.S = static_cast<int32_t>(p.S);
    tp.scale_log2 = p.scale_log2;
    tp.splits = 1;
    tp.chunk = p.K;
    tp.part_o = nullptr;
    tp.part_lse = nullptr;
    tp.block_shift = 0;
    tp.last_slot = nullptr;
    tp.o_scale = 1.f;
    if (which == QSA_KERNEL_GATHER_ONLY)
      e = launch_gather_only(tp, st);
    else
      e = stall_test ? launch_tc<false, true>(tp, st)
                     : (dump ? launch_tc<true>(tp, st) : launch_tc<false>(tp, st));
  } else if (p.G <= 8)
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
// 128-entry tile.  With num_splits <= 0: one chunk unless the (token, KV head)
// units would leave most SMs idle (fewer than SMs / 8), then enough chunks of
// at least 256 entries for about one unit per SM.  (Each unit carries a few
// microseconds of serial start and epilogue latency, so short chunks cost
// more than idle SMs until the units are that scarce.)  Deterministic for a
// given shape and device.
bool plan_splits(const qsa_shape_t* s, int32_t num_splits, SplitPlan* pl) {
  const int64_t K = s->topk;
  const int64_t max_splits = K > 0 ? (K + qsa::tc::kKeys - 1) / qsa::tc::kKeys : 1;
  int64_t splits = num_splits;
  if (num_splits <= 0) {
    const int nsm = sm_count();
    if (nsm <= 0) return false;
    const int64_t units = s->num_tokens * s->num_kv_heads;
    splits = 1;
    if (units > 0 && units * 8 < nsm) {
      splits = (nsm + units - 1) / units;
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
                       int32_t* status, void* stream, bool gather_only = false);

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
  const float sc = scale > 0.f ? scale : 0.0625f;
  tp.idx = idx;
  tp.n_valid = n_valid;
  tp.kraw = k;
  tp.vraw = v;
  tp.out = static_cast<__nv_bfloat16*>(out);
  tp.lse = lse;
  tp.status = status;
  tp.gathered = nullptr;
  tp.T = s->num_tokens;
  tp.idx_st = s->idx_stride_tok;
  tp.idx_sh = s->idx_stride_head;
  tp.o_st = s->o_stride_tok;
  tp.o_sh = s->o_stride_head;
  tp.lse_st = s->lse_stride_tok;
  tp.kv_ss = s->kv_stride_slot;
  tp.kv_sh = s->kv_stride_head;
  tp.Hkv = s->num_kv_heads;
  tp.G = s->num_q_heads / s->num_kv_heads;
  tp.K = s->topk;
  tp.S = static_cast<int32_t>(s->num_slots);
  tp.scale_log2 = sc * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
  tp.splits = pl.splits;
  tp.chunk = pl.chunk;
  tp.part_o = part_o;
  tp.part_lse = part_lse;
  tp.block_shift = 0;
  tp.last_slot = nullptr;
  tp.o_scale = fp8 ? v_scale : 1.f;
  tp.q_ptr = q;
  tp.q_st = s->q_stride_tok;
  tp.q_sh = s->q_stride_head;
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

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (cudaGetSymbolAddress allocates nothing).
cudaError_t noalloc_scratch_address(void** ptr) {
  static std::atomic<void*> cache[kMaxDevices];
  static std::mutex lock;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = cache[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> g(lock);
    p = cache[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      cache[dev].store(p, std::memory_order_release);
    }
  }
  *ptr = p;
  return cudaSuccess;
}

// Microblock (or token) lists on the tcgen05 kernel, BF16 or FP8 E4M3 cache.
qsa_status_t run_lists(const qsa_shape_t* shape, int32_t block_size, const int32_t* last_slot,
                       const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* topk_idx, const int32_t* n_valid, float scale,
                       float k_scale, float v_scale, bool fp8, void* out, float* lse,
                       int32_t* status, void* stream, bool gather_only) {
  qsa_status_t rc = validate(shape, q, k_cache, v_cache, topk_idx, out);
  if (rc != QSA_OK) return rc;
  if (gather_only && (!fp8 || block_size != 1 || last_slot != nullptr)) return QSA_ERR_UNSUPPORTED;
  if (fp8 && shape->topk > 0 && (shape->kv_stride_slot % 16 != 0 || shape->kv_stride_head % 16 != 0))
    return QSA_ERR_ALIGN;   // FP8 rows move in 16-byte pieces of 16 elements
  int shift = -1;
  for (int b = 0; b <= 4; ++b)
    if (block_size == (1 << b)) shift = b;
  if (shift < 0) return QSA_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(shape->topk) << shift) > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  if (shape->num_tokens == 0) return QSA_OK;
  static thread_local qsa::tc::TcParams tp;
  if (!make_tc_params(shape, q, &tp)) return QSA_ERR_UNSUPPORTED;
  const float sc = scale > 0.f ? scale : 0.0625f;
  tp.idx = topk_idx;
  tp.n_valid = n_valid;
  tp.kraw = k_cache;
  tp.vraw = v_cache;
  tp.out = static_cast<__nv_bfloat16*>(out);
  tp.lse = lse;
  tp.status = status;
  tp.gathered = nullptr;
  tp.T = shape->num_tokens;
  tp.idx_st = shape->idx_stride_tok;
  tp.idx_sh = shape->idx_stride_head;
  tp.o_st = shape->o_stride_tok;
  tp.o_sh = shape->o_stride_head;
  tp.lse_st = shape->lse_stride_tok;
  tp.kv_ss = shape->kv_stride_slot;
  tp.kv_sh = shape->kv_stride_head;
  tp.Hkv = shape->num_kv_heads;
  tp.G = shape->num_q_heads / shape->num_kv_heads;
  tp.K = shape->topk;
  tp.S = static_cast<int32_t>(shape->num_slots);
  // an FP8 cache's K scale multiplies every score; its V scale the output
  tp.scale_log2 = sc * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
  tp.o_scale = fp8 ? v_scale : 1.f;
  tp.splits = 1;
  tp.chunk = shape->topk << shift;
  tp.part_o = nullptr;
  tp.part_lse = nullptr;
  tp.block_shift = shift;
  tp.last_slot = last_slot;
  tp.q_ptr = q;
  tp.q_st = shape->q_stride_tok;
  tp.q_sh = shape->q_stride_head;
  const bool plain = shift == 0 && last_slot == nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (gather_only)
    e = launch_f8_gather_only(tp, st);
  else if (fp8)
    e = plain ? launch_f8<false>(tp, st) : launch_f8<true>(tp, st);
  else
    e = plain ? launch_tc<false>(tp, st) : launch_tc<false, false, true>(tp, st);
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
    if (rc != QSA_OK) return rc;
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
  // `stream` ends after the last copy down
  if (hp != nullptr)
    ok = ok && cudaEventRecord(hp->ev[1], down) == cudaSuccess && cudaStreamWaitEvent(st, hp->ev[1], 0) == cudaSuccess;
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
  if (need > 0 && noalloc_scratch_address(&scratch) != cudaSuccess) return QSA_ERR_CUDA;
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

qsa_status_t qsa_sparse_prefill_fp8_fwd_with(const qsa_shape_t* shape, int32_t block_size,
                                             const int32_t* last_slot, const void* q,
                                             const void* k_cache, const void* v_cache,
                                             const int32_t* topk_idx, const int32_t* n_valid,
                                             float scale, float k_scale, float v_scale, void* out,
                                             float* lse, int32_t* status, qsa_kernel_t kernel,
                                             void* stream) {
  if (kernel != QSA_KERNEL_AUTO && kernel != QSA_KERNEL_TCGEN05 && kernel != QSA_KERNEL_GATHER_ONLY)
    return QSA_ERR_UNSUPPORTED;
  return run_lists(shape, block_size, last_slot, q, k_cache, v_cache, topk_idx, n_valid, scale,
                   k_scale, v_scale, true, out, lse, status, stream, kernel == QSA_KERNEL_GATHER_ONLY);
}

qsa_status_t qsa_test_stalled_pipeline(const qsa_shape_t* shape, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* topk_idx, const int32_t* n_valid,
                                       float scale, void* out, float* lse, int32_t* status,
                                       void* stream) {
  if (status == nullptr) return QSA_ERR_NULL;
  return run_forward(shape, q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse, status,
                     nullptr, stream, QSA_KERNEL_TCGEN05, true);
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
