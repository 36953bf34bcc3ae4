// qsa_launch.cuh -- host-side argument checks, parameter set-up and launches
// of the attention kernels, shared by the library's entry points (libqsa.so)
// and its measurement / test-hook library (libqsa_debug.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "qsa.h"
#include "qsa_host.cuh"
#include "qsa_prefill_f8.cuh"
#include "qsa_prefill_mma.cuh"
#include "qsa_prefill_tc.cuh"

namespace qsa {
namespace launch {

using namespace qsa::host;

// Validates `s` and the pointers of a forward call.  Returns QSA_OK or the
// first error found; never touches device memory.
inline qsa_status_t validate(const qsa_shape_t* s, const void* q, const void* k, const void* v,
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

// block_size -> log2 (1, 2, 4, 8, 16), else -1.
inline int block_shift_of(int32_t block_size) {
  for (int b = 0; b <= 4; ++b)
    if (block_size == (1 << b)) return b;
  return -1;
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

// Fills the Q tensor map of the tcgen05 kernels.  Returns false when a TMA
// descriptor cannot express the Q layout or there is nothing to gather.
inline bool make_tc_params(const qsa_shape_t* s, const void* q, qsa::tc::TcParams* tp) {
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

// Every field of the tcgen05 kernels' parameters except the Q tensor map,
// for one unsplit pass over token (shift 0) or microblock lists.
// `score_scale` multiplies the softmax scale (an FP8 cache's k_scale) and
// `o_scale` the normalised output (its v_scale).
inline void fill_tc_params(qsa::tc::TcParams* tp, const qsa_shape_t* s, const void* q, const void* k,
                           const void* v, const int32_t* idx, const int32_t* n_valid, float scale,
                           float score_scale, float o_scale, void* out, float* lse, int32_t* status,
                           int shift, const int32_t* last_slot) {
  const float sc = scale > 0.f ? scale : 0.0625f;  // 1/sqrt(256)
  tp->idx = idx;
  tp->n_valid = n_valid;
  tp->kraw = k;
  tp->vraw = v;
  tp->out = static_cast<__nv_bfloat16*>(out);
  tp->lse = lse;
  tp->status = status;
  tp->gathered = nullptr;
  tp->T = s->num_tokens;
  tp->idx_st = s->idx_stride_tok;
  tp->idx_sh = s->idx_stride_head;
  tp->o_st = s->o_stride_tok;
  tp->o_sh = s->o_stride_head;
  tp->lse_st = s->lse_stride_tok;
  tp->kv_ss = s->kv_stride_slot;
  tp->kv_sh = s->kv_stride_head;
  tp->Hkv = s->num_kv_heads;
  tp->G = s->num_q_heads / s->num_kv_heads;
  tp->K = s->topk;
  tp->S = static_cast<int32_t>(s->num_slots);
  tp->scale_log2 = sc * score_scale * 1.4426950408889634f;
  tp->o_scale = o_scale;
  tp->splits = 1;
  tp->chunk = s->topk << shift;
  tp->part_o = nullptr;
  tp->part_lse = nullptr;
  tp->block_shift = shift;
  tp->last_slot = last_slot;
  tp->q_ptr = q;
  tp->q_st = s->q_stride_tok;
  tp->q_sh = s->q_stride_head;
}

// Persistent grid: one CTA per SM, or one per unit when there are fewer.
inline cudaError_t persistent_grid(const qsa::tc::TcParams& tp, unsigned* grid) {
  const int64_t units = tp.T * tp.Hkv * tp.splits;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  *grid = static_cast<unsigned>(units < nsm ? units : nsm);
  return cudaSuccess;
}

// The attention kernels rebalance registers between their warpgroups with
// setmaxnreg, which draws on the registers the block was launched with: a
// split larger than that would make a warpgroup wait for registers forever.
// Checked once per kernel against the compiled launch register count;
// `need` = 128 x the sum over the warpgroups of their registers per thread.
template <typename Kernel>
cudaError_t check_register_split(Kernel kernel, int threads, long need, std::atomic<int>* done) {
  if (done->load(std::memory_order_acquire)) return cudaSuccess;
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kernel);
  if (e != cudaSuccess) return e;
  if (static_cast<long>(attr.numRegs) * threads < need) return cudaErrorInvalidConfiguration;
  done->store(1, std::memory_order_release);
  return cudaSuccess;
}

template <bool kDump, bool kStall = false, bool kBlocks = false>
cudaError_t launch_tc(const qsa::tc::TcParams& tp, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  static std::atomic<int> regs_ok;
  auto kernel = qsa::tc::qsa_prefill_tc_kernel<kDump, kStall, kBlocks>;
  using namespace qsa::tc;
  cudaError_t e = check_register_split(
      kernel, kThreads, 128L * (kRegsSoftmax + long(kProducerGroups) * kRegsProducer + kRegsMma), &regs_ok);
  if (e != cudaSuccess) return e;
  e = set_smem_once(kernel, qsa::tc::SMEM_BYTES, done);
  if (e != cudaSuccess) return e;
  unsigned grid = 0;
  if ((e = persistent_grid(tp, &grid)) != cudaSuccess) return e;
  kernel<<<grid, qsa::tc::kThreads, qsa::tc::SMEM_BYTES, stream>>>(tp);
  return cudaGetLastError();
}

template <bool kBlocks, bool kDump = false>
cudaError_t launch_f8(const qsa::tc::TcParams& tp, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  static std::atomic<int> regs_ok;
  auto kernel = qsa::f8::qsa_prefill_f8_kernel<kBlocks, kDump>;
  using namespace qsa::f8;
  cudaError_t e = check_register_split(kernel, kThreads8,
                                       128L * (kRegsProd8 + kRegsMisc8 + 2L * kRegsSm8 + kRegsEpi8), &regs_ok);
  if (e != cudaSuccess) return e;
  e = set_smem_once(kernel, qsa::f8::F_SMEM, done);
  if (e != cudaSuccess) return e;
  unsigned grid = 0;
  if ((e = persistent_grid(tp, &grid)) != cudaSuccess) return e;
  kernel<<<grid, qsa::f8::kThreads8, qsa::f8::F_SMEM, stream>>>(tp);
  return cudaGetLastError();
}

}  // namespace launch
}  // namespace qsa
