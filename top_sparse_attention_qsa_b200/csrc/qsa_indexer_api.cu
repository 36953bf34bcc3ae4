// qsa_indexer_api.cu -- C ABI of the QSA indexer scores and top-K
// selection (include/qsa.h): host-side validation, tensor maps and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "qsa.h"
#include "qsa_host.cuh"
#include "qsa_indexer.cuh"

namespace {

using namespace qsa::host;


qsa_status_t validate_indexer(const qsa_indexer_shape_t* s) {
  if (s == nullptr) return QSA_ERR_NULL;
  if (s->num_tokens < 0 || s->num_blocks <= 0 || s->block_size < 1 || s->num_heads <= 0)
    return QSA_ERR_SHAPE;
  if (s->head_dim != qsa::ix::kDh) return QSA_ERR_UNSUPPORTED;
  const int H = s->num_heads;
  if (H != 1 && H != 2 && H != 4 && H != 8) return QSA_ERR_UNSUPPORTED;
  if (s->num_blocks >= 0x7fffffffLL || s->num_tokens > 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  if (s->score_stride_tok < s->num_blocks) return QSA_ERR_SHAPE;
  if (s->score_stride_tok >= 0x7fffffffLL) return QSA_ERR_UNSUPPORTED;
  if (s->q_stride_tok < 0 || s->q_stride_head < 0 || s->k_stride_block < 0) return QSA_ERR_SHAPE;
  return QSA_OK;
}

// Tensor maps of the score kernel: k_idx [NB][128] (box 64 x 128 blocks) and
// q_idx [T][H][128] (box 64 x H x 256/H tokens), both 128-byte swizzled.
bool make_ix_maps(const qsa_indexer_shape_t* s, const void* q, const void* k, qsa::ix::IxParams* p) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint32_t es2[2] = {1, 1}, es3[3] = {1, 1, 1};
  uint64_t st_b = static_cast<uint64_t>(s->k_stride_block) * 2;
  if (s->num_blocks == 1) st_b = 256;
  if (st_b < 256) return false;
  const cuuint64_t kd[2] = {128, static_cast<cuuint64_t>(s->num_blocks)};
  const cuuint64_t ks[1] = {st_b};
  const cuuint32_t kb[2] = {64, qsa::ix::kBlk};
  if (enc(&p->tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k), kd, ks, kb, es2,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const uint64_t H = static_cast<uint64_t>(s->num_heads);
  uint64_t st_h = static_cast<uint64_t>(s->q_stride_head) * 2;
  if (H == 1) st_h = 256;
  if (st_h < 256) return false;
  uint64_t st_t = static_cast<uint64_t>(s->q_stride_tok) * 2;
  if (s->num_tokens == 1) st_t = st_h * H;
  if (st_t < st_h * H) return false;
  const cuuint64_t qd[3] = {128, H, static_cast<cuuint64_t>(s->num_tokens)};
  const cuuint64_t qs[2] = {st_h, st_t};
  const cuuint32_t qb[3] = {64, static_cast<cuuint32_t>(H), static_cast<cuuint32_t>(qsa::ix::kRows / H)};
  return enc(&p->tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), qd, qs, qb, es3,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kH>
cudaError_t launch_ix(const qsa::ix::IxParams& p, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::ix::qsa_indexer_scores_kernel<kH>;
  cudaError_t e = set_smem_once(kernel, qsa::ix::SMEM_BYTES, done);
  if (e != cudaSuccess) return e;
  const int64_t units = ((p.T + p.tpt - 1) / p.tpt) * p.n_chunks;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(units < nsm ? units : nsm);
  kernel<<<grid, qsa::ix::kThreads, qsa::ix::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

template <int kR>
cudaError_t launch_topk(const qsa::ix::TopkParams& p, cudaStream_t stream) {
  static std::atomic<int> done[kMaxDevices];
  auto kernel = qsa::ix::qsa_topk_kernel<kR>;
  cudaError_t e = set_smem_once(kernel, qsa::ix::TK_SMEM, done);
  if (e != cudaSuccess) return e;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(p.T < nsm ? p.T : nsm);
  kernel<<<grid, qsa::ix::kTkThreads, qsa::ix::TK_SMEM, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

qsa_status_t qsa_indexer_scores(const qsa_indexer_shape_t* shape, const void* q_idx, const void* k_idx,
                                const int32_t* positions, const int32_t* seq_start, float* scores,
                                int32_t* status, void* stream) {
  qsa_status_t rc = validate_indexer(shape);
  if (rc != QSA_OK) return rc;
  if (shape->num_tokens == 0) return QSA_OK;
  if (q_idx == nullptr || k_idx == nullptr || positions == nullptr || seq_start == nullptr ||
      scores == nullptr)
    return QSA_ERR_NULL;
  if (shape->q_stride_tok % 8 || shape->q_stride_head % 8 || shape->k_stride_block % 8 ||
      !aligned16(q_idx) || !aligned16(k_idx))
    return QSA_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(scores) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_start) & 3u))
    return QSA_ERR_ALIGN;
  static thread_local qsa::ix::IxParams p;
  if (!make_ix_maps(shape, q_idx, k_idx, &p)) return QSA_ERR_UNSUPPORTED;
  p.positions = positions;
  p.seq_start = seq_start;
  p.scores = scores;
  p.status = status;
  p.T = shape->num_tokens;
  p.ld = shape->score_stride_tok;
  p.NB = static_cast<int32_t>(shape->num_blocks);
  p.H = shape->num_heads;
  p.tpt = qsa::ix::kRows / p.H;
  p.bs = shape->block_size;
  const int64_t tiles = (shape->num_blocks + qsa::ix::kBlk - 1) / qsa::ix::kBlk;
  p.n_chunks = static_cast<int32_t>((tiles + qsa::ix::kTilesPerUnit - 1) / qsa::ix::kTilesPerUnit);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (p.H) {
    case 1: e = launch_ix<1>(p, st); break;
    case 2: e = launch_ix<2>(p, st); break;
    case 4: e = launch_ix<4>(p, st); break;
    default: e = launch_ix<8>(p, st); break;
  }
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

qsa_status_t qsa_indexer_fold_heads(const qsa_indexer_shape_t* shape, const void* q_idx, void* q_folded,
                                    void* stream) {
  qsa_status_t rc = validate_indexer(shape);
  if (rc != QSA_OK) return rc;
  if (shape->num_tokens == 0) return QSA_OK;
  if (q_idx == nullptr || q_folded == nullptr) return QSA_ERR_NULL;
  if (shape->q_stride_tok % 8 || shape->q_stride_head % 8 || !aligned16(q_idx) || !aligned16(q_folded))
    return QSA_ERR_ALIGN;
  qsa::ix::FoldParams p;
  p.q = static_cast<const __nv_bfloat16*>(q_idx);
  p.folded = static_cast<__nv_bfloat16*>(q_folded);
  p.T = shape->num_tokens;
  p.q_st = shape->q_stride_tok;
  p.q_sh = shape->q_stride_head;
  const unsigned grid = static_cast<unsigned>((p.T * 16 + 255) / 256);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (shape->num_heads) {
    case 1: qsa::ix::qsa_indexer_fold_kernel<1><<<grid, 256, 0, st>>>(p); break;
    case 2: qsa::ix::qsa_indexer_fold_kernel<2><<<grid, 256, 0, st>>>(p); break;
    case 4: qsa::ix::qsa_indexer_fold_kernel<4><<<grid, 256, 0, st>>>(p); break;
    default: qsa::ix::qsa_indexer_fold_kernel<8><<<grid, 256, 0, st>>>(p); break;
  }
  return cudaGetLastError() == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

qsa_status_t qsa_topk_select(const qsa_indexer_shape_t* shape, const float* scores,
                             const int32_t* positions, const int32_t* seq_start, int64_t budget,
                             int32_t append_tail, int32_t* lists, int64_t list_stride_tok,
                             int32_t* n_valid, int32_t copies, int32_t* status, void* stream) {
  if (shape == nullptr) return QSA_ERR_NULL;
  if (shape->num_tokens < 0 || shape->num_blocks <= 0 || shape->block_size < 1) return QSA_ERR_SHAPE;
  if (shape->score_stride_tok < shape->num_blocks) return QSA_ERR_SHAPE;
  if (budget < 0 || budget >= 0x7fffffffLL) return QSA_ERR_SHAPE;
  const int64_t width = budget + (append_tail ? 1 : 0);
  if (list_stride_tok < width) return QSA_ERR_SHAPE;
  if (n_valid != nullptr && (copies < 1 || copies > 32)) return QSA_ERR_SHAPE;
  if (shape->num_blocks > 32768) return QSA_ERR_UNSUPPORTED;
  if (shape->num_tokens == 0 || width == 0) {
    if (shape->num_tokens == 0 || n_valid == nullptr) return QSA_OK;
  }
  if (positions == nullptr || seq_start == nullptr || (width > 0 && lists == nullptr)) return QSA_ERR_NULL;
  if (budget > 0 && scores == nullptr) return QSA_ERR_NULL;
  if (!aligned16(scores) || shape->score_stride_tok % 4 != 0 || (reinterpret_cast<uintptr_t>(lists) & 3u) ||
      (reinterpret_cast<uintptr_t>(n_valid) & 3u) || (reinterpret_cast<uintptr_t>(status) & 3u))
    return QSA_ERR_ALIGN;
  qsa::ix::TopkParams p;
  p.scores = scores;
  p.positions = positions;
  p.seq_start = seq_start;
  p.lists = lists;
  p.n_valid = n_valid;
  p.status = status;
  p.T = shape->num_tokens;
  p.ld = shape->score_stride_tok;
  p.list_st = list_stride_tok;
  p.NB = static_cast<int32_t>(shape->num_blocks);
  p.bs = shape->block_size;
  p.budget = static_cast<int32_t>(budget);
  p.width = static_cast<int32_t>(width);
  p.copies = copies;
  p.append_tail = append_tail ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = p.NB <= 16384 ? launch_topk<32>(p, st) : launch_topk<64>(p, st);
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

}  // extern "C"
