/*
 * qsa_oracle.h -- FP64 CPU oracle for QSA top-K sparse-attention prefill.
 *
 * TEST INFRASTRUCTURE ONLY.  This library is the plain, slow, obviously
 * correct definition that the CUDA path is checked against.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may call it.
 * It shares no code, header or constant with the CUDA library.
 *
 * What it computes (page "Qwen4-Exp QSA llega al Ascend de Huawei", section
 * "Lo que realmente añade la pull request"): for every query token t, KV head
 * g and query head h of that head's group,
 *
 *   J     = { j : j < n_valid[t,g] (K when absent), idx[t,g,j] in [0, S) }
 *   s_j   = scale * <q[t,h,:], k[idx_j,g,:]>
 *   out   = sum_j softmax(s)_j * v[idx_j,g,:],  lse = log(sum_j exp(s_j))
 *
 * and for an empty J, out = 0 exactly and lse = -inf (same page, bullet
 * "Límites de tamaño": fully masked rows keep the zero-output convention).
 * The default scale is 1/sqrt(head_dim) (same page: the original D256 scale
 * is kept).  All arithmetic is IEEE double; BF16 inputs are widened exactly.
 */
#ifndef QSA_ORACLE_H
#define QSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int64_t num_tokens;   /* T */
  int64_t num_q_heads;  /* Hq */
  int64_t num_kv_heads; /* Hkv; Hq must be a multiple of Hkv */
  int64_t head_dim;     /* D (any positive value) */
  int64_t topk;         /* K >= 0 */
  int64_t num_slots;    /* S: valid slot ids are [0, S) */
  /* strides in elements */
  int64_t q_stride_tok, q_stride_head;     /* q [T, Hq, D], dim stride 1 */
  int64_t kv_stride_slot, kv_stride_head;  /* k, v [S, Hkv, D], dim stride 1 */
  int64_t idx_stride_tok, idx_stride_head; /* idx [T, Hkv, K], entry stride 1 */
  const uint16_t* q;        /* BF16 bit patterns */
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;       /* -1 (or any negative) = empty entry */
  const int32_t* n_valid;   /* [T, Hkv] contiguous, or NULL meaning K */
  double scale;             /* <= 0 selects 1/sqrt(D) */
  /* Microblock lists (0 or 1 = token lists): entry j names block idx[j], the
   * slots idx[j]*block_size + r, r < block_size; n_valid counts entries. */
  int64_t block_size;
  /* [T] largest visible slot per token (slots above it are empty), or NULL. */
  const int32_t* last_slot;
} qsa_oracle_args;

/*
 * Computes the rows of the tokens listed in `tokens` (n_tokens entries, each
 * in [0, T)).  out is [n_tokens, Hq, D] and lse is [n_tokens, Hq], both
 * contiguous doubles owned by the caller.  n_threads <= 0 uses one thread.
 * Returns the number of list entries that named a slot outside [0, S) (those
 * entries are treated as empty), or -1 on an argument error.
 */
int64_t qsa_oracle_fwd(const qsa_oracle_args* a, const int64_t* tokens,
                       int64_t n_tokens, int n_threads, double* out,
                       double* lse);

/* Exact BF16 -> double widening of one bit pattern (exposed for tests). */
double qsa_oracle_bf16_to_double(uint16_t bits);

#ifdef __cplusplus
}
#endif

#endif
