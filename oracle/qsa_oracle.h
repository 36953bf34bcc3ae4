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
  /* FP8 KV cache (nonzero kv_fp8): k8 / v8 hold OCP FP8 E4M3 bytes with the
   * strides above, k and v are unused; element value = decoded byte times
   * k_scale (v_scale).  The pages name the cache format "fp8_e4m3" only
   * (page "Qwen4-Exp QSA llega al Ascend de Huawei", second of the two
   * observations on the NVIDIA side); the per-tensor scales are the plainest
   * reading of a scaled FP8 cache. */
  int32_t kv_fp8;
  const uint8_t* k8;
  const uint8_t* v8;
  double k_scale;
  double v_scale;
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

/* Exact OCP FP8 E4M3 -> double decoding of one byte (exposed for tests):
 * sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 holds the
 * subnormals m * 2^-9; S.1111.111 is NaN; there are no infinities. */
double qsa_oracle_e4m3_to_double(uint8_t bits);

/* ------------------------------------------------------------------------
 * QSA indexer (page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Por
 * qué QSA es la parte incómoda, en cifras": a multi-query indexer with 4
 * query heads sharing one key head of dim 128, compression ratio 4, a budget
 * of 2048 microblocks per query).  TEST INFRASTRUCTURE ONLY, like the rest of
 * this library.
 *
 * Readings where the page is silent: the score of microblock b for token t
 * is the plain sum over the query heads of <q_idx[t,i,:], k_idx[b,:]>; the
 * candidates of token t are the complete causal microblocks of its sequence,
 * b in [seq_start/bs, (pos+1)/bs); the selection is the `budget` highest
 * scores, ties to the smaller block index.
 * ---------------------------------------------------------------------- */

typedef struct {
  int64_t num_tokens;     /* T */
  int64_t num_heads;      /* indexer query heads (4) */
  int64_t head_dim;       /* 128 */
  int64_t num_blocks;     /* NB: rows of k_idx */
  int64_t block_size;     /* tokens per microblock (4) */
  int64_t q_stride_tok, q_stride_head;   /* q_idx [T, H, Dh] BF16 */
  int64_t k_stride_block;                /* k_idx [NB, Dh] BF16 */
  const uint16_t* q;
  const uint16_t* k;
  const int32_t* positions;              /* [T] slot of the token */
  const int32_t* seq_start;              /* [T] first slot of its sequence */
} qsa_oracle_indexer_args;

/* Candidate range of token t: [*b0, *b1). */
void qsa_oracle_indexer_candidates(const qsa_oracle_indexer_args* a, int64_t t,
                                   int64_t* b0, int64_t* b1);

/* scores [n_tokens, NB] doubles (row of token tokens[i]); entries outside the
 * token's candidate range are -inf.  Returns 0, or -1 on bad arguments. */
int qsa_oracle_indexer_scores(const qsa_oracle_indexer_args* a,
                              const int64_t* tokens, int64_t n_tokens,
                              int n_threads, double* scores);

/* Selection over given FP32 scores [T, ld] (the caller's scores; entries of
 * token t at columns [b0, b1) are its candidates).  Row t of sel holds the
 * chosen block ids in ascending order, then -1 padding; its width is budget,
 * plus one when append_tail is set: then the token's own block pos/bs follows
 * the chosen ones whenever it is incomplete ((pos+1) % bs != 0: a causal tail
 * of 1..bs-1 slots, masked above pos by the attention's last visible slot).
 * count[t] is the number of ids written.  Highest score first, ties to the
 * smaller block index; -0.0 and +0.0 are equal.  Returns 0, or -1. */
int qsa_oracle_topk(const qsa_oracle_indexer_args* a, const float* scores,
                    int64_t ld, int64_t budget, int append_tail, int32_t* sel,
                    int32_t* count);

#ifdef __cplusplus
}
#endif

#endif
