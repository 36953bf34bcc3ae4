/*
 * qsa_oracle.c -- FP64 CPU oracle for QSA top-K sparse-attention prefill.
 *
 * TEST INFRASTRUCTURE ONLY (see qsa_oracle.h).  Written directly from the
 * definition on page "Qwen4-Exp QSA llega al Ascend de Huawei", section
 * "Lo que realmente añade la pull request": attention restricted to the
 * cache rows named by the token's selected-slot list, softmax with the model's
 * D256 scale.  Nothing here is blocked, fused or reordered beyond the plain
 * definition; threads only split the independent query tokens.
 */
#include "qsa_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

double qsa_oracle_bf16_to_double(uint16_t bits) {
  /* BF16 is the top half of an IEEE binary32; the widening is exact. */
  uint32_t w = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

double qsa_oracle_e4m3_to_double(uint8_t bits) {
  const int sign = bits >> 7, e = (bits >> 3) & 15, m = bits & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

typedef struct {
  const qsa_oracle_args* a;
  const int64_t* tokens;
  int64_t n_tokens;
  double* out;
  double* lse;
  int64_t next;      /* shared work counter */
  int64_t oob;       /* out-of-range entries seen */
  int error;
} job_t;

/* One (token, query head) row, following the definition step by step. */
static int64_t one_row(const qsa_oracle_args* a, int64_t t, int64_t h,
                       double* out_row, double* lse_out, int64_t* sel,
                       double* s) {
  const int64_t D = a->head_dim;
  const int64_t G = a->num_q_heads / a->num_kv_heads;
  const int64_t g = h / G; /* contiguous GQA grouping */
  const double scale = a->scale > 0.0 ? a->scale : 1.0 / sqrt((double)D);
  int64_t oob = 0;

  /* Step 1: the selected entries J.  n_valid and negative ids both mask. */
  int64_t n_list = a->topk;
  if (a->n_valid) {
    int64_t nv = a->n_valid[t * a->num_kv_heads + g];
    if (nv < n_list) n_list = nv;
    if (n_list < 0) n_list = 0;
  }
  const int32_t* list = a->idx + t * a->idx_stride_tok + g * a->idx_stride_head;
  /* Microblock lists: entry j covers block_size consecutive slots, each a key
   * (page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Por qué QSA es
   * la parte incómoda, en cifras": QSA selects at microblock granularity). */
  const int64_t bs = a->block_size > 1 ? a->block_size : 1;
  const int64_t limit = a->last_slot ? a->last_slot[t] : INT64_MAX;
  int64_t n = 0;
  for (int64_t j = 0; j < n_list; ++j) {
    int64_t id = list[j];
    if (id < 0) continue;
    if (id * bs >= a->num_slots) {
      if (h % G == 0) ++oob; /* count each list entry once, not per head */
      continue;
    }
    for (int64_t r = 0; r < bs; ++r) {
      const int64_t slot = id * bs + r;
      if (slot >= a->num_slots || slot > limit) continue;
      sel[n++] = slot;
    }
  }

  /* Empty selection: zero output, lse = -inf. */
  if (n == 0) {
    for (int64_t d = 0; d < D; ++d) out_row[d] = 0.0;
    *lse_out = -INFINITY;
    return oob;
  }

  /* Step 2: scores s_j = scale * <q, k_j>. */
  const uint16_t* q = a->q + t * a->q_stride_tok + h * a->q_stride_head;
  for (int64_t j = 0; j < n; ++j) {
    double dot = 0.0;
    if (a->kv_fp8) {
      const uint8_t* kb = a->k8 + sel[j] * a->kv_stride_slot + g * a->kv_stride_head;
      for (int64_t d = 0; d < D; ++d)
        dot += qsa_oracle_bf16_to_double(q[d]) * (qsa_oracle_e4m3_to_double(kb[d]) * a->k_scale);
    } else {
      const uint16_t* kr = a->k + sel[j] * a->kv_stride_slot + g * a->kv_stride_head;
      for (int64_t d = 0; d < D; ++d)
        dot += qsa_oracle_bf16_to_double(q[d]) * qsa_oracle_bf16_to_double(kr[d]);
    }
    s[j] = scale * dot;
  }

  /* Step 3: softmax with the maximum subtracted (exact in real arithmetic). */
  double m = s[0];
  for (int64_t j = 1; j < n; ++j) if (s[j] > m) m = s[j];
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) { s[j] = exp(s[j] - m); l += s[j]; }

  /* Step 4: weighted sum of the selected V rows, normalised by l. */
  for (int64_t d = 0; d < D; ++d) out_row[d] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    const double p = s[j];
    if (a->kv_fp8) {
      const uint8_t* vb = a->v8 + sel[j] * a->kv_stride_slot + g * a->kv_stride_head;
      for (int64_t d = 0; d < D; ++d) out_row[d] += p * (qsa_oracle_e4m3_to_double(vb[d]) * a->v_scale);
    } else {
      const uint16_t* vr = a->v + sel[j] * a->kv_stride_slot + g * a->kv_stride_head;
      for (int64_t d = 0; d < D; ++d) out_row[d] += p * qsa_oracle_bf16_to_double(vr[d]);
    }
  }
  for (int64_t d = 0; d < D; ++d) out_row[d] /= l;
  *lse_out = m + log(l);
  return oob;
}

static void* worker(void* arg) {
  job_t* job = (job_t*)arg;
  const qsa_oracle_args* a = job->a;
  const int64_t Hq = a->num_q_heads, D = a->head_dim;
  const int64_t cap = (a->topk > 0 ? a->topk : 1) * (a->block_size > 1 ? a->block_size : 1);
  int64_t* sel = (int64_t*)malloc((size_t)cap * sizeof(int64_t));
  double* s = (double*)malloc((size_t)cap * sizeof(double));
  if (!sel || !s) {
    free(sel); free(s);
    __atomic_store_n(&job->error, 1, __ATOMIC_RELAXED);
    return NULL;
  }
  int64_t oob = 0;
  for (;;) {
    int64_t i = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
    if (i >= job->n_tokens) break;
    const int64_t t = job->tokens[i];
    for (int64_t h = 0; h < Hq; ++h)
      oob += one_row(a, t, h, job->out + (i * Hq + h) * D, job->lse + i * Hq + h, sel, s);
  }
  __atomic_fetch_add(&job->oob, oob, __ATOMIC_RELAXED);
  free(sel); free(s);
  return NULL;
}

int64_t qsa_oracle_fwd(const qsa_oracle_args* a, const int64_t* tokens,
                       int64_t n_tokens, int n_threads, double* out,
                       double* lse) {
  if (!a || n_tokens < 0 || (n_tokens > 0 && (!tokens || !out || !lse))) return -1;
  if (a->num_kv_heads <= 0 || a->num_q_heads <= 0 || a->head_dim <= 0 ||
      a->num_q_heads % a->num_kv_heads != 0 || a->topk < 0 || a->num_slots < 0)
    return -1;
  const int has_kv = a->kv_fp8 ? (a->k8 && a->v8) : (a->k && a->v);
  if (n_tokens > 0 && (!a->q || (a->topk > 0 && (!a->idx || !has_kv)))) return -1;
  for (int64_t i = 0; i < n_tokens; ++i)
    if (tokens[i] < 0 || tokens[i] >= a->num_tokens) return -1;

  job_t job;
  memset(&job, 0, sizeof job);
  job.a = a; job.tokens = tokens; job.n_tokens = n_tokens; job.out = out; job.lse = lse;

  if (n_threads <= 1 || n_tokens <= 1) {
    worker(&job);
  } else {
    if (n_threads > n_tokens) n_threads = (int)n_tokens;
    pthread_t* th = (pthread_t*)malloc((size_t)n_threads * sizeof(pthread_t));
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
      if (pthread_create(&th[i], NULL, worker, &job) != 0) break;
      ++started;
    }
    if (started == 0) worker(&job);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  if (job.error) return -1;
  return job.oob;
}

/* ------------------------------------------------------------------------
 * QSA indexer: candidate scores and top-budget selection.
 * ---------------------------------------------------------------------- */

void qsa_oracle_indexer_candidates(const qsa_oracle_indexer_args* a, int64_t t,
                                   int64_t* b0, int64_t* b1) {
  const int64_t bs = a->block_size > 0 ? a->block_size : 1;
  int64_t lo = a->seq_start[t] / bs;
  int64_t hi = ((int64_t)a->positions[t] + 1) / bs; /* complete blocks only */
  if (hi > a->num_blocks) hi = a->num_blocks;
  if (lo < 0) lo = 0;
  if (hi < lo) hi = lo;
  *b0 = lo;
  *b1 = hi;
}

int qsa_oracle_indexer_scores(const qsa_oracle_indexer_args* a,
                              const int64_t* tokens, int64_t n_tokens,
                              int n_threads, double* scores) {
  (void)n_threads;
  if (!a || (n_tokens > 0 && (!tokens || !scores || !a->q || !a->k))) return -1;
  const int64_t NB = a->num_blocks, Dh = a->head_dim;
  for (int64_t i = 0; i < n_tokens; ++i) {
    const int64_t t = tokens[i];
    if (t < 0 || t >= a->num_tokens) return -1;
    int64_t b0, b1;
    qsa_oracle_indexer_candidates(a, t, &b0, &b1);
    double* row = scores + i * NB;
    for (int64_t b = 0; b < NB; ++b) row[b] = -INFINITY;
    for (int64_t b = b0; b < b1; ++b) {
      const uint16_t* kr = a->k + b * a->k_stride_block;
      double sum = 0.0;
      for (int64_t h = 0; h < a->num_heads; ++h) {
        const uint16_t* qr = a->q + t * a->q_stride_tok + h * a->q_stride_head;
        double dot = 0.0;
        for (int64_t d = 0; d < Dh; ++d)
          dot += qsa_oracle_bf16_to_double(qr[d]) * qsa_oracle_bf16_to_double(kr[d]);
        sum += dot;
      }
      row[b] = sum;
    }
  }
  return 0;
}

typedef struct {
  float score;
  int64_t block;
} scored_t;

/* Higher score first; equal scores: smaller block first. */
static int by_score_then_index(const void* x, const void* y) {
  const scored_t* a = (const scored_t*)x;
  const scored_t* b = (const scored_t*)y;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->block > b->block) - (a->block < b->block);
}

static int by_block(const void* x, const void* y) {
  const int32_t a = *(const int32_t*)x, b = *(const int32_t*)y;
  return (a > b) - (a < b);
}

int qsa_oracle_topk(const qsa_oracle_indexer_args* a, const float* scores,
                    int64_t ld, int64_t budget, int append_tail, int32_t* sel,
                    int32_t* count) {
  if (!a || !scores || !sel || !count || budget < 0) return -1;
  const int64_t bs = a->block_size > 0 ? a->block_size : 1;
  const int64_t width = budget + (append_tail ? 1 : 0);
  scored_t* buf = (scored_t*)malloc((size_t)(a->num_blocks > 0 ? a->num_blocks : 1) * sizeof(scored_t));
  if (!buf) return -1;
  for (int64_t t = 0; t < a->num_tokens; ++t) {
    int64_t b0, b1;
    qsa_oracle_indexer_candidates(a, t, &b0, &b1);
    int64_t n = 0;
    for (int64_t b = b0; b < b1; ++b) {
      buf[n].score = scores[t * ld + b];
      buf[n].block = b;
      ++n;
    }
    qsort(buf, (size_t)n, sizeof(scored_t), by_score_then_index);
    int64_t k = n < budget ? n : budget;
    int32_t* out = sel + t * width;
    for (int64_t j = 0; j < k; ++j) out[j] = (int32_t)buf[j].block;
    qsort(out, (size_t)k, sizeof(int32_t), by_block);
    if (append_tail && ((int64_t)a->positions[t] + 1) % bs != 0)
      out[k++] = (int32_t)((int64_t)a->positions[t] / bs);
    for (int64_t j = k; j < width; ++j) out[j] = -1;
    count[t] = (int32_t)k;
  }
  free(buf);
  return 0;
}
