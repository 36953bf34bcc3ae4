/*
 * qsa.h -- C ABI of the B200 (sm_100a) QSA top-K sparse-attention prefill.
 *
 * The operation (page "Qwen4-Exp QSA llega al Ascend de Huawei", section
 * "Lo que realmente añade la pull request", and its bullets "Hardware y tipo
 * de dato", "Formas de cabeza", "Límites de tamaño"): for every query token t
 * and KV head g, with G = Hq / Hkv query heads per KV head (query head h uses
 * KV head h / G), attention restricted to the cache rows named by the
 * token's selected-slot list:
 *
 *   J        = { j < n_valid[t,g] (K when n_valid is NULL) : 0 <= idx[t,g,j] < S }
 *   s_j      = scale * < q[t,h,:], k_cache[idx[t,g,j], g, :] >
 *   out[t,h] = sum_{j in J} softmax_J(s)_j * v_cache[idx[t,g,j], g, :]
 *   lse[t,h] = log( sum_{j in J} exp(s_j) )           (natural log, FP32)
 *
 * The Q and K inputs are already rotated (RoPE applied); list order does not
 * matter, -1 marks an empty entry anywhere in a list (interior -1 included);
 * a row with an empty J gets out = +0.0 exactly and lse = -inf.  The default
 * scale is 1/sqrt(head_dim) = 1/16 (the model's D256 scale).
 *
 * Support set: BF16 Q/K/V/out, head_dim = 256, G in 1..16 (covers the local
 * head shapes (16,2), (24,2), (12,1), (6,1), (3,1)).  Anything else returns
 * QSA_ERR_UNSUPPORTED; there is no fallback path.
 *
 * Conventions for every entry point:
 *  - Device pointers unless stated; the caller owns every buffer.  The
 *    device entry points allocate nothing, free nothing and never
 *    synchronise the host; all work is enqueued on `stream` (a cudaStream_t
 *    passed as void*, NULL = legacy default stream).
 *  - Host-detectable errors are returned before anything is enqueued.
 *    QSA_ERR_CUDA means a CUDA runtime call failed (the launch itself, or a
 *    copy in the host-buffer variant).
 *  - A slot id >= num_slots is treated as empty and sets bit 0 of *status
 *    (a device int32 the caller zeroes; NULL disables the report).  The
 *    kernels never trap.
 *  - All strides are in elements.  Rows of Q, the caches and out must start on
 *    16-byte boundaries: base pointers 16-byte aligned and every stride other
 *    than the innermost a multiple of 8 elements (QSA_ERR_ALIGN otherwise).
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_ABI_VERSION 2

typedef enum {
  QSA_OK = 0,
  QSA_ERR_NULL = 1,        /* a required pointer is NULL */
  QSA_ERR_SHAPE = 2,       /* inconsistent sizes or strides */
  QSA_ERR_UNSUPPORTED = 3, /* head_dim != 256, G > 16, ... */
  QSA_ERR_ALIGN = 4,       /* a row is not 16-byte aligned */
  QSA_ERR_CUDA = 5,        /* a CUDA runtime call failed */
  QSA_ERR_SCRATCH = 6      /* the call needs more scratch than the library's
                              built-in array holds (allocation-free entry point) */
} qsa_status_t;

/* Bits of the device status word. */
#define QSA_STATUS_OOB_SLOT 1 /* some list entry named a slot >= num_slots */
#define QSA_STATUS_TIMEOUT 2  /* a pipeline wait inside the kernel exceeded its
                                 2 s bound; the kernel stopped early and its
                                 outputs are not valid */


typedef struct {
  int64_t num_tokens;     /* T >= 0: query tokens, packed over all sequences
                             (varlen needs no cu_seqlens: ids are physical) */
  int32_t num_q_heads;    /* Hq >= 1 */
  int32_t num_kv_heads;   /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t head_dim;       /* D, must be 256 */
  int32_t topk;           /* K >= 0 entries per list (K == 0: every row empty) */
  int64_t num_slots;      /* S: cache rows; ids outside [0, S) are empty */
  int64_t q_stride_tok, q_stride_head;     /* q       [T, Hq, D]  */
  int64_t kv_stride_slot, kv_stride_head;  /* k_cache, v_cache [S, Hkv, D],
                                              both with these strides */
  int64_t idx_stride_tok, idx_stride_head; /* topk_idx [T, Hkv, K], entries
                                              contiguous; head stride may be 0
                                              (one list shared by all heads) */
  int64_t o_stride_tok, o_stride_head;     /* out     [T, Hq, D]  */
  int64_t lse_stride_tok;                  /* lse     [T, Hq], head stride 1 */
} qsa_shape_t;

/*
 * Sparse prefill forward.
 *   q, k_cache, v_cache : BF16 (__nv_bfloat16 bits), device, layouts above.
 *   topk_idx            : int32 device [T, Hkv, K] physical slot ids, -1 empty.
 *   n_valid             : int32 device [T, Hkv] contiguous (entries at
 *                         positions >= n_valid are empty), or NULL (= K).
 *   scale               : softmax scale; <= 0 selects 1/sqrt(head_dim).
 *   out                 : BF16 device [T, Hq, D] (round to nearest even).
 *   lse                 : FP32 device [T, Hq] natural-log LSE, or NULL.
 *   status              : int32 device word (bit 0: out-of-range id), or NULL.
 *   stream              : cudaStream_t.
 * Enqueues one kernel launch (QSA_KERNEL_AUTO choice, see below).
 * Graph-capturable (no sync, no allocation).
 */
qsa_status_t qsa_sparse_prefill_fwd(const qsa_shape_t* shape, const void* q,
                                    const void* k_cache, const void* v_cache,
                                    const int32_t* topk_idx,
                                    const int32_t* n_valid, float scale,
                                    void* out, float* lse, int32_t* status,
                                    void* stream);

/* Kernel choice for qsa_sparse_prefill_fwd_with. */
typedef enum {
  QSA_KERNEL_AUTO = 0,      /* the tcgen05 kernel when a TMA descriptor can express the
                               Q layout and there is something to gather (K > 0,
                               0 < S < 2^31 - 1), otherwise the warp-MMA kernel */
  QSA_KERNEL_TCGEN05 = 1,   /* persistent warp-specialised cp.async-gather + tcgen05/TMEM
                               kernel only (QSA_ERR_UNSUPPORTED when the layout does not fit) */
  QSA_KERNEL_WARP_MMA = 2   /* cp.async-gather + mma.sync kernel (any valid layout) */
} qsa_kernel_t;

/* Same contract as qsa_sparse_prefill_fwd, with an explicit kernel choice.
 * qsa_sparse_prefill_fwd is this call with QSA_KERNEL_AUTO. */
qsa_status_t qsa_sparse_prefill_fwd_with(const qsa_shape_t* shape, const void* q,
                                         const void* k_cache, const void* v_cache,
                                         const int32_t* topk_idx,
                                         const int32_t* n_valid, float scale,
                                         void* out, float* lse, int32_t* status,
                                         qsa_kernel_t kernel, void* stream);

/*
 * Debug variant of the same kernel (the one QSA_KERNEL_AUTO picks): runs
 * the identical gather stage (same
 * index load, masking and copy addresses) and additionally writes, for
 * every list entry, the slot id of the row the gather actually copied into
 * shared memory (derived from the copy's source address), or -1 where the
 * entry was masked and zero-filled.  gathered_ids is int32 device
 * [T, Hkv, K] contiguous.  out/lse are written as by the forward call.
 */
qsa_status_t qsa_sparse_prefill_debug_gather(
    const qsa_shape_t* shape, const void* q, const void* k_cache,
    const void* v_cache, const int32_t* topk_idx, const int32_t* n_valid,
    float scale, void* out, float* lse, int32_t* status,
    int32_t* gathered_ids, void* stream);

/*
 * Debug dump for every gather path: the kernel of qsa_sparse_prefill_block_fwd
 * (cache_fp8 = 0, BF16 cache) or of qsa_sparse_prefill_fp8_fwd (cache_fp8 !=
 * 0, FP8 E4M3 cache, k_scale / v_scale as there), for token lists
 * (block_size 1, last_slot NULL) or microblock lists, computing out/lse as
 * that call does and additionally writing, for every key, the slot its K and
 * V rows were copied from.  Key j of the list of (t, g) is slot
 * idx[t,g,j / block_size] * block_size + j % block_size; its dump entry is
 * recovered from the source address of the copies the gather issued: the
 * slot, or -1 where the key was masked and its rows zero-filled (entry past
 * n_valid, negative, block or slot past the cache, slot past last_slot[t]),
 * or -2 if the K and V copies of the key disagreed (never expected).
 * gathered_ids is int32 device [T, Hkv, K * block_size] contiguous.  Other
 * arguments and errors as those calls.
 */
qsa_status_t qsa_sparse_prefill_debug_gather_lists(
    const qsa_shape_t* shape, int32_t block_size, const int32_t* last_slot,
    int32_t cache_fp8, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* topk_idx, const int32_t* n_valid, float scale,
    float k_scale, float v_scale, void* out, float* lse, int32_t* status,
    int32_t* gathered_ids, void* stream);

/*
 * Microblock lists (page "Qwen4-Exp QSA llega al Ascend de Huawei", section
 * "Por qué QSA es la parte incómoda, en cifras": QSA selects microblocks,
 * 2048 per query at compression ratio 4).  Entry j of a list names block
 * idx[t,g,j]; the block's block_size consecutive slots idx*block_size + r,
 * r < block_size, are each one key of the attention.  K = shape->topk and
 * n_valid count entries; an entry whose block starts at or beyond S is
 * empty and sets status bit 0; slots of a live block at or beyond S are
 * empty.  last_slot (int32 device [T], or NULL) is the largest slot each
 * token may see: slots above it are empty, which masks the part of the
 * newest block past the query's own position (the causal tail).  block_size
 * is 1, 2, 4, 8 or 16; K * block_size < 2^31.  Runs the tcgen05 kernel only
 * (QSA_ERR_UNSUPPORTED when the Q layout does not fit a TMA descriptor).
 * Other arguments and conventions as qsa_sparse_prefill_fwd.
 */
qsa_status_t qsa_sparse_prefill_block_fwd(const qsa_shape_t* shape,
                                          int32_t block_size,
                                          const int32_t* last_slot,
                                          const void* q, const void* k_cache,
                                          const void* v_cache,
                                          const int32_t* topk_idx,
                                          const int32_t* n_valid, float scale,
                                          void* out, float* lse,
                                          int32_t* status, void* stream);

/*
 * FP8 KV cache (page "Qwen4-Exp QSA llega al Ascend de Huawei", the
 * observations on the NVIDIA side: a KV cache in fp8_e4m3).  k_cache and
 * v_cache hold OCP FP8 E4M3 bytes (finite-only "e4m3fn"; the NaN bytes 0x7f /
 * 0xff give unspecified results) in the layout of qsa_shape_t, strides in
 * elements = bytes; element value = decoded byte * k_scale (v_scale), one
 * scale per tensor.  Q stays BF16; out is BF16; lse is natural-log FP32 of
 * the scaled scores, as for the BF16 cache.  Lists are token lists
 * (block_size 1, last_slot NULL) or microblock lists as in
 * qsa_sparse_prefill_block_fwd.
 *
 * The kernel's tensor cores read the FP8 cache tiles as gathered
 * (tcgen05 kind::f8f6f4).  Both MMA operands are E4M3, so the query (scaled
 * per head by a power of two that puts its largest |q| in [128, 256)) and
 * the softmax probabilities are each written as the sum of two E4M3 terms,
 * hi + lo / 16, with separate FP32 accumulators for the two terms.  The
 * query pair is exact for every element within a factor of about 2^13 of
 * its head's largest |q|; smaller elements lose low bits to E4M3's
 * subnormal floor (an error below 2^-21 times that largest |q|, far below
 * the rounding of the scores).  The probabilities keep 8
 * significant bits, as the BF16 kernel's BF16 P does.  k_scale multiplies the softmax scale and v_scale the
 * normalised output, both in FP32.  Non-finite query elements give
 * unspecified results for their unit.
 *
 * Cache strides (slot and head) must be multiples of 16 elements and the
 * cache bases 16-byte aligned (QSA_ERR_ALIGN otherwise).  Other arguments
 * and conventions as qsa_sparse_prefill_block_fwd.
 */
qsa_status_t qsa_sparse_prefill_fp8_fwd(const qsa_shape_t* shape,
                                        int32_t block_size,
                                        const int32_t* last_slot,
                                        const void* q, const void* k_cache,
                                        const void* v_cache,
                                        const int32_t* topk_idx,
                                        const int32_t* n_valid, float scale,
                                        float k_scale, float v_scale,
                                        void* out, float* lse,
                                        int32_t* status, void* stream);

/*
 * Split-K sparse attention for decode-shaped calls: few query tokens per KV
 * head (one per sequence in decode) with long lists.  Each list is cut into
 * chunks of a multiple of 128 entries; every (token, KV head, chunk) runs on
 * its own CTA of the tcgen05 kernel and writes a normalised partial output and
 * its log-sum-exp to `workspace`; a merge launch then combines the chunks
 *   lse = log sum_c exp(lse_c),  out = sum_c exp(lse_c - lse) out_c,
 * which is the same attention (the combine step of decode context
 * parallelism, page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Dónde
 * encaja esto en el despliegue del servicio de Qwen4Exp", vLLM #59279).
 * Same operation, arguments and conventions as qsa_sparse_prefill_fwd, plus:
 *   num_splits      : chunks per list (never shorter than 128 entries); <= 0
 *                     picks floor(SMs / units) chunks for the (token, KV
 *                     head) units (one wave over the SMs; one chunk once
 *                     the units exceed half the SMs), with chunks of at
 *                     least 256 entries.
 *   workspace       : caller-owned device scratch, 256-byte aligned, of at
 *                     least qsa_sparse_decode_workspace_bytes(shape,
 *                     num_splits) bytes (FP32 partial outputs and lse).  It
 *                     may be NULL when that size is 0 (a single chunk: the
 *                     call then runs the prefill kernel directly).
 * QSA_ERR_SHAPE when workspace_bytes is too small.  Two launches (split
 * kernel, merge kernel) on `stream`; no allocation, no sync.
 */
qsa_status_t qsa_sparse_decode_fwd(const qsa_shape_t* shape, const void* q,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* topk_idx,
                                   const int32_t* n_valid, float scale,
                                   void* out, float* lse, int32_t* status,
                                   int32_t num_splits, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * Split-K decode over an FP8 E4M3 KV cache: qsa_sparse_decode_fwd's chunking,
 * workspace and LSE merge, with the chunks computed by the FP8 kernel of
 * qsa_sparse_prefill_fp8_fwd (element value = stored byte * k_scale /
 * v_scale; token lists).  The workspace size is what
 * qsa_sparse_decode_workspace_bytes returns for the same shape and
 * num_splits.  Cache strides must be multiples of 16 elements (QSA_ERR_ALIGN
 * otherwise).  The pages measure decode over an fp8_e4m3 KV cache on
 * NVIDIA hardware (page "Qwen4-Exp QSA llega al Ascend de Huawei", the
 * observations on the NVIDIA side).
 */
qsa_status_t qsa_sparse_decode_fp8_fwd(const qsa_shape_t* shape, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* topk_idx,
                                       const int32_t* n_valid, float scale,
                                       float k_scale, float v_scale, void* out,
                                       float* lse, int32_t* status,
                                       int32_t num_splits, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Workspace bytes qsa_sparse_decode_fwd needs for this shape and num_splits
 * (0: no workspace needed, or an invalid shape).  With num_splits <= 0 the
 * answer depends on the current device's SM count. */
size_t qsa_sparse_decode_workspace_bytes(const qsa_shape_t* shape,
                                         int32_t num_splits);

/* Chunk count qsa_sparse_decode_fwd will use (0 for an invalid shape). */
int32_t qsa_sparse_decode_num_splits(const qsa_shape_t* shape,
                                     int32_t num_splits);

/*
 * Allocation-free decode.  The pages have no counterpart to this entry
 * point; it exists for callers that cannot call cudaMalloc: code that runs
 * where allocation is forbidden or unsafe (inside a caching allocator's own
 * hooks, a real-time loop that must never block on the driver, an embedding
 * runtime that owns every device allocation), and callers with no allocator
 * at all.  It computes exactly what qsa_sparse_decode_fwd computes, but its
 * scratch space (the partial outputs of the chunks) is a fixed array of
 * QSA_NOALLOC_SCRATCH_BYTES compiled into the library, so the caller passes
 * only inputs and outputs.
 *
 * Cost and limits:
 *  - Every GPU on which the library's device code is loaded holds the
 *    array (16 MiB) until the process exits.
 *  - Calls whose chunks need more than the array holds (see
 *    qsa_sparse_decode_workspace_bytes with the same shape and num_splits)
 *    return QSA_ERR_SCRATCH before anything is enqueued.
 *  - The first call on each device (and again after the current context
 *    changes, e.g. after cudaDeviceReset) looks up the array's device
 *    address, which allocates nothing, and caches it with the context.  A
 *    call that needs that lookup while `stream` is being captured returns
 *    QSA_ERR_UNSUPPORTED without enqueuing anything: make one call outside
 *    capture first; captured calls after it are fine.
 *  - All calls in the process share the one array per device: two calls
 *    whose work overlaps on the GPU (different streams, or host threads that
 *    do not order their streams) race on it.  Serialise them.  Nothing in the
 *    array needs to start at zero: every call overwrites each entry before
 *    reading it, and the previous call's contents are simply left behind.
 * Arguments as for qsa_sparse_decode_fwd, without workspace.
 */
#define QSA_NOALLOC_SCRATCH_BYTES (16u << 20)

qsa_status_t qsa_sparse_decode_fwd_noalloc(const qsa_shape_t* shape,
                                           const void* q, const void* k_cache,
                                           const void* v_cache,
                                           const int32_t* topk_idx,
                                           const int32_t* n_valid, float scale,
                                           void* out, float* lse,
                                           int32_t* status, int32_t num_splits,
                                           void* stream);

/* Device staging buffers for the host-buffer entry point (caller-owned,
 * sized for the layouts of `shape`; n_valid / lse / status may be NULL when
 * the matching host pointer is NULL). */
typedef struct {
  void* q;
  void* k_cache;
  void* v_cache;
  int32_t* topk_idx;
  int32_t* n_valid;
  void* out;
  float* lse;
  int32_t* status;
} qsa_device_buffers_t;

/*
 * Host-buffer variant.  Host pointers address buffers laid out exactly like
 * the device ones with the strides of `shape` (each part copied as one
 * contiguous span from its first to its last element); page-locked host
 * memory keeps the copies asynchronous.  The whole K and V caches go up
 * first; the query tokens are then cut into chunks of about 1024 (at most 8
 * chunks), and each chunk's Q / list / n_valid copies, forward kernel and
 * out / lse copies form a pipeline: the copies up and down run on two
 * streams the library keeps per device, overlapping the kernels on
 * `stream` (one chunk and one stream when T < 2048).  Every copy is one
 * cudaMemcpyAsync.  `stream` is ordered after all of it (events), so the
 * caller synchronises `stream` before reading out/lse; the call itself
 * never blocks on the device.  The status word (dev->status) is zeroed on
 * `stream` before the first launch.  Calls on one device are serialised by
 * a lock while they enqueue.
 */
qsa_status_t qsa_sparse_prefill_fwd_host(
    const qsa_shape_t* shape, const void* q_host, const void* k_cache_host,
    const void* v_cache_host, const int32_t* topk_idx_host,
    const int32_t* n_valid_host, float scale, void* out_host,
    float* lse_host, const qsa_device_buffers_t* dev, void* stream);

/*
 * QSA indexer and top-K microblock selection (page "Qwen4-Exp QSA llega al
 * Ascend de Huawei", section "Por qué QSA es la parte incómoda, en cifras":
 * a multi-query indexer, 4 query heads sharing one key head of dim 128, over
 * keys compressed 4x, choosing 2048 microblocks per query).  The page gives
 * the shapes only; this library computes, for query token t with slot
 * position pos[t] in a sequence starting at slot seq_start[t],
 *
 *   candidates(t) = { b : seq_start[t]/bs <= b < (pos[t]+1)/bs, b < NB }
 *                   (the complete causal microblocks; C division)
 *   score(t, b)   = sum_h < q_idx[t,h,:], k_idx[b,:] >   (FP32 accumulate)
 *
 * and selects the `budget` candidates of highest score (ties to the smaller
 * block; -0.0 equals +0.0), listed in ascending block order.  The token's
 * own incomplete block ((pos+1) % bs != 0: a causal tail of 1..bs-1 slots)
 * can follow them; qsa_sparse_prefill_block_fwd with last_slot = pos masks
 * its slots past the token.  Sequences must start on block boundaries.
 */
typedef struct {
  int64_t num_tokens;        /* T >= 0 */
  int32_t num_heads;         /* H: indexer query heads, 1, 2, 4 or 8 */
  int32_t head_dim;          /* must be 128 */
  int64_t num_blocks;        /* NB: rows of k_idx, 1 <= NB < 2^31 */
  int32_t block_size;        /* bs >= 1: slots per microblock (ratio 4) */
  int32_t reserved;          /* 0 */
  int64_t q_stride_tok, q_stride_head;  /* q_idx [T, H, 128] BF16, elements,
                                           multiples of 8 */
  int64_t k_stride_block;               /* k_idx [NB, 128] BF16, multiple of 8 */
  int64_t score_stride_tok;             /* scores [T, ld] FP32, ld >= NB */
} qsa_indexer_shape_t;

/*
 * Indexer scores.  q_idx, k_idx: BF16 device, 16-byte aligned.  positions,
 * seq_start: int32 device [T].  scores: FP32 device [T, ld]; row t is written
 * at the columns of candidates(t) only (all other entries are left as they
 * were).  status: device int32 (bit 1 on an internal timeout) or NULL.  One
 * launch of the persistent tcgen05 kernel on `stream`; no allocation.
 * QSA_ERR_UNSUPPORTED: head_dim != 128, H not in {1,2,4,8}, or a layout a
 * TMA descriptor cannot express.
 */
qsa_status_t qsa_indexer_scores(const qsa_indexer_shape_t* shape,
                                const void* q_idx, const void* k_idx,
                                const int32_t* positions,
                                const int32_t* seq_start, float* scores,
                                int32_t* status, void* stream);

/*
 * Head folding of the indexer query (optional step before
 * qsa_indexer_scores).  The score is linear in the query, so
 * sum_h <q_idx[t,h], k> = <s_t, k> with s_t = sum_h q_idx[t,h] (page "Qwen4-
 * Exp QSA llega al Ascend de Huawei", section "Por qué QSA es la parte
 * incómoda, en cifras": several indexer heads per token over one key head).
 * Writes, per token t and dim d, the FP32 head sum s (heads added in order
 * 0..H-1) as two BF16 values: q_folded[t][0][d] = hi = bf16(s) and
 * q_folded[t][1][d] = lo = bf16(s - hi), round to nearest, so that
 * |s - hi - lo| <= 2^-16 |s| (BF16 keeps 8 significant bits, so each
 * rounding is within 2^-8 of its argument).  q_folded: BF16 device
 * [T, 2, 128] contiguous,
 * caller-owned, 16-byte aligned.  Calling qsa_indexer_scores on it with
 * num_heads = 2 (strides 256 and 128) gives the scores of the H-head query
 * with half the tensor-core work; folding moves a score by at most
 * 2^-16 sum_d |s_d k[b,d]| <= 2^-16 sum_h sum_d |q_idx[t,h,d] k[b,d]|.  Uses num_tokens,
 * num_heads, head_dim and the q strides of `shape` (validated as for
 * qsa_indexer_scores).  One launch; no allocation.
 */
qsa_status_t qsa_indexer_fold_heads(const qsa_indexer_shape_t* shape,
                                    const void* q_idx, void* q_folded,
                                    void* stream);

/*
 * Top-K selection over scores laid out as qsa_indexer_scores writes them
 * (only the candidate columns of each row are read).
 *   budget      : blocks chosen per token, >= 0 (2048 in the model).
 *   append_tail : nonzero appends the token's own incomplete block.
 *   lists       : int32 device [T, list_stride_tok]; row t receives
 *                 width = budget + (append_tail ? 1 : 0) entries: the chosen
 *                 blocks ascending, the tail block, then -1.
 *   n_valid     : int32 device [T, copies] or NULL: the entry count of row t
 *                 written `copies` times (one per KV head of the attention
 *                 that reads the list with head stride 0), copies in 1..32.
 *   status      : device int32 (bit 1 when a row copy timed out) or NULL.
 * scores must be 16-byte aligned with score_stride_tok a multiple of 4
 * (QSA_ERR_ALIGN otherwise): each row's candidate span is copied to shared
 * memory whole, widened to 16-byte boundaries inside the row.  Candidates
 * per token are limited to 32768 (QSA_ERR_UNSUPPORTED when NB is larger).
 * One launch of persistent CTAs; no allocation.  The device memory read is
 * the candidate part of every score row.
 */
qsa_status_t qsa_topk_select(const qsa_indexer_shape_t* shape,
                             const float* scores, const int32_t* positions,
                             const int32_t* seq_start, int64_t budget,
                             int32_t append_tail, int32_t* lists,
                             int64_t list_stride_tok, int32_t* n_valid,
                             int32_t copies, int32_t* status, void* stream);

/* Static description of a status code. */
const char* qsa_status_string(qsa_status_t status);

/* QSA_ABI_VERSION of the built library. */
int32_t qsa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
