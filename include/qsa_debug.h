/*
 * qsa_debug.h -- measurement kernels and test hooks of the QSA library.
 *
 * These entry points are not part of the production library (libqsa.so).
 * They are built, with the QSA_DEBUG flag, into a second library,
 * libqsa_debug.so, which the test suite and the benchmark load next to it.
 * Nothing here is needed to compute attention.  Conventions (device
 * pointers, status codes, `stream` as void*) are those of qsa.h.
 */
#ifndef QSA_DEBUG_H
#define QSA_DEBUG_H

#include <stddef.h>
#include <stdint.h>

#include "qsa.h"

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_DEBUG_ABI_VERSION 1

/*
 * The KV gather of a prefill kernel, alone.  Runs the producer warps of the
 * tcgen05 prefill kernel (cache_fp8 = 0: BF16 cache, 512-byte rows) or of
 * the FP8 kernel (cache_fp8 != 0: E4M3 cache, 256-byte rows) over token
 * lists, with the same list reads, masking, 16-byte cp.async copies and
 * shared-memory ring, and a consumer warp that hands every ring slot back
 * as soon as it is full.  It writes nothing to global memory except out-of-
 * range ids into *status (bit 0).  Its time over a workload is the floor
 * the full prefill kernel could reach with free compute.  Arguments as for
 * qsa_sparse_prefill_fwd (FP8 cache strides must be multiples of 16);
 * QSA_ERR_UNSUPPORTED when the Q layout does not fit a TMA descriptor.
 */
qsa_status_t qsa_debug_gather_only(const qsa_shape_t* shape, int32_t cache_fp8,
                                   const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* topk_idx,
                                   const int32_t* n_valid, int32_t* status,
                                   void* stream);

/* Methods of qsa_debug_gather_peak. */
#define QSA_PEAK_CP_ASYNC 0 /* 16-byte cp.async per lane into a per-warp ring
                               of `depth` groups of 4 KB (depth 1, 2, 4 or 8) */
#define QSA_PEAK_LD_V4 1    /* 16-byte ld.global.cg.v4 per lane, `depth`
                               loads in flight per lane (4, 8 or 16; at most
                               16 warps per CTA for 16) */
#define QSA_PEAK_BULK 2     /* one 1-d cp.async.bulk per row, per-warp ring of
                               `depth` stages of 32 rows (1 to 4) */

/*
 * Random-row gather rate of the GPU, written independently of the prefill
 * kernels: reads rows ids[0 .. n_ids) of `table` (rows of row_bytes = 256
 * or 512 bytes, row_stride_bytes apart, a multiple of 16) into the SMs with
 * the given method, on a grid of (SM count x ctas_per_sm) CTAs of
 * 32 x warps threads, each CTA taking a contiguous share of the id list.
 * Only whole groups of ids are read (8 or 16 rows for QSA_PEAK_CP_ASYNC,
 * depth x 512 / row_bytes for QSA_PEAK_LD_V4, 32 for QSA_PEAK_BULK); the
 * bytes moved are therefore at most n_ids x row_bytes, and exactly that
 * when n_ids is a multiple of 1024.  Ids outside [0, rows) read row 0.
 *   sink       : QSA_PEAK_LD_V4 only: device uint32 array of sink_words >=
 *                grid x threads words (one folded word per thread keeps the
 *                loads live); may be NULL otherwise.
 *   status     : device int32 or NULL; bit 1 when a bounded wait of
 *                QSA_PEAK_BULK ran out (2 s).
 * QSA_ERR_UNSUPPORTED: an unsupported row_bytes / method / depth, more than
 * 1024 threads per SM (warps x 32 x ctas_per_sm), or a shared-memory ring
 * larger than one SM holds.  One launch; no allocation.
 */
qsa_status_t qsa_debug_gather_peak(const void* table, int64_t rows,
                                   int64_t row_stride_bytes, int32_t row_bytes,
                                   const int32_t* ids, int64_t n_ids,
                                   int32_t method, int32_t depth, int32_t warps,
                                   int32_t ctas_per_sm, uint32_t* sink,
                                   int64_t sink_words, int32_t* status,
                                   void* stream);

/*
 * Failure-detection test hook.  Runs the tcgen05 prefill kernel on the given
 * buffers with the producers' completion signal for the first shared-memory
 * slot of every CTA withheld, so that no pipeline stage can ever complete.
 * Every wait inside the kernel is bounded (2 s), so the kernel must end on
 * its own, with QSA_STATUS_TIMEOUT set in *status (required here) and the
 * CUDA context still usable; out/lse are left unspecified.  Same arguments
 * as qsa_sparse_prefill_fwd; QSA_ERR_UNSUPPORTED when the tcgen05 kernel
 * cannot take the layout.
 */
qsa_status_t qsa_test_stalled_pipeline(const qsa_shape_t* shape, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* topk_idx,
                                       const int32_t* n_valid, float scale,
                                       void* out, float* lse, int32_t* status,
                                       void* stream);

/* QSA_DEBUG_ABI_VERSION of the built library. */
int32_t qsa_debug_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_DEBUG_H */
