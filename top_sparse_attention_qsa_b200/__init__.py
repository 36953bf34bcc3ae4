"""QSA top-K sparse-attention prefill for B200 (sm_100a).

The compute path is libqsa.so (hand-written CUDA kernels behind the C ABI of
include/qsa.h); ``_capi`` is its ctypes binding.  The kernel entry points
are loaded on first use, so ``workloads`` (the seeded input generator)
imports without the library; using a kernel entry point without a built
libqsa.so raises ImportError (there is no fallback).
"""

_API = ("sparse_prefill_fwd", "sparse_prefill_debug_gather", "sparse_prefill_fwd_host",
        "sparse_prefill_block_fwd", "sparse_prefill_fp8_fwd",
        "sparse_decode_fwd", "sparse_decode_fwd_noalloc", "sparse_decode_fp8_fwd",
        "decode_workspace_bytes", "decode_num_splits",
        "indexer_scores", "topk_select", "indexer_select",
        "status_string", "abi_version", "QSAError", "STATUS_OOB_SLOT", "STATUS_TIMEOUT")


def __getattr__(name):
    if name in _API:
        from . import _capi
        return getattr(_capi, name)
    raise AttributeError(name)


__all__ = list(_API)
