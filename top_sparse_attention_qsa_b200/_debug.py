"""ctypes binding of libqsa_debug.so (include/qsa_debug.h): the measurement
kernels and test hooks that the production library leaves out.

Argument marshalling only.  Importing this module fails loudly when
libqsa_debug.so has not been built (`python -m top_sparse_attention_qsa_b200.build`
builds both libraries).
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _capi
from ._capi import QSAError, _check_kv, _need, _ptr, make_shape

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqsa_debug.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m top_sparse_attention_qsa_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

# Every symbol include/qsa_debug.h declares.
EXPORTS = ("qsa_debug_gather_only", "qsa_debug_gather_peak", "qsa_test_stalled_pipeline",
           "qsa_debug_abi_version")

PEAK_CP_ASYNC, PEAK_LD_V4, PEAK_BULK = 0, 1, 2
PEAK_METHODS = {"cp_async": PEAK_CP_ASYNC, "ld_v4": PEAK_LD_V4, "bulk": PEAK_BULK}

_vp = ctypes.c_void_p
_Shape = ctypes.POINTER(_capi.Shape)
_lib.qsa_debug_gather_only.restype = ctypes.c_int
_lib.qsa_debug_gather_only.argtypes = [_Shape, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.qsa_debug_gather_peak.restype = ctypes.c_int
_lib.qsa_debug_gather_peak.argtypes = [_vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, _vp, ctypes.c_int64,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp,
                                       ctypes.c_int64, _vp, _vp]
_lib.qsa_test_stalled_pipeline.restype = ctypes.c_int
_lib.qsa_test_stalled_pipeline.argtypes = [_Shape, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp]
_lib.qsa_debug_abi_version.restype = ctypes.c_int32
_lib.qsa_debug_abi_version.argtypes = []


def library():
    return _lib


def abi_version() -> int:
    return int(_lib.qsa_debug_abi_version())


def _raise(rc: int):
    if rc != _capi.QSA_OK:
        raise QSAError(rc)


def gather_only(q, k_cache, v_cache, topk_idx, n_valid=None, status=None, stream=None):
    """The KV gather of the tcgen05 prefill kernel (BF16 cache) or of the FP8
    kernel (float8_e4m3fn cache) alone, over token lists: the floor of that
    kernel on the same lists.  Writes nothing but the status word."""
    dev = q.device
    fp8 = k_cache.dtype == torch.float8_e4m3fn
    cdt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", cdt, dev)
    _need(v_cache, "v_cache", cdt, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, topk_idx, q)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_debug_gather_only(ctypes.byref(shape), 1 if fp8 else 0, _ptr(q), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid), _ptr(status), stream))


def gather_peak(table, ids, row_bytes: int, method: str = "cp_async", depth: int = 4, warps: int = 8,
                ctas_per_sm: int = 1, sink=None, status=None, stream=None):
    """Random-row gather rate probe: reads rows `ids` (int32) of `table`
    (a CUDA tensor whose dim 0 indexes rows; row_bytes of each row are read)
    into the SMs.  `sink` (uint32/int32 CUDA tensor, >= grid x threads words)
    is needed for method "ld_v4"."""
    dev = table.device
    if table.device.type != "cuda" or ids.device != dev or ids.dtype != torch.int32:
        raise ValueError("table and ids must be CUDA tensors on one device, ids int32")
    if not ids.is_contiguous():
        raise ValueError("ids must be contiguous")
    rows = table.shape[0]
    stride = table.stride(0) * table.element_size()
    sink_words = 0 if sink is None else sink.numel()
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_debug_gather_peak(_ptr(table), rows, stride, int(row_bytes), _ptr(ids), ids.numel(),
                                      PEAK_METHODS[method], int(depth), int(warps), int(ctas_per_sm),
                                      _ptr(sink), sink_words, _ptr(status), stream))


def run_stalled_pipeline_check(q, k_cache, v_cache, topk_idx, status, n_valid=None, scale: float = 0.0,
                               stream=None):
    """Failure-detection hook: runs the tcgen05 kernel with one pipeline signal
    withheld; the kernel must stop on its own and set STATUS_TIMEOUT in `status`."""
    dev = q.device
    for name, x, dt in (("q", q, torch.bfloat16), ("k_cache", k_cache, torch.bfloat16),
                        ("v_cache", v_cache, torch.bfloat16), ("topk_idx", topk_idx, torch.int32),
                        ("status", status, torch.int32)):
        _need(x, name, dt, dev)
    _check_kv(k_cache, v_cache)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_test_stalled_pipeline(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(topk_idx), _ptr(n_valid), float(scale), _ptr(out),
                                          _ptr(lse), _ptr(status), stream))
