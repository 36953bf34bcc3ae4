"""ctypes binding of libqsa.so (include/qsa.h).

Argument marshalling only: tensors become pointers, sizes and strides; every
step of the computation runs in the library's CUDA kernels.  Importing this
module fails loudly when libqsa.so has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m top_sparse_attention_qsa_b200.build` "
        "(the QSA kernels have no CPU or Python fallback)")

_lib = ctypes.CDLL(LIB_PATH)

QSA_OK, QSA_ERR_NULL, QSA_ERR_SHAPE, QSA_ERR_UNSUPPORTED, QSA_ERR_ALIGN, QSA_ERR_CUDA, QSA_ERR_SCRATCH = range(7)
NOALLOC_SCRATCH_BYTES = 16 << 20
STATUS_OOB_SLOT = 1
STATUS_TIMEOUT = 2
KERNEL_AUTO, KERNEL_TCGEN05, KERNEL_WARP_MMA = 0, 1, 2
KERNELS = {"auto": KERNEL_AUTO, "tcgen05": KERNEL_TCGEN05, "warp_mma": KERNEL_WARP_MMA}
HEAD_DIM = 256

# Every symbol include/qsa.h declares.
EXPORTS = ("qsa_sparse_prefill_fwd", "qsa_sparse_prefill_fwd_with", "qsa_sparse_prefill_debug_gather",
           "qsa_sparse_prefill_debug_gather_lists", "qsa_sparse_prefill_block_fwd",
           "qsa_sparse_prefill_fwd_host", "qsa_sparse_decode_fwd", "qsa_sparse_decode_workspace_bytes",
           "qsa_sparse_decode_num_splits", "qsa_sparse_decode_fwd_noalloc",
           "qsa_sparse_prefill_fp8_fwd", "qsa_sparse_decode_fp8_fwd", "qsa_indexer_scores",
           "qsa_indexer_fold_heads", "qsa_topk_select", "qsa_status_string", "qsa_abi_version")


class Shape(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("num_slots", ctypes.c_int64),
        ("q_stride_tok", ctypes.c_int64),
        ("q_stride_head", ctypes.c_int64),
        ("kv_stride_slot", ctypes.c_int64),
        ("kv_stride_head", ctypes.c_int64),
        ("idx_stride_tok", ctypes.c_int64),
        ("idx_stride_head", ctypes.c_int64),
        ("o_stride_tok", ctypes.c_int64),
        ("o_stride_head", ctypes.c_int64),
        ("lse_stride_tok", ctypes.c_int64),
    ]


class IndexerShape(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("num_blocks", ctypes.c_int64),
        ("block_size", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("q_stride_tok", ctypes.c_int64),
        ("q_stride_head", ctypes.c_int64),
        ("k_stride_block", ctypes.c_int64),
        ("score_stride_tok", ctypes.c_int64),
    ]


class DeviceBuffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q", "k_cache", "v_cache", "topk_idx", "n_valid", "out", "lse", "status")]


_vp = ctypes.c_void_p
_lib.qsa_sparse_prefill_fwd.restype = ctypes.c_int
_lib.qsa_sparse_prefill_fwd.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp,
                                        ctypes.c_float, _vp, _vp, _vp, _vp]
_lib.qsa_sparse_prefill_fwd_with.restype = ctypes.c_int
_lib.qsa_sparse_prefill_fwd_with.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp,
                                             ctypes.c_float, _vp, _vp, _vp, ctypes.c_int, _vp]
_lib.qsa_sparse_prefill_debug_gather.restype = ctypes.c_int
_lib.qsa_sparse_prefill_debug_gather.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp,
                                                 ctypes.c_float, _vp, _vp, _vp, _vp, _vp]
_lib.qsa_sparse_prefill_fwd_host.restype = ctypes.c_int
_lib.qsa_sparse_prefill_fwd_host.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp,
                                             ctypes.c_float, _vp, _vp,
                                             ctypes.POINTER(DeviceBuffers), _vp]
_lib.qsa_sparse_decode_fwd.restype = ctypes.c_int
_lib.qsa_sparse_decode_fwd.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                                       _vp, _vp, _vp, ctypes.c_int32, _vp, ctypes.c_size_t, _vp]
_lib.qsa_sparse_decode_workspace_bytes.restype = ctypes.c_size_t
_lib.qsa_sparse_decode_workspace_bytes.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32]
_lib.qsa_sparse_decode_num_splits.restype = ctypes.c_int32
_lib.qsa_sparse_decode_num_splits.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32]
_lib.qsa_sparse_decode_fwd_noalloc.restype = ctypes.c_int
_lib.qsa_sparse_decode_fwd_noalloc.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp,
                                               ctypes.c_float, _vp, _vp, _vp, ctypes.c_int32, _vp]
_lib.qsa_sparse_prefill_debug_gather_lists.restype = ctypes.c_int
_lib.qsa_sparse_prefill_debug_gather_lists.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32, _vp, ctypes.c_int32,
                                                       _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float,
                                                       ctypes.c_float, _vp, _vp, _vp, _vp, _vp]
_lib.qsa_sparse_prefill_block_fwd.restype = ctypes.c_int
_lib.qsa_sparse_prefill_block_fwd.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32, _vp, _vp, _vp, _vp,
                                              _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp]
_lib.qsa_sparse_prefill_fp8_fwd.restype = ctypes.c_int
_lib.qsa_sparse_prefill_fp8_fwd.argtypes = [ctypes.POINTER(Shape), ctypes.c_int32, _vp, _vp, _vp, _vp, _vp,
                                            _vp, ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _vp,
                                            _vp, _vp]
_lib.qsa_sparse_decode_fp8_fwd.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                                           ctypes.c_float, ctypes.c_float, _vp, _vp, _vp, ctypes.c_int32,
                                           _vp, ctypes.c_size_t, _vp]
_lib.qsa_indexer_scores.argtypes = [ctypes.POINTER(IndexerShape), _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.qsa_indexer_fold_heads.argtypes = [ctypes.POINTER(IndexerShape), _vp, _vp, _vp]
_lib.qsa_topk_select.argtypes = [ctypes.POINTER(IndexerShape), _vp, _vp, _vp, ctypes.c_int64, ctypes.c_int32,
                                 _vp, ctypes.c_int64, _vp, ctypes.c_int32, _vp, _vp]
_lib.qsa_status_string.restype = ctypes.c_char_p
_lib.qsa_status_string.argtypes = [ctypes.c_int]
_lib.qsa_abi_version.restype = ctypes.c_int32
_lib.qsa_abi_version.argtypes = []


class QSAError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"qsa status {code}: {status_string(code)}")
        self.code = code


def status_string(code: int) -> str:
    return _lib.qsa_status_string(int(code)).decode()


def abi_version() -> int:
    return int(_lib.qsa_abi_version())


def library():
    return _lib


def _ptr(x: Optional[torch.Tensor]):
    return None if x is None else x.data_ptr()


def _need(x: torch.Tensor, name: str, dtype, device=None, host=False):
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if x.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {x.dtype}")
    if host:
        if x.device.type != "cpu":
            raise ValueError(f"{name} must be a host tensor")
    elif x.device.type != "cuda" or (device is not None and x.device != device):
        raise ValueError(f"{name} must be a CUDA tensor on {device}")


def make_shape(q, k_cache, topk_idx, out, lse=None) -> Shape:
    """Shape/stride descriptor of a call (no checks beyond ranks: the library
    validates sizes, strides and alignment itself)."""
    if q.dim() != 3 or k_cache.dim() != 3 or topk_idx.dim() != 3 or out.dim() != 3:
        raise ValueError("q, caches, topk_idx and out must be 3-d")
    T, Hq, D = q.shape
    S, Hkv, _ = k_cache.shape
    K = topk_idx.shape[2]
    if topk_idx.shape[0] != T or topk_idx.shape[1] != Hkv:
        raise ValueError("topk_idx must be [T, Hkv, K]")
    if tuple(out.shape) != (T, Hq, D):
        raise ValueError("out must be [T, Hq, D]")
    if q.stride(2) != 1 or k_cache.stride(2) != 1 or out.stride(2) != 1 or (K > 1 and topk_idx.stride(2) != 1):
        raise ValueError("innermost dimensions must be contiguous")
    if lse is not None and (tuple(lse.shape) != (T, Hq) or (Hq > 1 and lse.stride(1) != 1)):
        raise ValueError("lse must be [T, Hq] with unit head stride")
    return Shape(T, Hq, Hkv, D, K, S,
                 q.stride(0), q.stride(1), k_cache.stride(0), k_cache.stride(1),
                 topk_idx.stride(0), topk_idx.stride(1), out.stride(0), out.stride(1),
                 lse.stride(0) if lse is not None else Hq)


def _check_kv(k_cache, v_cache):
    if tuple(v_cache.shape) != tuple(k_cache.shape) or v_cache.stride() != k_cache.stride():
        raise ValueError("k_cache and v_cache must have the same shape and strides")


def _raise(rc: int):
    if rc != QSA_OK:
        raise QSAError(rc)


def sparse_prefill_fwd(q, k_cache, v_cache, topk_idx, n_valid=None, scale: float = 0.0,
                       out=None, lse=None, status=None, stream=None, want_lse: bool = True,
                       kernel: str = "auto"):
    """QSA sparse prefill on the GPU.  Returns (out [T,Hq,D] bf16, lse [T,Hq] fp32 or None).
    kernel: "auto" | "tcgen05" | "warp_mma" (see qsa_kernel_t)."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(topk_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = _lib.qsa_sparse_prefill_fwd_with(ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                          _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid),
                                          float(scale), _ptr(out), _ptr(lse), _ptr(status),
                                          KERNELS[kernel], stream)
    _raise(rc)
    return out, lse


def sparse_prefill_debug_gather(q, k_cache, v_cache, topk_idx, n_valid=None, scale: float = 0.0,
                                status=None, stream=None):
    """Same kernel with the gather dump: returns (out, lse, gathered_ids [T,Hkv,K] int32)."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    ids = torch.empty(topk_idx.shape, dtype=torch.int32, device=dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = _lib.qsa_sparse_prefill_debug_gather(ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                              _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid),
                                              float(scale), _ptr(out), _ptr(lse), _ptr(status),
                                              _ptr(ids), stream)
    _raise(rc)
    return out, lse, ids


def sparse_prefill_fwd_host(q, k_cache, v_cache, topk_idx, n_valid, scale, out, lse,
                            dev_bufs: dict, stream=None):
    """Host-buffer entry point: host tensors in and out (pinned for async copies),
    device staging tensors in `dev_bufs` (keys as in qsa_device_buffers_t).
    The library pipelines the copies of token chunks with their kernels on
    its own copy streams and orders `stream` after the last copy down; the
    caller synchronises `stream`."""
    for name, x, dt in (("q", q, torch.bfloat16), ("k_cache", k_cache, torch.bfloat16),
                        ("v_cache", v_cache, torch.bfloat16), ("topk_idx", topk_idx, torch.int32),
                        ("out", out, torch.bfloat16)):
        _need(x, name, dt, host=True)
    _check_kv(k_cache, v_cache)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, host=True)
    if lse is not None:
        _need(lse, "lse", torch.float32, host=True)
    dev = dev_bufs["q"].device
    host = {"q": q, "k_cache": k_cache, "v_cache": v_cache, "topk_idx": topk_idx, "out": out}
    for name, h in host.items():
        d = dev_bufs[name]
        _need(d, "dev." + name, h.dtype, dev)
        if d.stride() != h.stride() or d.shape != h.shape:
            raise ValueError(f"dev.{name} must match the host tensor's shape and strides")
    db = DeviceBuffers(*[_ptr(dev_bufs.get(n)) for n in
                         ("q", "k_cache", "v_cache", "topk_idx", "n_valid", "out", "lse", "status")])
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = _lib.qsa_sparse_prefill_fwd_host(ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                          _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid),
                                          float(scale), _ptr(out), _ptr(lse), ctypes.byref(db),
                                          stream)
    _raise(rc)
    return out, lse


def decode_workspace_bytes(q, k_cache, topk_idx, num_splits: int = 0, out=None, lse=None) -> int:
    """Scratch bytes sparse_decode_fwd needs (0 when a single chunk runs)."""
    if out is None:
        out = q
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    return int(_lib.qsa_sparse_decode_workspace_bytes(ctypes.byref(shape), int(num_splits)))


def decode_num_splits(q, k_cache, topk_idx, num_splits: int = 0) -> int:
    shape = make_shape(q, k_cache, topk_idx, q)
    return int(_lib.qsa_sparse_decode_num_splits(ctypes.byref(shape), int(num_splits)))


def sparse_decode_fwd(q, k_cache, v_cache, topk_idx, n_valid=None, scale: float = 0.0,
                      num_splits: int = 0, workspace=None, out=None, lse=None, status=None,
                      stream=None, want_lse: bool = True):
    """Split-K sparse attention (decode-shaped calls).  `workspace` is a CUDA
    tensor of at least decode_workspace_bytes(...) bytes (allocated here with
    torch when None).  Returns (out, lse)."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(topk_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    need = int(_lib.qsa_sparse_decode_workspace_bytes(ctypes.byref(shape), int(num_splits)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", workspace.dtype, dev)
        ws_bytes = workspace.numel() * workspace.element_size()
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = _lib.qsa_sparse_decode_fwd(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(topk_idx), _ptr(n_valid), float(scale), _ptr(out), _ptr(lse),
                                    _ptr(status), int(num_splits), _ptr(workspace), ws_bytes, stream)
    _raise(rc)
    return out, lse


def sparse_decode_fwd_noalloc(q, k_cache, v_cache, topk_idx, out, lse=None, n_valid=None,
                              scale: float = 0.0, num_splits: int = 0, status=None, stream=None):
    """Allocation-free decode for callers that cannot allocate device memory.

    Same result as sparse_decode_fwd, but the library keeps the chunk
    scratch in its own fixed device array (NOALLOC_SCRATCH_BYTES), and the
    caller provides every output buffer (`out`, optional `lse`), so neither
    this call nor the library allocates.  Concurrent calls on the same device
    must be serialised (they share the array); the first call on a device
    should precede any stream capture.  Raises QSAError(QSA_ERR_SCRATCH) when
    the chunks would not fit."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    _need(out, "out", torch.bfloat16, dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(topk_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = _lib.qsa_sparse_decode_fwd_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                            _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid),
                                            float(scale), _ptr(out), _ptr(lse), _ptr(status),
                                            int(num_splits), stream)
    _raise(rc)
    return out, lse


def sparse_prefill_block_fwd(q, k_cache, v_cache, block_idx, block_size: int, last_slot=None,
                             n_valid=None, scale: float = 0.0, out=None, lse=None, status=None,
                             stream=None, want_lse: bool = True):
    """Microblock lists: block_idx [T, Hkv, E] names blocks of `block_size`
    consecutive slots; last_slot [T] int32 bounds the slots each token sees."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.bfloat16, dev)
    _need(v_cache, "v_cache", torch.bfloat16, dev)
    _need(block_idx, "block_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if last_slot is not None:
        _need(last_slot, "last_slot", torch.int32, dev)
        if not last_slot.is_contiguous() or tuple(last_slot.shape) != (q.shape[0],):
            raise ValueError("last_slot must be a contiguous [T] tensor")
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(block_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, block_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_sparse_prefill_block_fwd(ctypes.byref(shape), int(block_size), _ptr(last_slot),
                                             _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_idx),
                                             _ptr(n_valid), float(scale), _ptr(out), _ptr(lse),
                                             _ptr(status), stream))
    return out, lse


def sparse_prefill_fp8_fwd(q, k_cache, v_cache, topk_idx, k_scale: float = 1.0, v_scale: float = 1.0,
                           n_valid=None, scale: float = 0.0, block_size: int = 1, last_slot=None,
                           out=None, lse=None, status=None, stream=None, want_lse: bool = True):
    """FP8 E4M3 KV cache (torch.float8_e4m3fn [S, Hkv, 256]); element value =
    stored value * k_scale (v_scale).  Token lists (block_size 1) or
    microblock lists with an optional last_slot [T] int32."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.float8_e4m3fn, dev)
    _need(v_cache, "v_cache", torch.float8_e4m3fn, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if last_slot is not None:
        _need(last_slot, "last_slot", torch.int32, dev)
        if not last_slot.is_contiguous() or tuple(last_slot.shape) != (q.shape[0],):
            raise ValueError("last_slot must be a contiguous [T] tensor")
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(topk_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_sparse_prefill_fp8_fwd(ctypes.byref(shape), int(block_size), _ptr(last_slot), _ptr(q),
                                           _ptr(k_cache), _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid),
                                           float(scale), float(k_scale), float(v_scale), _ptr(out),
                                           _ptr(lse), _ptr(status), stream))
    return out, lse


def sparse_prefill_debug_gather_lists(q, k_cache, v_cache, topk_idx, block_size: int = 1, last_slot=None,
                                      n_valid=None, scale: float = 0.0, k_scale: float = 1.0,
                                      v_scale: float = 1.0, status=None, stream=None):
    """The kernel of sparse_prefill_block_fwd (BF16 cache) or
    sparse_prefill_fp8_fwd (float8_e4m3fn cache) with the gather dump:
    returns (out, lse, gathered [T, Hkv, K * block_size] int32), the slot each
    key's rows were copied from, -1 where masked."""
    dev = q.device
    fp8 = k_cache.dtype == torch.float8_e4m3fn
    cdt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", cdt, dev)
    _need(v_cache, "v_cache", cdt, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if last_slot is not None:
        _need_tok(last_slot, "last_slot", q.shape[0], dev)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(topk_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if status is not None:
        _need(status, "status", torch.int32, dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    T, Hkv, K = topk_idx.shape
    ids = torch.empty((T, Hkv, K * int(block_size)), dtype=torch.int32, device=dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_sparse_prefill_debug_gather_lists(
        ctypes.byref(shape), int(block_size), _ptr(last_slot), 1 if fp8 else 0, _ptr(q), _ptr(k_cache),
        _ptr(v_cache), _ptr(topk_idx), _ptr(n_valid), float(scale), float(k_scale), float(v_scale), _ptr(out),
        _ptr(lse), _ptr(status), _ptr(ids), stream))
    return out, lse, ids


def sparse_decode_fp8_fwd(q, k_cache, v_cache, topk_idx, k_scale: float = 1.0, v_scale: float = 1.0,
                          n_valid=None, scale: float = 0.0, num_splits: int = 0, workspace=None, out=None,
                          lse=None, status=None, stream=None, want_lse: bool = True):
    """Split-K decode over an FP8 E4M3 cache (torch.float8_e4m3fn).  A
    workspace of decode_workspace_bytes(...) bytes is allocated when none is
    given."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    _need(k_cache, "k_cache", torch.float8_e4m3fn, dev)
    _need(v_cache, "v_cache", torch.float8_e4m3fn, dev)
    _need(topk_idx, "topk_idx", torch.int32, dev)
    _check_kv(k_cache, v_cache)
    if n_valid is not None:
        _need(n_valid, "n_valid", torch.int32, dev)
        if not n_valid.is_contiguous() or tuple(n_valid.shape) != tuple(topk_idx.shape[:2]):
            raise ValueError("n_valid must be a contiguous [T, Hkv] tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_shape(q, k_cache, topk_idx, out, lse)
    need = int(_lib.qsa_sparse_decode_workspace_bytes(ctypes.byref(shape), int(num_splits)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_sparse_decode_fp8_fwd(ctypes.byref(shape), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(topk_idx), _ptr(n_valid), float(scale), float(k_scale),
                                          float(v_scale), _ptr(out), _ptr(lse), _ptr(status), int(num_splits),
                                          _ptr(workspace), ws_bytes, stream))
    return out, lse


# ------------------------------------------------------------------ indexer

INDEXER_HEAD_DIM = 128
TOPK_MAX_CANDIDATES = 32768


def make_indexer_shape(q_idx, k_idx, block_size: int, scores=None) -> IndexerShape:
    """Shape/stride descriptor of an indexer call: q_idx [T, H, 128],
    k_idx [NB, 128] (BF16), scores [T, ld] (FP32)."""
    if q_idx.dim() != 3 or k_idx.dim() != 2:
        raise ValueError("q_idx must be [T, H, Dh] and k_idx [NB, Dh]")
    T, H, Dh = q_idx.shape
    NB = k_idx.shape[0]
    if k_idx.shape[1] != Dh:
        raise ValueError("q_idx and k_idx head dims differ")
    if q_idx.stride(2) != 1 or k_idx.stride(1) != 1:
        raise ValueError("innermost dimensions must be contiguous")
    ld = NB
    if scores is not None:
        if scores.dim() != 2 or scores.shape[0] != T or scores.shape[1] < NB or scores.stride(1) != 1:
            raise ValueError("scores must be [T, >= NB] with unit column stride")
        ld = scores.stride(0)
    return IndexerShape(T, H, Dh, NB, int(block_size), 0, q_idx.stride(0), q_idx.stride(1),
                        k_idx.stride(0), ld)


def _need_tok(x, name, T, dev):
    _need(x, name, torch.int32, dev)
    if not x.is_contiguous() or tuple(x.shape) != (T,):
        raise ValueError(f"{name} must be a contiguous [T] int32 tensor")


def indexer_fold_heads(q_idx, k_idx, out=None, stream=None):
    """The head sum of q_idx [T, H, 128] as two BF16 terms: [T, 2, 128]
    (hi = bf16(s), lo = bf16(s - hi)), a two-head query with the same scores."""
    dev = q_idx.device
    _need(q_idx, "q_idx", torch.bfloat16, dev)
    T = q_idx.shape[0]
    if out is None:
        out = torch.empty((T, 2, q_idx.shape[2]), dtype=torch.bfloat16, device=dev)
    _need(out, "q_folded", torch.bfloat16, dev)
    if not out.is_contiguous() or tuple(out.shape) != (T, 2, q_idx.shape[2]):
        raise ValueError("q_folded must be a contiguous [T, 2, Dh] tensor")
    shape = make_indexer_shape(q_idx, k_idx, 1)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_indexer_fold_heads(ctypes.byref(shape), _ptr(q_idx), _ptr(out), stream))
    return out


def indexer_scores(q_idx, k_idx, positions, seq_start, block_size: int = 4, scores=None, status=None,
                   stream=None, fold=None, q_folded=None):
    """FP32 scores [T, NB]: sum over the H indexer heads of <q_idx[t,h], k_idx[b]>
    at the complete causal microblocks of each token (other entries untouched;
    a new buffer starts as -inf).  With `fold` (default: H >= 4) the heads
    are first summed into a two-term BF16 query (qsa_indexer_fold_heads,
    into `q_folded` when given) and the scores computed from that."""
    dev = q_idx.device
    _need(q_idx, "q_idx", torch.bfloat16, dev)
    _need(k_idx, "k_idx", torch.bfloat16, dev)
    if fold is None:
        fold = q_idx.dim() == 3 and q_idx.shape[1] >= 4
    if fold:
        q_idx = indexer_fold_heads(q_idx, k_idx, out=q_folded, stream=stream)
    T = q_idx.shape[0]
    _need_tok(positions, "positions", T, dev)
    _need_tok(seq_start, "seq_start", T, dev)
    if scores is None:
        # rows padded to a multiple of 4 floats: the selection copies 16-byte spans
        NB = k_idx.shape[0]
        scores = torch.full((T, (NB + 3) // 4 * 4), float("-inf"), dtype=torch.float32, device=dev)[:, :NB]
    _need(scores, "scores", torch.float32, dev)
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = make_indexer_shape(q_idx, k_idx, block_size, scores)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_indexer_scores(ctypes.byref(shape), _ptr(q_idx), _ptr(k_idx), _ptr(positions),
                                   _ptr(seq_start), _ptr(scores), _ptr(status), stream))
    return scores


def topk_select(scores, positions, seq_start, num_blocks: int, budget: int, block_size: int = 4,
                append_tail: bool = False, lists=None, n_valid=None, copies: int = 1, status=None,
                stream=None):
    """Ascending block ids of the `budget` highest-scoring candidates of each
    token (ties to the smaller block), then with `append_tail` the token's own
    incomplete block, -1 padded: lists [T, budget (+1)] int32, and the entry
    count per token written `copies` times: n_valid [T, copies] int32."""
    dev = scores.device
    _need(scores, "scores", torch.float32, dev)
    T = scores.shape[0]
    _need_tok(positions, "positions", T, dev)
    _need_tok(seq_start, "seq_start", T, dev)
    width = int(budget) + (1 if append_tail else 0)
    if lists is None:
        lists = torch.empty((T, width), dtype=torch.int32, device=dev)
    _need(lists, "lists", torch.int32, dev)
    if lists.dim() != 2 or lists.shape[0] != T or lists.shape[1] < width or (width > 1 and lists.stride(1) != 1):
        raise ValueError("lists must be [T, >= width] with unit column stride")
    if n_valid is None:
        n_valid = torch.empty((T, copies), dtype=torch.int32, device=dev)
    _need(n_valid, "n_valid", torch.int32, dev)
    if not n_valid.is_contiguous() or tuple(n_valid.shape) != (T, copies):
        raise ValueError("n_valid must be a contiguous [T, copies] tensor")
    if scores.dim() != 2 or scores.shape[1] < num_blocks or (scores.shape[1] > 1 and scores.stride(1) != 1):
        raise ValueError("scores must be [T, >= num_blocks] with unit column stride")
    if status is not None:
        _need(status, "status", torch.int32, dev)
    shape = IndexerShape(T, 0, INDEXER_HEAD_DIM, int(num_blocks), int(block_size), 0, 0, 0, 0, scores.stride(0))
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    _raise(_lib.qsa_topk_select(ctypes.byref(shape), _ptr(scores), _ptr(positions), _ptr(seq_start),
                                int(budget), 1 if append_tail else 0, _ptr(lists), lists.stride(0),
                                _ptr(n_valid), int(copies), _ptr(status), stream))
    return lists, n_valid


def indexer_select(q_idx, k_idx, positions, seq_start, budget: int, block_size: int = 4,
                   append_tail: bool = True, copies: int = 1, scores=None, stream=None):
    """Indexer scores then top-K selection (two launches); returns
    (lists, n_valid, scores)."""
    scores = indexer_scores(q_idx, k_idx, positions, seq_start, block_size, scores=scores, stream=stream)
    lists, nv = topk_select(scores, positions, seq_start, k_idx.shape[0], budget, block_size, append_tail,
                            copies=copies, stream=stream)
    return lists, nv, scores
