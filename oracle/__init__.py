"""FP64 CPU oracle for QSA top-K sparse-attention prefill.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package.  It is the plain, slow
definition the CUDA library is checked against and shares no code with it.

The arithmetic lives in ``qsa_oracle.c`` (plain C, IEEE double); this module
compiles it with gcc and marshals numpy/torch-CPU arrays into its C struct.

What it computes (page "Qwen4-Exp QSA llega al Ascend de Huawei", section
"Lo que realmente añade la pull request"): per query token and query head,
softmax(scale * q K_sel^T) V_sel over the cache rows the token's list names,
with the D256 default scale 1/sqrt(D); an entry is empty when it is negative,
outside [0, S) or at position >= n_valid; a row with no entry gives out = 0
and lse = -inf (same page, "Límites de tamaño").  lse is the natural log of
sum_j exp(s_j) with the scale included (the pages never define it; this is
the plain reading).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqsa_oracle.so")


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    hdr = os.path.join(_HERE, "qsa_oracle.h")
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-I", _HERE,
           "-fPIC", "-shared", "-pthread", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class _Args(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_q_heads", ctypes.c_int64),
        ("num_kv_heads", ctypes.c_int64),
        ("head_dim", ctypes.c_int64),
        ("topk", ctypes.c_int64),
        ("num_slots", ctypes.c_int64),
        ("q_stride_tok", ctypes.c_int64),
        ("q_stride_head", ctypes.c_int64),
        ("kv_stride_slot", ctypes.c_int64),
        ("kv_stride_head", ctypes.c_int64),
        ("idx_stride_tok", ctypes.c_int64),
        ("idx_stride_head", ctypes.c_int64),
        ("q", ctypes.c_void_p),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("idx", ctypes.c_void_p),
        ("n_valid", ctypes.c_void_p),
        ("scale", ctypes.c_double),
        ("block_size", ctypes.c_int64),
        ("last_slot", ctypes.c_void_p),
        ("kv_fp8", ctypes.c_int32),
        ("k8", ctypes.c_void_p),
        ("v8", ctypes.c_void_p),
        ("k_scale", ctypes.c_double),
        ("v_scale", ctypes.c_double),
    ]


class _IndexerArgs(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int64),
        ("num_heads", ctypes.c_int64),
        ("head_dim", ctypes.c_int64),
        ("num_blocks", ctypes.c_int64),
        ("block_size", ctypes.c_int64),
        ("q_stride_tok", ctypes.c_int64),
        ("q_stride_head", ctypes.c_int64),
        ("k_stride_block", ctypes.c_int64),
        ("q", ctypes.c_void_p),
        ("k", ctypes.c_void_p),
        ("positions", ctypes.c_void_p),
        ("seq_start", ctypes.c_void_p),
    ]


class Oracle:
    """ctypes handle on one build of qsa_oracle.c (the default build, or a
    copy with a planted mistake that the pin tests must reject)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.qsa_oracle_fwd.restype = ctypes.c_int64
        lib.qsa_oracle_fwd.argtypes = [ctypes.POINTER(_Args), ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        lib.qsa_oracle_bf16_to_double.restype = ctypes.c_double
        lib.qsa_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.qsa_oracle_e4m3_to_double.restype = ctypes.c_double
        lib.qsa_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.qsa_oracle_indexer_scores.restype = ctypes.c_int
        lib.qsa_oracle_indexer_scores.argtypes = [ctypes.POINTER(_IndexerArgs), ctypes.c_void_p,
                                                  ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
        lib.qsa_oracle_topk.restype = ctypes.c_int
        lib.qsa_oracle_topk.argtypes = [ctypes.POINTER(_IndexerArgs), ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        self.lib = lib
        self.path = lib_path

    def bf16_to_double(self, bits: int) -> float:
        return self.lib.qsa_oracle_bf16_to_double(ctypes.c_uint16(bits))

    def sparse_prefill(self, q, k_cache, v_cache, topk_idx, n_valid=None, scale=0.0,
                       tokens=None, n_threads=None, block_size=1, last_slot=None,
                       k_scale=1.0, v_scale=1.0):
        """k_cache / v_cache are BF16, or FP8 E4M3 (torch float8_e4m3fn, or
        uint8 bytes) whose elements are the decoded byte times k_scale /
        v_scale."""
        return _sparse_prefill(self.lib, q, k_cache, v_cache, topk_idx, n_valid, scale,
                               tokens, n_threads, block_size, last_slot, k_scale, v_scale)

    def e4m3_to_double(self, bits: int) -> float:
        return self.lib.qsa_oracle_e4m3_to_double(int(bits))


    def indexer_scores(self, q_idx, k_idx, positions, seq_start, block_size=4, tokens=None):
        """FP64 indexer scores [n, NB]: sum over heads of <q_idx[t,h], k_idx[b]>,
        -inf outside the token's complete causal microblocks."""
        a, keep = _indexer_args(q_idx, k_idx, positions, seq_start, block_size)
        T = a.num_tokens
        if tokens is None:
            tokens = np.arange(T, dtype=np.int64)
        tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
        out = np.zeros((tokens.shape[0], a.num_blocks), dtype=np.float64)
        rc = self.lib.qsa_oracle_indexer_scores(ctypes.byref(a), tokens.ctypes.data, tokens.shape[0], 1,
                                                out.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        return out

    def topk(self, scores, positions, seq_start, num_blocks, budget, block_size=4, append_tail=False):
        """Selection over given FP32 scores [T, ld]: ascending block ids of the
        `budget` highest candidates (ties to the smaller id), then with
        `append_tail` the token's own incomplete block, -1 padded; and counts."""
        sc = np.ascontiguousarray(_as_f32(scores))
        T, ld = sc.shape
        pos = np.ascontiguousarray(_as_i32(positions))
        s0 = np.ascontiguousarray(_as_i32(seq_start))
        a = _IndexerArgs(T, 0, 0, num_blocks, block_size, 0, 0, 0, None, None, pos.ctypes.data,
                         s0.ctypes.data)
        sel = np.zeros((T, budget + (1 if append_tail else 0)), dtype=np.int32)
        cnt = np.zeros((T,), dtype=np.int32)
        rc = self.lib.qsa_oracle_topk(ctypes.byref(a), sc.ctypes.data, ld, budget, int(bool(append_tail)),
                                      sel.ctypes.data, cnt.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        return sel, cnt


def _as_f32(x):
    if hasattr(x, "numpy") and not isinstance(x, np.ndarray):
        x = x.detach().cpu().numpy()
    x = np.asarray(x)
    if x.dtype != np.float32:
        raise TypeError(f"expected float32, got {x.dtype}")
    return x


def _indexer_args(q_idx, k_idx, positions, seq_start, block_size):
    q = _as_u16(q_idx)
    k = _as_u16(k_idx)
    T, H, Dh = q.shape
    NB, Dk = k.shape
    if Dk != Dh:
        raise ValueError("q_idx / k_idx head dims differ")
    qs = _strides(q, 3)
    ks = _strides(k, 2)
    if qs[2] != 1 or ks[1] != 1:
        raise ValueError("head dim must be contiguous")
    pos = np.ascontiguousarray(_as_i32(positions))
    s0 = np.ascontiguousarray(_as_i32(seq_start))
    if pos.shape != (T,) or s0.shape != (T,):
        raise ValueError("positions / seq_start must be [T]")
    a = _IndexerArgs(T, H, Dh, NB, block_size, qs[0], qs[1], ks[0], q.ctypes.data, k.ctypes.data,
                     pos.ctypes.data, s0.ctypes.data)
    return a, (q, k, pos, s0)


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def _as_u16(x):
    """BF16 data (torch bf16 tensor or uint16/int16 numpy bits) -> uint16 ndarray view."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        x = x.detach()
        if x.device.type != "cpu":
            raise ValueError("oracle inputs must be on the host")
        import torch
        x = x.view(torch.int16).numpy()
    x = np.asarray(x)
    if x.dtype not in (np.uint16, np.int16):
        raise TypeError(f"expected BF16 bit patterns, got {x.dtype}")
    return x.view(np.uint16)


def _as_i32(x):
    if x is None:
        return None
    if hasattr(x, "numpy") and not isinstance(x, np.ndarray):
        if x.device.type != "cpu":
            raise ValueError("oracle inputs must be on the host")
        x = x.detach().numpy()
    x = np.asarray(x)
    if x.dtype != np.int32:
        raise TypeError(f"expected int32, got {x.dtype}")
    return x


def _strides(arr, nd):
    if arr.ndim != nd:
        raise ValueError(f"expected {nd}-d array, got shape {arr.shape}")
    st = [s // arr.itemsize for s in arr.strides]
    if any(s * arr.itemsize != b for s, b in zip(st, arr.strides)):
        raise ValueError("strides must be whole elements")
    return st


def bf16_to_double(bits: int) -> float:
    return default().bf16_to_double(bits)


def sparse_prefill(q, k_cache, v_cache, topk_idx, n_valid=None, scale=0.0,
                   tokens=None, n_threads=None, block_size=1, last_slot=None,
                   k_scale=1.0, v_scale=1.0):
    return default().sparse_prefill(q, k_cache, v_cache, topk_idx, n_valid, scale,
                                    tokens, n_threads, block_size, last_slot, k_scale, v_scale)


def _as_u8(x):
    """FP8 E4M3 data (torch float8_e4m3fn tensor or uint8 numpy bytes) -> uint8 ndarray view."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.float8_e4m3fn":
        x = x.detach()
        if x.device.type != "cpu":
            raise ValueError("oracle inputs must be on the host")
        import torch
        x = x.view(torch.uint8).numpy()
    x = np.asarray(x)
    if x.dtype != np.uint8:
        raise TypeError(f"expected FP8 E4M3 bytes, got {x.dtype}")
    return x


def _is_fp8(x):
    return (hasattr(x, "dtype") and str(x.dtype) == "torch.float8_e4m3fn") or \
        (isinstance(x, np.ndarray) and x.dtype == np.uint8)


def _sparse_prefill(lib, q, k_cache, v_cache, topk_idx, n_valid, scale, tokens, n_threads,
                    block_size=1, last_slot=None, k_scale=1.0, v_scale=1.0):
    """FP64 oracle.  q [T,Hq,D], k_cache/v_cache [S,Hkv,D] (BF16, host),
    topk_idx [T,Hkv,K] int32, n_valid [T,Hkv] int32 or None.

    block_size > 1: list entries name microblocks of that many consecutive
    slots (n_valid counts entries); last_slot [T] int32 bounds the slots each
    token sees (None: no bound).

    Returns (out [n,Hq,D] float64, lse [n,Hq] float64, n_out_of_range) for the
    tokens listed in ``tokens`` (all tokens when None).
    """
    fp8 = _is_fp8(k_cache)
    q = _as_u16(q)
    if fp8:
        k = _as_u8(k_cache); v = _as_u8(v_cache)
    else:
        k = _as_u16(k_cache); v = _as_u16(v_cache)
    idx = _as_i32(topk_idx); nv = _as_i32(n_valid)
    T, Hq, D = q.shape
    S, Hkv, Dk = k.shape
    if v.shape != k.shape or Dk != D:
        raise ValueError("k_cache/v_cache shape mismatch")
    qs = _strides(q, 3); ks = _strides(k, 3); vs = _strides(v, 3)
    if ks != vs:
        raise ValueError("k_cache and v_cache must share strides")
    if qs[2] != 1 or ks[2] != 1:
        raise ValueError("head dim must be contiguous")
    if idx.shape[0] != T or idx.shape[1] != Hkv:
        raise ValueError("topk_idx shape mismatch")
    K = idx.shape[2]
    ist = _strides(idx, 3)
    if ist[2] != 1 and K > 1:
        raise ValueError("list entries must be contiguous")
    if nv is not None:
        if nv.shape != (T, Hkv):
            raise ValueError("n_valid shape mismatch")
        nv = np.ascontiguousarray(nv)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64))
    n = tokens.shape[0]
    out = np.zeros((n, Hq, D), dtype=np.float64)
    lse = np.zeros((n, Hq), dtype=np.float64)
    ls = _as_i32(last_slot)
    if ls is not None:
        if ls.shape != (T,):
            raise ValueError("last_slot must be [T]")
        ls = np.ascontiguousarray(ls)
    a = _Args(T, Hq, Hkv, D, K, S, qs[0], qs[1], ks[0], ks[1], ist[0], ist[1],
              q.ctypes.data, None if fp8 else k.ctypes.data, None if fp8 else v.ctypes.data,
              idx.ctypes.data, nv.ctypes.data if nv is not None else None, float(scale),
              int(block_size), ls.ctypes.data if ls is not None else None,
              1 if fp8 else 0, k.ctypes.data if fp8 else None, v.ctypes.data if fp8 else None,
              float(k_scale), float(v_scale))
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    rc = lib.qsa_oracle_fwd(ctypes.byref(a), tokens.ctypes.data, n, int(n_threads),
                                out.ctypes.data, lse.ctypes.data)
    if rc < 0:
        raise ValueError("oracle rejected its arguments")
    return out, lse, int(rc)
