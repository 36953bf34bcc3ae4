"""Shared parity helpers: run the CUDA path through the C ABI, run the FP64
oracle on the same (host copies of the) inputs, compare.

Tolerances: |out - ref| <= 1e-2 + 1e-2 |ref| on the BF16 output and
|lse - ref| <= 1e-3 on the FP32 log-sum-exp; rows with an empty selection
must be exactly +0.0 with lse = -inf.  The pages' own operator thresholds
(page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Nueve pruebas que
pasaron": atol = rtol = 0.025, relative L2 < 0.008) are checked as well.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

OUT_ATOL = 1e-2
OUT_RTOL = 1e-2
LSE_ATOL = 1e-3
PAGES_ATOL = PAGES_RTOL = 0.025
PAGES_REL_L2 = 0.008


def run_gpu(w, kernel="auto", **kw):
    from top_sparse_attention_qsa_b200 import _capi
    return _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                    kernel=kernel, **kw)


def host(x):
    return None if x is None else x.detach().cpu()


def run_oracle(w, tokens=None):
    return oracle.sparse_prefill(host(w.q), host(w.k_cache), host(w.v_cache), host(w.topk_idx),
                                 host(w.n_valid), w.scale, tokens=tokens)


def compare(out_gpu, lse_gpu, ref_out, ref_lse, label=""):
    """out_gpu [n,Hq,D] bf16 (host), lse_gpu [n,Hq] fp32 (host); refs float64."""
    o = out_gpu.to(torch.float64).numpy()
    ls = lse_gpu.to(torch.float64).numpy()
    empty = np.isneginf(ref_lse)
    stats = {"rows": int(ref_lse.size), "empty_rows": int(empty.sum())}
    if empty.any():
        eo = out_gpu.view(torch.int16).numpy()[empty]
        assert np.all(eo == 0), f"{label}: empty rows not exactly +0.0"
        assert np.all(np.isneginf(ls[empty])), f"{label}: empty rows need lse = -inf"
    full = ~empty
    if not full.any():
        return stats
    assert np.all(np.isfinite(ls[full])), f"{label}: non-finite lse on a non-empty row"
    of, rf = o[full], ref_out[full]
    err = np.abs(of - rf)
    bound = OUT_ATOL + OUT_RTOL * np.abs(rf)
    worst = float((err / bound).max())
    assert np.all(np.isfinite(of)), f"{label}: non-finite output"
    assert worst <= 1.0, f"{label}: out error {err.max():.3e} exceeds 1e-2 + 1e-2|ref| (ratio {worst:.2f})"
    lerr = float(np.abs(ls[full] - ref_lse[full]).max())
    assert lerr <= LSE_ATOL, f"{label}: lse error {lerr:.3e} > {LSE_ATOL}"
    # the pages' thresholds
    assert np.all(err <= PAGES_ATOL + PAGES_RTOL * np.abs(rf))
    rel_l2 = float(np.linalg.norm(of - rf) / max(np.linalg.norm(rf), 1e-300))
    assert rel_l2 < PAGES_REL_L2, f"{label}: relative L2 {rel_l2:.4f}"
    stats.update(max_abs_err=float(err.max()), tol_ratio=worst, lse_err=lerr, rel_l2=rel_l2)
    return stats


def sample_tokens(T, K, n_random=40, seed=0, extra=()):
    g = np.random.default_rng(seed)
    base = {0, 1, 2, T - 1, T - 2}
    for x in (K - 2, K - 1, K, K + 1):
        if 0 <= x < T:
            base.add(x)
    base.update(int(x) for x in extra if 0 <= x < T)
    base.update(int(x) for x in g.choice(T, size=min(n_random, T), replace=False))
    return np.array(sorted(base), dtype=np.int64)


def expected_gather(w):
    """The ids the gather must load: the list entry where it is a live slot,
    -1 where it is masked (integer work: compared bit-exactly)."""
    idx = host(w.topk_idx).to(torch.int64)
    K = idx.shape[2]
    S = w.k_cache.shape[0]
    live = (idx >= 0) & (idx < S)
    if w.n_valid is not None:
        live &= torch.arange(K)[None, None, :] < host(w.n_valid).to(torch.int64)[:, :, None]
    return torch.where(live, idx, torch.full_like(idx, -1)).to(torch.int32)


def expected_gather_lists(w, block_size=1, last_slot=None):
    """The slot the gather must copy for every key of a token or microblock
    list, [T, Hkv, K * block_size] int32: key j of (t, g) reads slot
    idx[t,g,j // bs] * bs + j % bs when the entry is live (j // bs <
    n_valid, id >= 0, its block starts inside the cache) and the slot is
    inside the cache and at most last_slot[t]; -1 otherwise.  Integer work,
    compared bit-exactly."""
    idx = host(w.topk_idx).to(torch.int64)
    T, Hkv, K = idx.shape
    S = w.k_cache.shape[0]
    bs = int(block_size)
    live = idx >= 0
    if w.n_valid is not None:
        live &= torch.arange(K)[None, None, :] < host(w.n_valid).to(torch.int64)[:, :, None]
    live &= idx * bs < S
    slot = idx[..., None] * bs + torch.arange(bs)[None, None, None, :]          # [T, Hkv, K, bs]
    ok = live[..., None] & (slot < S)
    if last_slot is not None:
        ok &= slot <= host(last_slot).to(torch.int64)[:, None, None, None]
    return torch.where(ok, slot, torch.full_like(slot, -1)).reshape(T, Hkv, K * bs).to(torch.int32)
