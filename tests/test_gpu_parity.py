"""CUDA path (through the C ABI) against the FP64 oracle, element by element.

Covers the five workload configurations (full or sampled rows at full size),
the pages' operator cases (page "Qwen4-Exp QSA llega al Ascend de Huawei",
section "Nueve pruebas que pasaron": widths 1/63/64/65/2051 with unordered
slots, default and explicit scale, fully masked rows, zero rows, zero width,
non-contiguous tensors, causal tails 0-3, two requests sharing a prefix,
cache reuse, the local head shapes at 1 and 257 query rows, the long
prefill), and the bit-exact gather dump.
"""
import numpy as np
import pytest
import torch

from top_sparse_attention_qsa_b200 import workloads as W
from parity import compare, expected_gather, host, run_gpu, run_oracle, sample_tokens

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"
KERNELS = ["tcgen05", "warp_mma"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from top_sparse_attention_qsa_b200 import _capi  # noqa: F401  (fails loudly if unbuilt)


def check_all(w, label, kernel="auto"):
    out, lse = run_gpu(w, kernel)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = run_oracle(w)
    return compare(host(out), host(lse), ref_out, ref_lse, label)


def check_sampled(w, label, tokens, kernel="auto"):
    out, lse = run_gpu(w, kernel)
    torch.cuda.synchronize()
    o, ls = host(out), host(lse)
    # properties that hold at any size: every row finite, empty rows exact
    assert torch.isfinite(o.float()).all(), f"{label}: non-finite output"
    ref_out, ref_lse, _ = run_oracle(w, tokens=tokens)
    t = torch.as_tensor(tokens)
    return compare(o[t], ls[t], ref_out, ref_lse, label)


# --- the five configurations ------------------------------------------------

@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name", ["tiny", "c2"])
def test_config_full(name, kernel):
    w = W.make(name, device=DEV)
    print(name, kernel, check_all(w, name, kernel))


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name", ["c3", "c4", "c5"])
def test_config_sampled(name, kernel):
    w = W.make(name, device=DEV)
    s = w.shape
    extra = []
    if name == "c3":
        extra = [8190, 8191, 8192, 8193, 8192 + 1023, 8192 + 1024]   # second sequence start
    tokens = sample_tokens(s["T"], s["K"], n_random=48, seed=len(name), extra=extra)
    print(name, kernel, check_sampled(w, name, tokens, kernel))


@pytest.mark.parametrize("kernel", KERNELS)
def test_very_long_lists(kernel):
    """40000 distinct entries per (token, KV head): 313 tiles per unit, long
    runs of lazy rescales, heads (24,2); every row against the oracle."""
    w = W.generic_case(T=6, S=50000, Hq=24, Hkv=2, K=40000, seed=71, device=DEV)
    # a rising score trend along each list makes the running max move often
    ramp = torch.linspace(0.0, 3.0, 50000, device=DEV)[:, None, None]
    w.k_cache = (w.k_cache.float() * (1.0 + ramp)).to(torch.bfloat16)
    print(check_all(w, "very long lists", kernel))


def test_pages_long_prefill():
    """7810 query tokens x 65536-slot cache x 2051 slots, sampled rows + all finite."""
    w = W.make("pages_long", device=DEV)
    tokens = sample_tokens(7810, 2051, n_random=24, seed=8)
    print(check_sampled(w, "pages_long", tokens))


# --- gather dump --------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "c2", "c5"])
def test_gather_dump_bit_exact(name):
    from top_sparse_attention_qsa_b200 import _capi
    w = W.make(name, device=DEV)
    out, lse, ids = _capi.sparse_prefill_debug_gather(w.q, w.k_cache, w.v_cache, w.topk_idx,
                                                      w.n_valid, w.scale)
    ref_out, ref_lse = run_gpu(w)
    torch.cuda.synchronize()
    assert torch.equal(host(ids), expected_gather(w))
    # the dump variant computes the same result bit for bit
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


# --- the pages' operator cases ------------------------------------------------

@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("K", [1, 63, 64, 65, 127, 128, 129, 2051])
@pytest.mark.parametrize("heads", [(12, 1), (24, 2)])
def test_widths_unordered(K, heads, kernel):
    w = W.generic_case(T=19, S=4096, Hq=heads[0], Hkv=heads[1], K=K, seed=K, device=DEV)
    check_all(w, f"width{K}", kernel)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("heads", W.HEAD_SHAPES)
@pytest.mark.parametrize("T", [1, 257])
def test_head_shapes_rows(heads, T, kernel):
    w = W.generic_case(T=T, S=3000, Hq=heads[0], Hkv=heads[1], K=130, seed=T + heads[0], device=DEV)
    check_all(w, f"heads{heads}T{T}", kernel)


@pytest.mark.parametrize("scale", [0.0, 1.0 / 16, 0.037, 0.25])
def test_default_and_explicit_scale(scale):
    w = W.generic_case(T=33, S=777, Hq=6, Hkv=1, K=100, seed=3, device=DEV, scale=scale)
    check_all(w, f"scale{scale}")


def test_default_scale_is_d256():
    w = W.generic_case(T=9, S=500, Hq=16, Hkv=2, K=70, seed=4, device=DEV)
    a, la = run_gpu(w)
    w.scale = 1.0 / 16
    b, lb = run_gpu(w)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("kernel", KERNELS)
def test_masked_rows_and_interior_padding(kernel):
    w = W.generic_case(T=40, S=1000, Hq=24, Hkv=2, K=96, seed=5, device=DEV)
    idx = w.topk_idx.clone()
    idx[3] = -1                                # fully masked token, both heads
    idx[7, 1] = -1                             # one head masked
    idx[10, :, ::3] = -1                       # interior -1
    idx[11, 0, 1:] = -1                        # single live entry
    idx[12, :, :-1] = -7                       # other negative values also mask
    nv = torch.full((40, 2), 96, dtype=torch.int32, device=DEV)
    nv[20] = 0                                 # n_valid = 0 -> empty
    nv[21, 1] = 1
    nv[22] = 65                                # tail beyond n_valid holds live ids but is ignored
    nv[23] = 200                               # n_valid > K clamps to K
    w.topk_idx, w.n_valid = idx.contiguous(), nv
    st = check_all(w, "masked", kernel)
    assert st["empty_rows"] >= 24 + 12 + 24


def test_zero_query_rows():
    w = W.generic_case(T=17, S=600, Hq=12, Hkv=1, K=200, seed=6, device=DEV)
    w.q[::2] = 0
    check_all(w, "zero_q")


def test_zero_width():
    w = W.generic_case(T=5, S=64, Hq=6, Hkv=1, K=0, seed=1, device=DEV)
    out, lse = run_gpu(w)
    torch.cuda.synchronize()
    assert torch.all(out.view(torch.int16) == 0)
    assert torch.all(torch.isneginf(lse))


def test_non_contiguous_tensors():
    T, S, Hq, Hkv, K, D = 37, 900, 24, 2, 150, 256
    gen = torch.Generator(device=DEV).manual_seed(12)
    qbuf = W.normal_bf16((T, Hq + 3, D + 16), gen, DEV)
    q = qbuf[:, 1:Hq + 1, 8:D + 8]                         # padded token/head strides
    kv = W.normal_bf16((S, Hkv, 2, D), gen, DEV)           # packed [K, V] cache rows
    idx_buf = W.random_lists(T, 1, K + 13, S, gen, DEV)
    idx = idx_buf[:, :, :K].expand(T, Hkv, K)              # one list shared by both heads
    w = W.Workload("strided", q, kv[:, :, 0], kv[:, :, 1], idx, None, 0.0,
                   torch.zeros(T, dtype=torch.int64), torch.zeros(T, dtype=torch.int64))
    from top_sparse_attention_qsa_b200 import _capi
    obuf = torch.full((T, Hq + 1, D + 8), 7.0, dtype=torch.bfloat16, device=DEV)
    out = obuf[:, :Hq, :D]
    lbuf = torch.full((T, Hq + 5), 7.0, dtype=torch.float32, device=DEV)
    lse = lbuf[:, :Hq]
    _capi.sparse_prefill_fwd(q, w.k_cache, w.v_cache, idx, None, 0.0, out=out, lse=lse)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = run_oracle(w)
    compare(host(out), host(lse), ref_out, ref_lse, "strided")
    # nothing outside the views was written
    assert torch.all(obuf[:, Hq:] == 7.0) and torch.all(obuf[:, :, D:] == 7.0)
    assert torch.all(lbuf[:, Hq:] == 7.0)


@pytest.mark.parametrize("r", [0, 1, 2, 3])
def test_causal_tail_remainders(r):
    """2048 selected slots plus a causal tail of r tokens (compression ratio 4)."""
    T, S, K = 24, 8192, 2048 + r
    gen = torch.Generator(device=DEV).manual_seed(100 + r)
    w = W.generic_case(T=T, S=S, Hq=16, Hkv=2, K=K, seed=200 + r, device=DEV)
    pos = torch.arange(S - T, S, device=DEV)
    body = W.random_subset_rows(torch.zeros(T * 2, dtype=torch.int64, device=DEV),
                                (pos - r).repeat_interleave(2), 2048, gen, DEV).view(T, 2, 2048)
    tail = (pos[:, None] - r + 1 + torch.arange(r, device=DEV)[None, :])[:, None, :].expand(T, 2, r)
    w.topk_idx = torch.cat([body, tail], dim=2).to(torch.int32).contiguous()
    check_all(w, f"tail{r}")


def test_two_requests_shared_prefix_and_cache_reuse():
    w = W.two_request_case(prefix=700, len_a=300, len_b=260, K=512, heads=(12, 1), device=DEV)
    check_all(w, "two_request")
    out1, lse1 = run_gpu(w)
    q1 = w.q
    # cache reuse: a second pass over the same cache with new queries
    gen = torch.Generator(device=DEV).manual_seed(77)
    w.q = W.normal_bf16(tuple(w.q.shape), gen, DEV)
    check_all(w, "two_request_reuse")
    # and the first queries again give the first answer bit for bit
    w.q = q1
    out3, lse3 = run_gpu(w)
    assert torch.equal(out1, out3) and torch.equal(lse1, lse3)


def test_out_of_range_slots_flag_status():
    from top_sparse_attention_qsa_b200 import _capi
    w = W.generic_case(T=12, S=300, Hq=6, Hkv=1, K=90, seed=8, device=DEV)
    w.topk_idx[2, 0, 5] = 300
    w.topk_idx[9, 0, 0] = 123456
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, None, 0.0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & _capi.STATUS_OOB_SLOT
    ref_out, ref_lse, n_oob = run_oracle(w)
    assert n_oob == 2
    compare(host(out), host(lse), ref_out, ref_lse, "oob")
    w2 = W.generic_case(T=12, S=300, Hq=6, Hkv=1, K=90, seed=8, device=DEV)
    status.zero_()
    _capi.sparse_prefill_fwd(w2.q, w2.k_cache, w2.v_cache, w2.topk_idx, None, 0.0, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_permutation_and_determinism():
    w = W.generic_case(T=50, S=5000, Hq=12, Hkv=1, K=700, seed=9, device=DEV)
    a, la = run_gpu(w)
    b, lb = run_gpu(w)
    assert torch.equal(a, b) and torch.equal(la, lb)          # deterministic
    perm = torch.argsort(torch.rand(w.topk_idx.shape, device=DEV), dim=2)
    w.topk_idx = torch.gather(w.topk_idx, 2, perm).contiguous()
    c, lc = run_gpu(w)
    torch.cuda.synchronize()
    o = c.double().cpu().numpy()
    r = a.double().cpu().numpy()
    assert np.all(np.abs(o - r) <= 1e-2 + 1e-2 * np.abs(r))
    assert float((lc - la).abs().max()) <= 1e-3


def test_host_buffer_entry_point_matches_device():
    from top_sparse_attention_qsa_b200 import _capi
    w = W.make("tiny", device=DEV)
    ref_out, ref_lse = run_gpu(w)
    hq = host(w.q).pin_memory()
    hk = host(w.k_cache).pin_memory()
    hv = host(w.v_cache).pin_memory()
    hi = host(w.topk_idx).pin_memory()
    ho = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(w.q.shape[:2], dtype=torch.float32).pin_memory()
    bufs = dict(q=torch.empty_like(w.q), k_cache=torch.empty_like(w.k_cache),
                v_cache=torch.empty_like(w.v_cache), topk_idx=torch.empty_like(w.topk_idx),
                out=torch.empty_like(w.q), lse=torch.empty(w.q.shape[:2], device=DEV),
                status=torch.ones(1, dtype=torch.int32, device=DEV))
    _capi.sparse_prefill_fwd_host(hq, hk, hv, hi, None, w.scale, ho, hl, bufs)
    torch.cuda.synchronize()
    assert torch.equal(ho, host(ref_out)) and torch.equal(hl, host(ref_lse))
    assert int(bufs["status"].item()) == 0


def test_host_buffer_entry_point_pipelined_chunks():
    """T = 4096 (c2): the host entry point cuts the tokens into 4 chunks whose
    copies overlap the kernels on three streams; results equal the device
    entry point's bit for bit, n_valid included, and the caller's stream is
    ordered after the last copy down."""
    from top_sparse_attention_qsa_b200 import _capi
    w = W.make("c2", device=DEV)
    ref_out, ref_lse = run_gpu(w)
    torch.cuda.synchronize()
    hq, hk, hv = host(w.q).pin_memory(), host(w.k_cache).pin_memory(), host(w.v_cache).pin_memory()
    hi = host(w.topk_idx).pin_memory()
    hn = host(w.n_valid).pin_memory() if w.n_valid is not None else None
    ho = torch.full(w.q.shape, 3.0, dtype=torch.bfloat16).pin_memory()
    hl = torch.full(w.q.shape[:2], 3.0, dtype=torch.float32).pin_memory()
    bufs = dict(q=torch.empty_like(w.q), k_cache=torch.empty_like(w.k_cache),
                v_cache=torch.empty_like(w.v_cache), topk_idx=torch.empty_like(w.topk_idx),
                n_valid=torch.empty_like(w.n_valid) if hn is not None else None,
                out=torch.empty_like(w.q), lse=torch.empty(w.q.shape[:2], device=DEV),
                status=torch.ones(1, dtype=torch.int32, device=DEV))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _capi.sparse_prefill_fwd_host(hq, hk, hv, hi, hn, w.scale, ho, hl, bufs, stream=s.cuda_stream)
    s.synchronize()                                        # the caller's stream alone
    assert torch.equal(ho, host(ref_out)) and torch.equal(hl, host(ref_lse))
    assert int(bufs["status"].item()) == 0


def test_misaligned_pointer_rejected():
    from top_sparse_attention_qsa_b200 import _capi
    w = W.generic_case(T=4, S=64, Hq=3, Hkv=1, K=8, seed=1, device=DEV)
    buf = torch.zeros(4 * 3 * 256 + 4, dtype=torch.bfloat16, device=DEV)
    q_bad = buf[4:].view(4, 3, 256)                        # 8-byte offset
    q_bad.copy_(w.q)
    with pytest.raises(_capi.QSAError) as e:
        _capi.sparse_prefill_fwd(q_bad, w.k_cache, w.v_cache, w.topk_idx)
    assert e.value.code == _capi.QSA_ERR_ALIGN
