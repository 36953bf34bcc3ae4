"""FP8 E4M3 KV cache (qsa_sparse_prefill_fp8_fwd) against the FP64 oracle.

The pages name the cache format only (page "Qwen4-Exp QSA llega al Ascend de
Huawei", observations on the NVIDIA side: an fp8_e4m3 KV cache); element
value = stored E4M3 value times a per-tensor scale.  Same tolerance as the
BF16 path (the kernel's only extra rounding is Q and P in FP16, which is no
coarser than the BF16 path's P).
"""
import pytest
import torch

import oracle
from top_sparse_attention_qsa_b200 import workloads as W
from parity import compare, host, sample_tokens

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


@pytest.fixture(scope="module")
def C():
    from top_sparse_attention_qsa_b200 import _capi
    return _capi


def fp8_case(T, S, heads, K, seed, std=1.0):
    w = W.generic_case(T=T, S=S, Hq=heads[0], Hkv=heads[1], K=K, seed=seed, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(seed + 1000)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, DEV, std=std)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, DEV)
    return w, k8, v8


def oracle_fp8(w, k8, v8, ks, vs, tokens=None, block_size=1, last=None):
    return oracle.sparse_prefill(host(w.q), host(k8), host(v8), host(w.topk_idx), host(w.n_valid), w.scale,
                                 tokens=tokens, block_size=block_size, last_slot=host(last),
                                 k_scale=ks, v_scale=vs)


@pytest.mark.parametrize("heads", [(3, 1), (6, 1), (12, 1), (16, 2), (24, 2)])
@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.37, 1.9)])
def test_head_shapes_and_scales(C, heads, scales):
    # K = 700: five 128-key tiles and a ragged one; ragged n_valid
    w, k8, v8 = fp8_case(T=40, S=3000, heads=heads, K=700, seed=heads[0] * 7 + 1, std=2.0)
    gen = torch.Generator(device=DEV).manual_seed(heads[0])
    w.n_valid = torch.randint(0, 701, (40, heads[1]), generator=gen, device=DEV, dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, *scales, n_valid=w.n_valid,
                                        scale=w.scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_lse, _ = oracle_fp8(w, k8, v8, *scales)
    compare(host(out), host(lse), ref_out, ref_lse, f"fp8 {heads} {scales}")


def test_masks_empty_rows_and_out_of_range(C):
    w, k8, v8 = fp8_case(T=12, S=900, heads=(16, 2), K=300, seed=5)
    w.topk_idx[3] = -1                          # empty rows
    w.topk_idx[5, 1, 17] = 900                  # id == S: masked and reported
    w.topk_idx[7, 0, ::3] = -1                  # interior holes
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 4.0, n_valid=w.n_valid,
                                        status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & C.STATUS_OOB_SLOT
    ref_out, ref_lse, n_oob = oracle_fp8(w, k8, v8, 0.5, 4.0)
    assert n_oob >= 1
    st = compare(host(out), host(lse), ref_out, ref_lse, "fp8 masks")
    assert st["empty_rows"] >= 16


def test_runs_of_empty_units(C):
    """Ten units per CTA (one KV head: unit = token, CTA b takes tokens b,
    b + SMs, ...), the rounds alternating full, empty (runs of three), short
    and one-key units, so that the two O buffers and the hand-off of l and m
    to the epilogue warps wrap their barrier phases on empty units too."""
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    pattern = [256, 0, 0, 0, 200, 0, 1, 256, 0, 130]
    T = nsm * len(pattern)
    w, k8, v8 = fp8_case(T=T, S=4096, heads=(16, 1), K=256, seed=23)
    nv = torch.tensor([pattern[t // nsm] for t in range(T)], dtype=torch.int32, device=DEV)
    w.n_valid = nv.reshape(T, 1).contiguous()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.75, 1.5, n_valid=w.n_valid,
                                        scale=w.scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_lse, _ = oracle_fp8(w, k8, v8, 0.75, 1.5)
    st = compare(host(out), host(lse), ref_out, ref_lse, "fp8 empty-unit runs")
    assert st["empty_rows"] >= 16 * nsm * pattern.count(0)


def test_block_lists_with_tail(C):
    T, S, bs = 25, 4001, 4
    w, k8, v8 = fp8_case(T=T, S=S, heads=(24, 2), K=1, seed=11)
    gen = torch.Generator(device=DEV).manual_seed(12)
    nb = (S + bs - 1) // bs
    w.topk_idx = W.random_lists(T, 2, 130, nb, gen, DEV)
    w.n_valid = torch.randint(0, 131, (T, 2), generator=gen, device=DEV, dtype=torch.int32)
    last = torch.randint(S // 2, S, (T,), generator=gen, device=DEV, dtype=torch.int32)
    out, lse = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.8, 1.25, n_valid=w.n_valid,
                                        block_size=bs, last_slot=last)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle_fp8(w, k8, v8, 0.8, 1.25, block_size=bs, last=last)
    compare(host(out), host(lse), ref_out, ref_lse, "fp8 blocks")


def test_c5_size_sampled(C):
    """c5's shape (8192 tokens at 122880.., 131072 slots, (24,2), 2048 entries)
    with an FP8 cache, as the bench times it."""
    w = W.make("c5", device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(77)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, DEV)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, DEV)
    out, lse = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid,
                                        scale=w.scale)
    torch.cuda.synchronize()
    tokens = sample_tokens(w.shape["T"], w.shape["K"], n_random=20, seed=8)
    ref_out, ref_lse, _ = oracle_fp8(w, k8, v8, 0.5, 2.0, tokens=tokens)
    t = torch.as_tensor(tokens)
    print(compare(host(out)[t], host(lse)[t], ref_out, ref_lse, "c5 fp8"))


def test_large_and_tiny_queries(C):
    # the query is scaled per head by a power of two before its split into two
    # E4M3 terms, so magnitudes far outside E4M3's range stay exact
    w, k8, v8 = fp8_case(T=6, S=300, heads=(12, 1), K=100, seed=21)
    w.q[2] *= 1e-3                              # a whole token of tiny queries
    w.q[3, 5, 7] = 3000.0                       # far beyond E4M3's 448
    w.q[4, 2] = 0.0                             # an all-zero head: uniform weights
    out, lse = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle_fp8(w, k8, v8, 0.5, 2.0)
    compare(host(out), host(lse), ref_out, ref_lse, "fp8 query range")


@pytest.mark.parametrize("splits", [0, 1, 4, 16])
def test_split_k_decode(C, splits):
    """Decode over an FP8 cache: 16 sequences of 8192 slots, one query token
    each, 2048-entry lists, cut into chunks merged by their log-sum-exp."""
    w = W.config_decode(device=DEV, seed=51, B=16, ctx=8192, heads=(24, 2), topk=2048, local=256)
    gen = torch.Generator(device=DEV).manual_seed(52)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, DEV, std=2.0)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, DEV)
    w.n_valid[3] = 0                              # an empty row
    w.n_valid[5] = 700                            # a ragged one
    out, lse = C.sparse_decode_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid,
                                       scale=w.scale, num_splits=splits)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle_fp8(w, k8, v8, 0.5, 2.0)
    compare(host(out), host(lse), ref_out, ref_lse, f"fp8 decode splits={splits}")
