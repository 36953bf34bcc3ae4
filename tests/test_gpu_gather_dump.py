"""Bit-exact gather dumps for every gather path of the prefill.

Selection and gather are integer work: the rows a kernel copies must be
exactly the rows the lists name.  qsa_sparse_prefill_debug_gather_lists runs
the kernel of qsa_sparse_prefill_block_fwd (BF16 cache) or
qsa_sparse_prefill_fp8_fwd (FP8 E4M3 cache) with a dump of the slot each
key's K and V copies read, recovered from the copies' source addresses.  The
dump is compared bit for bit with the expansion of the lists (parity.py:
expected_gather_lists), on token lists and microblock lists (page
"Qwen4-Exp QSA llega al Ascend de Huawei", section "Por qué QSA es la parte
incómoda, en cifras": selection at microblock granularity, with the causal
tail), including masked entries, out-of-range blocks and the full c5 sizes.
The outputs of the dumping kernel are checked against the oracle too.
"""
import pytest
import torch

import oracle
from top_sparse_attention_qsa_b200 import workloads as W
from parity import compare, expected_gather, expected_gather_lists, host, sample_tokens

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


@pytest.fixture(scope="module")
def C():
    from top_sparse_attention_qsa_b200 import _capi
    return _capi


def fp8_caches(w, seed):
    gen = torch.Generator(device=DEV).manual_seed(seed)
    return (W.normal_fp8(tuple(w.k_cache.shape), gen, DEV), W.normal_fp8(tuple(w.v_cache.shape), gen, DEV))


def oracle_rows(w, k, v, tokens, bs=1, last=None, ks=1.0, vs=1.0):
    kw = {} if k.dtype == torch.bfloat16 else dict(k_scale=ks, v_scale=vs)
    return oracle.sparse_prefill(host(w.q), host(k), host(v), host(w.topk_idx), host(w.n_valid), w.scale,
                                 tokens=tokens, block_size=bs, last_slot=host(last), **kw)


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_token_lists_c2(C, cache):
    w = W.make("c2", device=DEV)
    k, v = (w.k_cache, w.v_cache) if cache == "bf16" else fp8_caches(w, 11)
    out, lse, ids = C.sparse_prefill_debug_gather_lists(w.q, k, v, w.topk_idx, 1, None, w.n_valid, w.scale,
                                                        k_scale=0.5, v_scale=2.0)
    torch.cuda.synchronize()
    assert torch.equal(host(ids), expected_gather(w))
    tokens = sample_tokens(w.shape["T"], w.shape["K"], n_random=16, seed=3)
    ref_out, ref_lse, _ = oracle_rows(w, k, v, tokens, ks=0.5, vs=2.0)
    t = torch.as_tensor(tokens)
    compare(host(out)[t], host(lse)[t], ref_out, ref_lse, f"dump c2 {cache}")


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16])
def test_block_lists_with_masks(C, cache, bs):
    T, S = 23, 3001                      # S not a multiple of the block size
    gen = torch.Generator(device=DEV).manual_seed(700 + bs)
    w = W.generic_case(T=T, S=S, Hq=24, Hkv=2, K=1, seed=bs, device=DEV)
    nb = (S + bs - 1) // bs
    E = min(300 // bs + 7, nb)
    w.topk_idx = W.random_lists(T, 2, E, nb, gen, DEV)
    w.topk_idx[2, :, ::5] = -1                      # interior -1
    w.topk_idx[4, 1, 3] = nb + 2                    # a block past the cache: empty, status bit 0
    w.topk_idx[5, 0, 0] = -7                        # another negative id
    w.n_valid = torch.randint(0, E + 1, (T, 2), generator=gen, device=DEV, dtype=torch.int32)
    w.n_valid[4, 1] = E
    last = torch.randint(S // 3, S + 5, (T,), generator=gen, device=DEV, dtype=torch.int32)
    k, v = (w.k_cache, w.v_cache) if cache == "bf16" else fp8_caches(w, bs)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse, ids = C.sparse_prefill_debug_gather_lists(w.q, k, v, w.topk_idx, bs, last, w.n_valid, w.scale,
                                                        k_scale=0.75, v_scale=1.5, status=status)
    torch.cuda.synchronize()
    assert torch.equal(host(ids), expected_gather_lists(w, bs, last))
    assert int(status.item()) & C.STATUS_OOB_SLOT
    ref_out, ref_lse, n_oob = oracle_rows(w, k, v, None, bs, last, 0.75, 1.5)
    assert n_oob == 1
    compare(host(out), host(lse), ref_out, ref_lse, f"dump bs{bs} {cache}")


def test_c5_block4_full_size(C):
    """The microblock bench workload at full size: 8192 tokens x 2 KV heads x
    512 blocks of 4, the newest block cut at the token's own slot."""
    w = W.make("c5_block4", device=DEV)
    _, _, ids = C.sparse_prefill_debug_gather_lists(w.q, w.k_cache, w.v_cache, w.topk_idx, w.block_size,
                                                    w.last_slot, w.n_valid, w.scale)
    torch.cuda.synchronize()
    exp = expected_gather_lists(w, w.block_size, w.last_slot)
    assert int((exp < 0).sum()) > 0                  # the causal tail is masked somewhere
    assert torch.equal(host(ids), exp)


def test_c5_fp8_full_size(C):
    """c5's token lists (unsorted, 2048 per token and KV head) over an FP8 cache."""
    w = W.make("c5", device=DEV)
    k8, v8 = fp8_caches(w, 5)
    w.k_cache = w.v_cache = None
    w.k_cache, w.v_cache = k8, v8
    _, _, ids = C.sparse_prefill_debug_gather_lists(w.q, k8, v8, w.topk_idx, 1, None, w.n_valid, w.scale,
                                                    k_scale=0.5, v_scale=2.0)
    torch.cuda.synchronize()
    assert torch.equal(host(ids), expected_gather(w))


def test_c5_block4_fp8_sampled_outputs(C):
    """Microblock lists over an FP8 cache: dump exact, outputs on sampled rows."""
    w = W.config_c5_block4(device=DEV, T=1024, S=131072)
    k8, v8 = fp8_caches(w, 6)
    out, lse, ids = C.sparse_prefill_debug_gather_lists(w.q, k8, v8, w.topk_idx, w.block_size, w.last_slot,
                                                        w.n_valid, w.scale, k_scale=0.5, v_scale=2.0)
    torch.cuda.synchronize()
    assert torch.equal(host(ids), expected_gather_lists(w, w.block_size, w.last_slot))
    tokens = sample_tokens(1024, 0, n_random=10, seed=8)
    ref_out, ref_lse, _ = oracle_rows(w, k8, v8, tokens, w.block_size, w.last_slot, 0.5, 2.0)
    t = torch.as_tensor(tokens)
    compare(host(out)[t], host(lse)[t], ref_out, ref_lse, "c5_block4 fp8")


def test_dumping_kernel_matches_plain_kernel(C):
    """The dump changes nothing else: out and lse equal the plain call's bit for bit."""
    w = W.config_c5_block4(device=DEV, T=512, S=65536)
    a, la = C.sparse_prefill_block_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.block_size, w.last_slot,
                                       w.n_valid, w.scale)
    b, lb, _ = C.sparse_prefill_debug_gather_lists(w.q, w.k_cache, w.v_cache, w.topk_idx, w.block_size,
                                                   w.last_slot, w.n_valid, w.scale)
    k8, v8 = fp8_caches(w, 7)
    c, lc = C.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid, scale=w.scale,
                                     block_size=w.block_size, last_slot=w.last_slot)
    d, ld, _ = C.sparse_prefill_debug_gather_lists(w.q, k8, v8, w.topk_idx, w.block_size, w.last_slot,
                                                   w.n_valid, w.scale, k_scale=0.5, v_scale=2.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert torch.equal(c, d) and torch.equal(lc, ld)
