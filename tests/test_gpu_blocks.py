"""Microblock lists (qsa_sparse_prefill_block_fwd) against the FP64 oracle.

QSA selects microblocks (page "Qwen4-Exp QSA llega al Ascend de Huawei",
section "Por qué QSA es la parte incómoda, en cifras": a budget of 2048
microblocks per query at compression ratio 4).  Each list entry names a block
of block_size consecutive cache slots; a per-token last visible slot masks the
part of the newest block beyond the query (the causal tail).
"""
import numpy as np
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


def run_blocks(C, w, bs, last=None, **kw):
    return C.sparse_prefill_block_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, bs, last, w.n_valid,
                                      w.scale, **kw)


def oracle_blocks(w, bs, last=None, tokens=None):
    return oracle.sparse_prefill(host(w.q), host(w.k_cache), host(w.v_cache), host(w.topk_idx),
                                 host(w.n_valid), w.scale, tokens=tokens, block_size=bs,
                                 last_slot=host(last))


def test_c5_block4_sampled():
    from top_sparse_attention_qsa_b200 import _capi as C
    w = W.make("c5_block4", device=DEV)
    out, lse = run_blocks(C, w, w.block_size, w.last_slot)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    tokens = sample_tokens(w.shape["T"], 0, n_random=24, seed=5)
    ref_out, ref_lse, _ = oracle_blocks(w, w.block_size, w.last_slot, tokens)
    t = torch.as_tensor(tokens)
    print(compare(host(out)[t], host(lse)[t], ref_out, ref_lse, "c5_block4"))


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("heads", [(12, 1), (24, 2)])
def test_block_sizes(C, bs, heads):
    T, S = 21, 3001                     # S not a multiple of the block size
    gen = torch.Generator(device=DEV).manual_seed(bs * 100 + heads[0])
    w = W.generic_case(T=T, S=S, Hq=heads[0], Hkv=heads[1], K=1, seed=bs, device=DEV)
    nb = (S + bs - 1) // bs
    E = min(300 // bs + 7, nb)
    w.topk_idx = W.random_lists(T, heads[1], E, nb, gen, DEV)
    w.topk_idx[2, :, ::5] = -1
    w.n_valid = torch.randint(0, E + 1, (T, heads[1]), generator=gen, device=DEV, dtype=torch.int32)
    last = torch.randint(S // 3, S + 5, (T,), generator=gen, device=DEV, dtype=torch.int32)
    out, lse = run_blocks(C, w, bs, last)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle_blocks(w, bs, last)
    compare(host(out), host(lse), ref_out, ref_lse, f"bs{bs}")


def test_block_size_one_is_the_token_path(C):
    w = W.generic_case(T=30, S=5000, Hq=16, Hkv=2, K=700, seed=9, device=DEV)
    a, la = run_blocks(C, w, 1)
    b, lb = C.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                 kernel="tcgen05")
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_block_out_of_range_and_masks(C):
    T, S, bs = 9, 1000, 4                # 250 blocks
    w = W.generic_case(T=T, S=S, Hq=6, Hkv=1, K=1, seed=4, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(3)
    w.topk_idx = W.random_lists(T, 1, 60, 250, gen, DEV)
    w.topk_idx[1, 0, 7] = 250            # block starts at slot 1000 = S: out of range
    w.topk_idx[4] = -1                   # empty row
    last = torch.full((T,), S - 1, dtype=torch.int32, device=DEV)
    last[6] = 3                          # only slots 0..3 visible
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = run_blocks(C, w, bs, last, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & C.STATUS_OOB_SLOT
    ref_out, ref_lse, n_oob = oracle_blocks(w, bs, last)
    assert n_oob == 1
    st = compare(host(out), host(lse), ref_out, ref_lse, "block_masks")
    assert st["empty_rows"] >= 6


def test_pages_budget_2048_microblocks(C):
    """The pages' budget: 2048 microblocks of 4 (8192 keys) per query."""
    w = W.config_c5_block4(device=DEV, T=64, S=65536, heads=(24, 2), blocks=2048, local_blocks=64)
    out, lse = run_blocks(C, w, 4, w.last_slot)
    torch.cuda.synchronize()
    tokens = sample_tokens(64, 0, n_random=12, seed=2)
    ref_out, ref_lse, _ = oracle_blocks(w, 4, w.last_slot, tokens)
    t = torch.as_tensor(tokens)
    compare(host(out)[t], host(lse)[t], ref_out, ref_lse, "budget2048")
