"""QSA indexer scores and top-K selection against the FP64 oracle.

The indexer (page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Por qué
QSA es la parte incómoda, en cifras"): 4 query heads sharing one key head of
dim 128, one key per microblock of 4 slots, a budget of 2048 microblocks per
query.  Scores are FP32 on the GPU and FP64 in the oracle: they must agree
within 2^-14 * sum_h sum_d |q_hd k_d| (twice the n*u bound of an FP32 dot
product of n = 512 terms, u = 2^-24, whatever the summation order).  The
selection is an integer decision taken on FP32 scores, so both sides take it
on the same FP32 scores (the GPU's, copied to the host): bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from top_sparse_attention_qsa_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"
SCORE_REL = 2.0 ** -14


@pytest.fixture(scope="module")
def C():
    from top_sparse_attention_qsa_b200 import _capi
    return _capi


def _host(x):
    return x.detach().cpu()


def check_scores(orc, w, got, tokens=None):
    """GPU scores (host float32 [n, NB]) of `tokens` against the oracle."""
    q, k = _host(w.q_idx), _host(w.k_idx)
    pos, s0 = _host(w.positions), _host(w.seq_start)
    ref = orc.indexer_scores(q, k, pos, s0, w.block_size, tokens=tokens)
    bound = orc.indexer_scores(q.abs(), k.abs(), pos, s0, w.block_size, tokens=tokens)
    got = got.double().numpy()
    cand = np.isfinite(ref)
    # candidate entries within the bound; the rest untouched (the -inf fill)
    err = np.abs(got[cand] - ref[cand])
    assert np.all(err <= SCORE_REL * bound[cand]), float((err / bound[cand]).max())
    assert np.all(np.isneginf(got[~cand]))
    return cand


def check_selection(orc, w, scores, lists, nv, budget, tail, rows=None):
    """GPU lists [T, width] against the oracle's selection on the same FP32 scores."""
    if rows is not None:
        r = torch.tensor(rows, device=scores.device)
        scores, lists, nv = scores[r], lists[r], nv[r]
        pos, s0 = _host(w.positions)[rows].numpy(), _host(w.seq_start)[rows].numpy()
    else:
        pos, s0 = _host(w.positions).numpy(), _host(w.seq_start).numpy()
    sc = np.ascontiguousarray(_host(scores).numpy())
    sel, cnt = orc.topk(sc, pos, s0, w.k_idx.shape[0], budget, w.block_size, tail)
    got = _host(lists).numpy()
    gnv = _host(nv).numpy()
    np.testing.assert_array_equal(got, sel)
    for c in range(gnv.shape[1]):
        np.testing.assert_array_equal(gnv[:, c], cnt)


@pytest.mark.parametrize("H,fold", [(4, True), (4, False), (1, False), (2, False), (8, True), (8, False)])
def test_scores_small_ragged(C, orc, H, fold):
    # 300 tokens (several 256/H-token tiles and a ragged one), 700 block keys
    # (several 128-block tiles and a ragged one), two sequences, tails 0..3;
    # H >= 4 with and without the head folding
    w = W.config_indexer(device=DEV, seed=5 + H, T=300, S=2800, heads=H, budget=64,
                         seq_starts=[0, 1400])
    scores = C.indexer_scores(w.q_idx, w.k_idx, w.positions, w.seq_start, w.block_size, fold=fold)
    torch.cuda.synchronize()
    check_scores(orc, w, _host(scores))


@pytest.mark.parametrize("H", [1, 2, 4, 8])
def test_fold_heads(C, H):
    """hi + lo against the FP64 head sum: |s - hi - lo| <= 2^-16 |s| (two
    roundings to 8 significant bits) plus the
    FP32 sum's own error (at most (H - 1) 2^-24 sum_h |q_h|, taken as H
    2^-24 sum_h |q_h| to cover the 2^-16 term's argument too); hi is the
    BF16 rounding of the FP32 sum, so |lo| <= half an ulp of hi <= 2^-8 |hi|;
    a strided q (head stride 256) and T = 33."""
    g = torch.Generator(device=DEV).manual_seed(70 + H)
    base = W.normal_bf16((33, H, 256), g, DEV)
    q = base[:, :, :128]
    assert q.stride(1) == 256
    k = W.normal_bf16((8, 128), g, DEV)
    f = C.indexer_fold_heads(q, k)
    torch.cuda.synchronize()
    qd = _host(q).double()
    s = qd.sum(1)
    hi, lo = _host(f[:, 0]).double(), _host(f[:, 1]).double()
    bound = 2.0 ** -16 * s.abs() + H * 2.0 ** -24 * qd.abs().sum(1)
    assert bool(((hi + lo - s).abs() <= bound).all())
    assert bool((lo.abs() <= 2.0 ** -8 * hi.abs()).all())
    if H == 1:
        assert torch.equal(hi, qd[:, 0]) and bool((lo == 0).all())


@pytest.mark.parametrize("budget,tail", [(0, True), (1, False), (37, True), (128, False), (2048, True)])
def test_selection_small(C, orc, budget, tail):
    w = W.config_indexer(device=DEV, seed=17, T=300, S=2800, heads=4, seq_starts=[0, 1400])
    lists, nv, scores = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, budget,
                                         w.block_size, append_tail=tail, copies=2)
    torch.cuda.synchronize()
    check_selection(orc, w, scores, lists, nv, budget, tail)


def test_selection_large_rows(C, orc):
    # 12000 candidates per row: the 512-thread variant of the selection
    w = W.config_indexer(device=DEV, seed=23, T=96, S=48000, heads=4)
    lists, nv, scores = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, 2048,
                                         w.block_size, append_tail=True)
    torch.cuda.synchronize()
    check_selection(orc, w, scores, lists, nv, 2048, True)
    check_scores(orc, w, _host(scores)[:8], tokens=list(range(8)))


def test_full_size_sampled(C, orc):
    """8192 tokens over 32768 block keys (131072 slots), budget 2048, as
    timed: scores of sampled tokens and the selection of sampled rows."""
    w = W.config_indexer(device=DEV)
    lists, nv, scores = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, w.budget,
                                         w.block_size, append_tail=True, copies=2)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    toks = sorted(set([0, 1, 2, 3, 4095, 8191] + list(rng.choice(8192, 10, replace=False))))
    check_scores(orc, w, _host(scores[torch.tensor(toks, device=DEV)]), tokens=toks)
    rows = sorted(set([0, 1, 2, 3, 8191] + list(rng.choice(8192, 120, replace=False))))
    check_selection(orc, w, scores, lists, nv, w.budget, True, rows=rows)
    # every row: count = budget + tail, ids ascending and causal
    nvh = _host(nv)
    pos = _host(w.positions).long()
    want = w.budget + ((pos + 1) % 4 != 0).int()
    assert torch.equal(nvh[:, 0], want.to(torch.int32))
    L = _host(lists).long()
    assert bool((L[:, 1:w.budget] > L[:, :w.budget - 1]).all())
    assert bool((L[:, :w.budget] < ((pos + 1) // 4)[:, None]).all())


def test_ties_and_signed_zeros(C, orc):
    """Hand-made score rows: many exact ties, -0.0 against +0.0."""
    T, NB = 4, 5000
    w = W.config_indexer(device=DEV, seed=29, T=T, S=4 * NB, heads=4)
    sc = torch.randint(-3, 4, (T, NB), dtype=torch.int32).float()
    sc[1] = 0.0
    sc[1, ::2] = -0.0
    sc[2, 100:4000] = 7.0
    scores = sc.to(DEV)
    for budget in (1, 10, 1000, 3900):
        lists, nv = C.topk_select(scores, w.positions, w.seq_start, NB, budget, w.block_size,
                                  append_tail=True)
        torch.cuda.synchronize()
        check_selection(orc, w, scores, lists, nv, budget, True)


@pytest.mark.parametrize("NB,step", [(32768, 1 / 16), (32768, 1 / 1024), (12000, 1 / 8)])
def test_ties_inside_threshold_bin(C, orc, NB, step):
    """Normal scores on a grid of `step`: the bin that holds the budget-th
    score has a few hundred keys (the lists' path) and the exact threshold
    value is shared by many of them, which are taken in block order; rows
    of 32768 and 12000 candidates."""
    T = 24
    w = W.config_indexer(device=DEV, seed=47, T=T, S=4 * NB, heads=4)
    g = torch.Generator().manual_seed(int(1 / step))
    sc = torch.round(torch.randn(T, NB, generator=g) / step) * step
    sc[5] = -sc[5]
    scores = sc.to(DEV)
    for budget in (2048, 777):
        lists, nv = C.topk_select(scores, w.positions, w.seq_start, NB, budget, w.block_size,
                                  append_tail=True)
        torch.cuda.synchronize()
        check_selection(orc, w, scores, lists, nv, budget, True)


def test_edge_cases(C, orc):
    # single token, no complete block yet (positions 0..2), a block boundary,
    # one key; budget 0 with and without the tail
    for T, S, pos in ((1, 4, [2]), (4, 4, [0, 1, 2, 3]), (3, 12, [3, 7, 11])):
        w = W.config_indexer(device=DEV, seed=31, T=T, S=S, heads=4)
        w.positions = torch.tensor(pos, dtype=torch.int32, device=DEV)
        for budget, tail in ((0, False), (0, True), (1, True), (5, True)):
            lists, nv, scores = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, budget,
                                                 w.block_size, append_tail=tail)
            torch.cuda.synchronize()
            check_scores(orc, w, _host(scores))
            check_selection(orc, w, scores, lists, nv, budget, tail)


def test_zero_rows_tie_at_zero(C, orc):
    # a zero indexer query gives +/-0.0 for every block: the first blocks win
    w = W.config_indexer(device=DEV, seed=37, T=8, S=4096, heads=4)
    w.q_idx[3] = 0
    lists, nv, scores = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, 16,
                                         w.block_size, append_tail=False)
    torch.cuda.synchronize()
    check_selection(orc, w, scores, lists, nv, 16, False)
    lo = int(w.seq_start[3]) // 4
    assert _host(lists)[3].tolist() == list(range(lo, lo + 16))


def test_pipeline_into_block_attention(C, orc):
    """Indexer -> top-K -> microblock attention with two KV heads sharing the
    list (head stride 0), against the oracle attention over the same lists."""
    T, S = 40, 1024
    w = W.config_indexer(device=DEV, seed=41, T=T, S=S, heads=4, seq_starts=[0, 512])
    lists, nv, _ = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, 24, w.block_size,
                                    append_tail=True, copies=2)
    gen = torch.Generator(device=DEV).manual_seed(43)
    q = W.normal_bf16((T, 24, 256), gen, DEV)
    k = W.normal_bf16((S, 2, 256), gen, DEV)
    v = W.normal_bf16((S, 2, 256), gen, DEV)
    idx = lists[:, None, :].expand(T, 2, lists.shape[1])
    out, lse = C.sparse_prefill_block_fwd(q, k, v, idx, 4, w.positions, nv, 0.0)
    torch.cuda.synchronize()
    ref_o, ref_l, _ = oracle.sparse_prefill(_host(q), _host(k), _host(v), _host(idx).contiguous(), _host(nv),
                                         0.0, block_size=4, last_slot=_host(w.positions))
    o = _host(out).double().numpy()
    assert np.all(np.abs(o - ref_o) <= 1e-2 + 1e-2 * np.abs(ref_o))
    assert np.all(np.abs(_host(lse).double().numpy() - ref_l) <= 1e-3)


@pytest.mark.parametrize("bs", [1, 2, 8, 3])
def test_other_block_sizes(C, orc, bs):
    """Compression ratios other than 4 (the kernels take any block size >= 1):
    the candidate ranges, the selection and the tail follow the block size;
    two sequences starting on block boundaries."""
    S = 1200 * bs
    w = W.config_indexer(device=DEV, seed=60 + bs, T=150, S=S, heads=4, block_size=bs,
                         seq_starts=[0, 600 * bs])
    lists, nv, scores = C.indexer_select(w.q_idx, w.k_idx, w.positions, w.seq_start, 40, bs,
                                         append_tail=True, copies=2)
    torch.cuda.synchronize()
    check_scores(orc, w, _host(scores))
    check_selection(orc, w, scores, lists, nv, 40, True)
