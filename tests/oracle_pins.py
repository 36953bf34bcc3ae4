"""Checks that pin the FP64 oracle to facts other than itself.

Each check takes an oracle handle (``oracle.Oracle``) so that the same checks
also run against copies of the oracle with a planted mistake, which must fail
at least one of them (tests/test_oracle_mutants.py).

Pins (what the pages and the mathematics fix):
* dense_causal  -- when a list holds every causal slot 0..t, sparse attention
  is dense causal attention: torch's scaled_dot_product_attention and
  logsumexp in float64 (library routines) must agree.
* packing       -- the layout identity of page "Qwen4-Exp QSA llega al Ascend
  de Huawei", section "Lo que realmente añade la pull request":
  softmax(scale [Q,0][K,V]^T)[K,V] = [P K, P V] with the D256 scale.
* permutation   -- the result does not depend on list order or interleaved
  -1 padding (same page, "Nueve pruebas": unordered physical slots).
* head_padding  -- padding the group with extra query heads (12->16, 6->8,
  3->4; same page, "Formas de cabeza") leaves the real heads unchanged.
* closed_forms  -- zero queries give the mean of the selected V rows with
  lse = ln n; one entry gives that V row with lse = its score; an empty row
  gives exact zeros with lse = -inf ("Límites de tamaño"); duplicates count
  twice; out-of-range slots are reported and ignored.
* brute_force   -- an independent numpy evaluation without the max trick.
* worked_example -- the hand-derived fixture in tests/golden.
* split_merge   -- attention over a list equals the log-sum-exp merge of
  attention over any split of it (the combine step of split-K decode).
* block_lists   -- a microblock list equals the token list naming each of its
  slots (with the cache end and the token's last visible slot applied).
* indexer_scores -- page "Qwen4-Exp QSA llega al Ascend de Huawei", section
  "Por qué QSA es la parte incómoda, en cifras" (4 query heads sharing one
  key head, dim 128, compression 4): with one head the scores are a plain
  matrix product (numpy matmul); with four they are the sum of the one-head
  scores; the candidate ranges of hand-picked positions (causal tails 0..3,
  a later sequence start) are the complete causal blocks; strides do not
  matter.
* fp8_cache     -- page "Qwen4-Exp QSA llega al Ascend de Huawei" names an
  fp8_e4m3 KV cache: the byte decoding equals torch's float8_e4m3fn over all
  256 patterns; with power-of-two scales the FP8 attention equals the
  (pinned) BF16 attention on the dequantized caches bit for bit; with other
  scales it equals torch's scaled_dot_product_attention in float64 on the
  dequantized values.
* topk          -- the selection equals a lexicographic sort on (-score,
  block) by numpy (library routine); every chosen score >= every unchosen
  one; all-equal scores take the first blocks; -0.0 ties +0.0; the causal
  tail is appended for remainders 1..3 only.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from top_sparse_attention_qsa_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = dict(rtol=1e-12, atol=1e-12)


def _np64(x):
    return x.to(torch.float64).numpy()


def _expand_kv(x, G):
    # [S, Hkv, D] -> [Hq, S, D] with head h reading KV head h // G
    return x.to(torch.float64).permute(1, 0, 2).repeat_interleave(G, dim=0)


def check_bf16_widening(orc):
    bits = torch.arange(0, 1 << 16, dtype=torch.int32)
    keep = ((bits >> 7) & 0xFF) != 0xFF                   # drop inf/nan exponents
    bits = bits[keep][::37]
    want = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.bf16_to_double(int(b) & 0xFFFF) for b in bits.tolist()])
    np.testing.assert_array_equal(got, want)


def check_dense_causal(orc, shapes=((3, 1), (6, 1), (12, 1), (16, 2), (24, 2)), T=24, seed=11):
    for i, (Hq, Hkv) in enumerate(shapes):
        G = Hq // Hkv
        gen = torch.Generator().manual_seed(seed + i)
        D = W.HEAD_DIM
        q = W.normal_bf16((T, Hq, D), gen, "cpu")
        k = W.normal_bf16((T, Hkv, D), gen, "cpu", std=2.0)
        v = W.normal_bf16((T, Hkv, D), gen, "cpu")
        K = T + 5
        idx = torch.full((T, Hkv, K), -1, dtype=torch.int32)
        for t in range(T):
            for g in range(Hkv):
                perm = torch.randperm(t + 1, generator=gen).to(torch.int32)
                slots = torch.randperm(K, generator=gen)[: t + 1]
                idx[t, g, slots] = perm          # every causal slot, scattered
        for scale in (0.0, 0.037):
            out, lse, oob = orc.sparse_prefill(q, k, v, idx, None, scale)
            assert oob == 0
            sc = scale if scale > 0 else 1.0 / math.sqrt(D)
            qd = q.to(torch.float64).permute(1, 0, 2)[None]          # [1,Hq,T,D]
            kd = _expand_kv(k, G)[None]
            vd = _expand_kv(v, G)[None]
            ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=sc)
            ref = ref[0].permute(1, 0, 2).numpy()
            scores = (qd @ kd.transpose(-1, -2)) * sc
            mask = torch.ones(T, T, dtype=torch.bool).tril()
            scores = scores.masked_fill(~mask, float("-inf"))
            ref_lse = torch.logsumexp(scores, dim=-1)[0].permute(1, 0).numpy()
            np.testing.assert_allclose(out, ref, **TOL)
            np.testing.assert_allclose(lse, ref_lse, **TOL)


def _small_case(Hq, Hkv, T=6, S=40, K=9, seed=3):
    return W.generic_case(T, S, Hq, Hkv, K, seed)


def check_packing(orc, shapes=((3, 1), (16, 2))):
    for Hq, Hkv in shapes:
        w = _small_case(Hq, Hkv)
        scale = 1.0 / 16                      # the original D256 scale is kept
        C = torch.cat([w.k_cache, w.v_cache], dim=-1)          # [S, Hkv, 512]
        Qp = torch.cat([w.q, torch.zeros_like(w.q)], dim=-1)   # [T, Hq, 512]
        packed, lse_p, _ = orc.sparse_prefill(Qp, C, C, w.topk_idx, None, scale)
        pv, lse, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, None, scale)
        pk, _, _ = orc.sparse_prefill(w.q, w.k_cache, w.k_cache, w.topk_idx, None, scale)
        np.testing.assert_allclose(packed[..., 256:], pv, **TOL)
        np.testing.assert_allclose(packed[..., :256], pk, **TOL)
        np.testing.assert_allclose(lse_p, lse, **TOL)


def check_permutation(orc, shapes=((6, 1), (24, 2))):
    for j, (Hq, Hkv) in enumerate(shapes):
        w = _small_case(Hq, Hkv, K=13, seed=5 + j)
        gen = torch.Generator().manual_seed(99 + j)
        T, _, K = w.topk_idx.shape
        K2 = K + 7
        idx2 = torch.full((T, Hkv, K2), -1, dtype=torch.int32)
        for t in range(T):
            for g in range(Hkv):
                pos = torch.randperm(K2, generator=gen)[:K]
                idx2[t, g, pos] = w.topk_idx[t, g, torch.randperm(K, generator=gen)]
        a = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx)
        b = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, idx2)
        np.testing.assert_allclose(b[0], a[0], **TOL)
        np.testing.assert_allclose(b[1], a[1], **TOL)
        # n_valid masks the tail exactly like -1 does, whatever the tail holds
        nv = torch.randint(0, K + 1, (T, Hkv), generator=gen, dtype=torch.int32)
        ar = torch.arange(K)[None, None, :]
        masked = torch.where(ar < nv[:, :, None], w.topk_idx, torch.full_like(w.topk_idx, -1))
        c = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, nv)
        d = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, masked)
        np.testing.assert_array_equal(c[0], d[0])
        np.testing.assert_array_equal(c[1], d[1])


def check_head_padding(orc, pad=((12, 1, 16), (6, 1, 8), (3, 1, 4), (24, 2, 16))):
    for Hq, Hkv, Gp in pad:
        w = _small_case(Hq, Hkv, seed=17)
        G = Hq // Hkv
        T, _, D = w.q.shape
        gen = torch.Generator().manual_seed(5)
        qp = W.normal_bf16((T, Hkv * Gp, D), gen, "cpu", std=3.0)   # garbage heads
        real = [g * Gp + r for g in range(Hkv) for r in range(G)]
        qp[:, real] = w.q
        a = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx)
        b = orc.sparse_prefill(qp, w.k_cache, w.v_cache, w.topk_idx)
        np.testing.assert_allclose(b[0][:, real], a[0], **TOL)
        np.testing.assert_allclose(b[1][:, real], a[1], **TOL)


def check_closed_forms(orc):
    D = W.HEAD_DIM
    w = _small_case(12, 1, T=5, S=30, K=7, seed=23)
    S = 30
    # zero queries: uniform weights -> mean of the selected rows, lse = ln n
    q0 = torch.zeros_like(w.q)
    nv = torch.tensor([[7], [3], [1], [5], [2]], dtype=torch.int32)
    out, lse, _ = orc.sparse_prefill(q0, w.k_cache, w.v_cache, w.topk_idx, nv)
    vd = _np64(w.v_cache)
    for t in range(5):
        n = int(nv[t, 0])
        rows = w.topk_idx[t, 0, :n].long().numpy()
        mean = vd[rows, 0, :].mean(axis=0)
        for h in range(12):
            np.testing.assert_allclose(out[t, h], mean, **TOL)
            np.testing.assert_allclose(lse[t, h], math.log(n), **TOL)
    # one entry: that V row exactly, lse = scale * q.k
    one = w.topk_idx[:, :, :1].contiguous()
    out, lse, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, one)
    qd, kd = _np64(w.q), _np64(w.k_cache)
    for t in range(5):
        s = int(one[t, 0, 0])
        np.testing.assert_array_equal(out[t], np.broadcast_to(vd[s, 0], (12, D)))
        np.testing.assert_allclose(lse[t], (qd[t] @ kd[s, 0]) / 16.0, **TOL)
    # duplicates: [a, a] -> v_a, lse = s_a + ln 2
    dup = torch.cat([one, one], dim=2)
    out2, lse2, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, dup)
    np.testing.assert_allclose(out2, out, **TOL)
    np.testing.assert_allclose(lse2, lse + math.log(2.0), **TOL)
    # empty rows (all -1, n_valid = 0, K = 0): exact +0.0 and -inf
    empty = torch.full((5, 1, 4), -1, dtype=torch.int32)
    for args in ((empty, None), (w.topk_idx, torch.zeros((5, 1), dtype=torch.int32)),
                 (torch.empty((5, 1, 0), dtype=torch.int32), None)):
        out, lse, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, *args)
        assert np.all(out == 0.0) and not np.any(np.signbit(out))
        assert np.all(np.isneginf(lse))
    # an out-of-range slot is reported and ignored
    bad = w.topk_idx.clone()
    bad[:, :, 0] = S + 3
    out_b, lse_b, oob = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, bad)
    assert oob == 5
    out_r, lse_r, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx[:, :, 1:].contiguous())
    np.testing.assert_allclose(out_b, out_r, **TOL)
    np.testing.assert_allclose(lse_b, lse_r, **TOL)


def check_brute_force(orc, shapes=((3, 1), (16, 2))):
    for Hq, Hkv in shapes:
        w = _small_case(Hq, Hkv, T=7, S=50, K=11, seed=31)
        G = Hq // Hkv
        qd, kd, vd = _np64(w.q), _np64(w.k_cache), _np64(w.v_cache)
        idx = w.topk_idx.numpy()
        ref = np.zeros(qd.shape)
        ref_lse = np.zeros(qd.shape[:2])
        for t in range(qd.shape[0]):
            for h in range(Hq):
                rows = idx[t, h // G]
                e = np.exp(np.array([qd[t, h] @ kd[r, h // G] for r in rows]) / 16.0)
                ref[t, h] = (e[:, None] * vd[rows, h // G]).sum(0) / e.sum()
                ref_lse[t, h] = np.log(e.sum())
        out, lse, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx)
        np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-11, atol=1e-12)


def check_worked_example(orc):
    with open(os.path.join(GOLDEN, "worked_example_three_keys.json")) as f:
        ex = json.load(f)
    D, S = ex["head_dim"], ex["num_slots"]
    q = torch.zeros((1, 1, D))
    for d, x in ex["q_nonzero"].items():
        q[0, 0, int(d)] = x
    k = torch.full((S, 1, D), ex["filler_value"])
    v = torch.full((S, 1, D), ex["filler_value"])
    for s, row in ex["k_rows"].items():
        k[int(s), 0] = 0
        for d, x in row.items():
            k[int(s), 0, int(d)] = x
    for s, row in ex["v_rows"].items():
        v[int(s), 0] = 0
        for d, x in row.items():
            v[int(s), 0, int(d)] = x
    idx = torch.tensor(ex["list"], dtype=torch.int32).view(1, 1, -1)
    out, lse, _ = orc.sparse_prefill(q.to(torch.bfloat16), k.to(torch.bfloat16),
                                     v.to(torch.bfloat16), idx, None, ex["scale"])
    want = np.zeros(D)
    for d, x in ex["expected_out_nonzero"].items():
        want[int(d)] = float(x)
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], float(ex["expected_lse"]), rtol=1e-14)


def check_split_merge(orc):
    """Attention over a list equals the lse-weighted mix of attention over any
    split of the list into chunks (the combine step of split-K / decode
    context parallelism): lse = log sum_c exp(lse_c), out = sum_c
    exp(lse_c - lse) out_c; an empty chunk has lse_c = -inf and weight 0."""
    w = W.generic_case(T=5, S=900, Hq=24, Hkv=2, K=300, seed=41)
    full, lse_full, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx)
    for bounds in ((0, 128, 256, 300), (0, 7, 8, 300), (0, 300, 300)):
        outs, lses = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            o, l, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx[:, :, a:b].contiguous())
            outs.append(o)
            lses.append(l)
        L = np.stack(lses)                                  # [chunks, T, Hq]
        m = L.max(axis=0)
        wts = np.where(np.isneginf(L), 0.0, np.exp(L - m))
        lse = m + np.log(wts.sum(axis=0))
        out = (wts[..., None] * np.stack(outs)).sum(axis=0) / wts.sum(axis=0)[..., None]
        np.testing.assert_allclose(out, full, **TOL)
        np.testing.assert_allclose(lse, lse_full, **TOL)


def check_block_lists(orc):
    """A microblock list equals the token list that names each of its slots
    (entry b -> slots b*bs .. b*bs+bs-1), with slots beyond the cache or the
    token's last visible slot dropped; block size 1 is the token list."""
    gen = torch.Generator().manual_seed(61)
    T, S, Hq, Hkv, E = 6, 203, 16, 2, 9
    q = W.normal_bf16((T, Hq, 256), gen, "cpu")
    k = W.normal_bf16((S, Hkv, 256), gen, "cpu")
    v = W.normal_bf16((S, Hkv, 256), gen, "cpu")
    for bs in (1, 2, 4):
        nb = (S + bs - 1) // bs
        blocks = torch.stack([torch.randperm(nb, generator=gen)[:E] for _ in range(T * Hkv)]).view(T, Hkv, E)
        blocks[0, 0, 3] = -1
        blocks = blocks.to(torch.int32)
        last = torch.randint(S // 2, S, (T,), generator=gen, dtype=torch.int32)
        nv = torch.randint(0, E + 1, (T, Hkv), generator=gen, dtype=torch.int32)
        got = orc.sparse_prefill(q, k, v, blocks, nv, 0.0, block_size=bs, last_slot=last)
        tok = torch.full((T, Hkv, E * bs), -1, dtype=torch.int32)
        for t in range(T):
            for g in range(Hkv):
                for j in range(int(nv[t, g])):
                    b = int(blocks[t, g, j])
                    if b < 0:
                        continue
                    for r in range(bs):
                        s_ = b * bs + r
                        if s_ < S and s_ <= int(last[t]):
                            tok[t, g, j * bs + r] = s_
        want = orc.sparse_prefill(q, k, v, tok, None, 0.0)
        np.testing.assert_allclose(got[0], want[0], **TOL)
        np.testing.assert_allclose(got[1], want[1], **TOL)


# Positions with causal tails 0..3 at ratio 4 and a second sequence starting
# at slot 16, with their complete-block candidate ranges worked out by hand:
# a token at position p sees blocks [start/4, (p+1)/4).
IDX_POS = [3, 4, 5, 6, 7, 30, 43, 0]
IDX_START = [0, 0, 0, 0, 0, 16, 16, 0]
IDX_RANGES = [(0, 1), (0, 1), (0, 1), (0, 1), (0, 2), (4, 7), (4, 11), (0, 0)]


def check_indexer_scores(orc):
    gen = torch.Generator().manual_seed(71)
    T, NB, Dh = len(IDX_POS), 11, 128
    pos = torch.tensor(IDX_POS, dtype=torch.int32)
    s0 = torch.tensor(IDX_START, dtype=torch.int32)
    k = W.normal_bf16((NB, Dh), gen, "cpu")
    q = W.normal_bf16((T, 4, Dh), gen, "cpu")
    got = orc.indexer_scores(q, k, pos, s0, block_size=4)
    # candidate ranges: finite exactly on [lo, hi)
    for t, (lo, hi) in enumerate(IDX_RANGES):
        fin = np.isfinite(got[t])
        assert fin[lo:hi].all() and not fin[:lo].any() and not fin[hi:].any(), t
    mask = np.isfinite(got)
    kd = _np64(k)
    # one head: a plain matrix product
    for h in range(4):
        one = orc.indexer_scores(q[:, h:h + 1].contiguous(), k, pos, s0, block_size=4)
        want = _np64(q[:, h]) @ kd.T
        np.testing.assert_allclose(one[mask], want[mask], rtol=1e-12, atol=1e-12)
    # four heads: the sum of the one-head scores (matmul of the head sum)
    want = _np64(q).sum(axis=1) @ kd.T
    np.testing.assert_allclose(got[mask], want[mask], rtol=1e-12, atol=1e-12)
    # padded strides and a token subset give the same values
    qp = torch.zeros((T, 6, Dh + 64), dtype=torch.bfloat16)
    qp[:, 1:5, :Dh] = q
    kp = torch.zeros((NB, Dh + 32), dtype=torch.bfloat16)
    kp[:, :Dh] = k
    sub = orc.indexer_scores(qp[:, 1:5, :Dh], kp[:, :Dh], pos, s0, block_size=4, tokens=[6, 2])
    np.testing.assert_array_equal(sub, got[[6, 2]])


def _lexsort_select(scores, lo, hi, budget):
    b = np.arange(lo, hi)
    order = np.lexsort((b, -scores[lo:hi].astype(np.float64)))
    return np.sort(b[order[:budget]])


def check_topk(orc):
    rng = np.random.default_rng(73)
    T, NB = len(IDX_POS), 11
    pos = np.array(IDX_POS, dtype=np.int32)
    s0 = np.array(IDX_START, dtype=np.int32)
    sc = rng.standard_normal((T, NB)).astype(np.float32)
    sc[6, [5, 8, 9]] = sc[6, 6]                  # ties inside the longest row
    for budget in (0, 1, 2, 3, 5, 20):
        for tail in (False, True):
            sel, cnt = orc.topk(sc, pos, s0, NB, budget, block_size=4, append_tail=tail)
            assert sel.shape == (T, budget + int(tail))
            for t, (lo, hi) in enumerate(IDX_RANGES):
                want = list(_lexsort_select(sc[t], lo, hi, budget))
                # every chosen score is >= every unchosen candidate score
                rest = [b for b in range(lo, hi) if b not in want]
                if want and rest:
                    assert sc[t, want].min() >= sc[t, rest].max()
                rem = (IDX_POS[t] + 1) % 4
                if tail and rem:
                    want.append(IDX_POS[t] // 4)
                n = len(want)
                assert cnt[t] == n, (budget, tail, t)
                np.testing.assert_array_equal(sel[t, :n], want)
                assert (sel[t, n:] == -1).all()
    # all-equal scores take the first blocks of the range
    eq = np.full((T, NB), 0.5, dtype=np.float32)
    sel, cnt = orc.topk(eq, pos, s0, NB, 3, block_size=4)
    np.testing.assert_array_equal(sel[6], [4, 5, 6])
    # -0.0 ties +0.0: the smaller block index wins either way round
    z = np.full((T, NB), -1.0, dtype=np.float32)
    z[6, 5], z[6, 7] = -0.0, 0.0
    assert orc.topk(z, pos, s0, NB, 1, block_size=4)[0][6, 0] == 5
    z[6, 5], z[6, 7] = 0.0, -0.0
    assert orc.topk(z, pos, s0, NB, 1, block_size=4)[0][6, 0] == 5
    # the tail block follows the chosen ones for remainders 1..3 only
    sel, cnt = orc.topk(sc, pos, s0, NB, 0, block_size=4, append_tail=True)
    assert [int(c) for c in cnt] == [0, 1, 1, 1, 0, 1, 0, 1]
    assert int(sel[5, 0]) == 7 and int(sel[1, 0]) == 1


def check_fp8_cache(orc):
    # byte decoding against torch's float8_e4m3fn (library routine)
    allb = torch.arange(256, dtype=torch.uint8)
    ref = allb.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_to_double(b) for b in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    np.testing.assert_array_equal(got[fin], ref[fin])
    gen = torch.Generator().manual_seed(83)
    T, S, Hq, Hkv, K, D = 7, 60, 16, 2, 11, 256
    q = W.normal_bf16((T, Hq, D), gen, "cpu")
    k8 = W.normal_fp8((S, Hkv, D), gen, "cpu", std=3.0)
    v8 = W.normal_fp8((S, Hkv, D), gen, "cpu")
    k8[0, 0, :8] = torch.tensor([2 ** -9, -2 ** -8, 448.0, -448.0, 0.0, -0.0, 2 ** -6, 3 * 2 ** -9]).to(torch.float8_e4m3fn)
    idx = torch.stack([torch.randperm(S, generator=gen)[:K] for _ in range(T * Hkv)]).view(T, Hkv, K).to(torch.int32)
    idx[:, 0, 0] = 0                                   # every token sees the subnormal row
    # power-of-two scales: the dequantized caches are exact in BF16
    ks, vs = 0.5, 4.0
    got = orc.sparse_prefill(q, k8, v8, idx, None, 0.0, k_scale=ks, v_scale=vs)
    kb = (k8.to(torch.float64) * ks).to(torch.bfloat16)
    vb = (v8.to(torch.float64) * vs).to(torch.bfloat16)
    assert torch.equal(kb.to(torch.float64), k8.to(torch.float64) * ks)
    want = orc.sparse_prefill(q, kb, vb, idx, None, 0.0)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])
    # other scales: dense causal attention (every causal slot listed) against
    # torch's SDPA on the dequantized values in float64
    T2 = 12
    q2 = W.normal_bf16((T2, 6, D), gen, "cpu")
    k2 = W.normal_fp8((T2, 1, D), gen, "cpu", std=2.0)
    v2 = W.normal_fp8((T2, 1, D), gen, "cpu")
    idx2 = torch.full((T2, 1, T2), -1, dtype=torch.int32)
    for t in range(T2):
        idx2[t, 0, : t + 1] = torch.randperm(t + 1, generator=gen).to(torch.int32)
    ks, vs = 0.37, 1.9
    out, lse, _ = orc.sparse_prefill(q2, k2, v2, idx2, None, 0.0, k_scale=ks, v_scale=vs)
    qd = q2.to(torch.float64).permute(1, 0, 2)[None]
    kd = (k2.to(torch.float64) * ks).permute(1, 0, 2).repeat_interleave(6, dim=0)[None]
    vd = (v2.to(torch.float64) * vs).permute(1, 0, 2).repeat_interleave(6, dim=0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=1 / 16)
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), **TOL)
    sc = (qd @ kd.transpose(-1, -2)) / 16
    sc = sc.masked_fill(~torch.ones(T2, T2, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(sc, dim=-1)[0].permute(1, 0).numpy(), **TOL)


ALL_CHECKS = [check_bf16_widening, check_dense_causal, check_packing, check_permutation,
              check_head_padding, check_closed_forms, check_brute_force, check_worked_example,
              check_split_merge, check_block_lists, check_indexer_scores, check_topk,
              check_fp8_cache]
