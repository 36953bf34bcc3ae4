"""The synthetic inputs have the structure their configurations describe.

Both sides of every parity test read the same generated lists, so a slip in
the generator would not show up as a parity failure; it would only make the
measured workload differ from the described one.  These CPU checks pin each
configuration's lists: distinct causal ids inside the token's own sequence,
the local window present, the random part of the stated size drawn from
before the window, the order (sorted or not), the ragged short rows and the
-1 padding.  c4 and c5 are generated with fewer tokens (same rule, same
cache geometry) to keep the suite fast.
"""
import pytest
import torch

from top_sparse_attention_qsa_b200 import workloads as W

CASES = {
    # name: (builder kwargs, local window, sorted?)
    "tiny": (dict(), 16, True),
    "c2": (dict(), 64, True),
    "c3": (dict(), 128, True),
    "c4": (dict(T=3000), 128, True),
    "c5": (dict(T=400), 256, False),
}


def _lists(name):
    kw, local, ordered = CASES[name]
    w = W.make(name, device="cpu", **kw)
    return w, local, ordered


@pytest.mark.parametrize("name", sorted(CASES))
def test_list_structure(name):
    w, L, ordered = _lists(name)
    idx = w.topk_idx.long()
    T, H, K = idx.shape
    pos = w.positions.long()
    s0 = w.seq_start.long()
    n_caus = pos - s0 + 1
    n_valid = torch.minimum(n_caus, torch.full_like(n_caus, K))
    if w.n_valid is not None:
        assert torch.equal(w.n_valid.long(), n_valid[:, None].expand(T, H))
    ar = torch.arange(K)
    live = ar[None, None, :] < n_valid[:, None, None]
    # padding past n_valid is -1; live entries are causal and inside the own sequence
    assert bool((idx[~live.expand(T, H, K)] == -1).all())
    lo, hi = s0[:, None, None], pos[:, None, None]
    ok = (idx >= lo) & (idx <= hi)
    assert bool(ok[live.expand(T, H, K)].all())
    # distinct live ids per list
    srt = torch.sort(torch.where(live.expand(T, H, K), idx, torch.full_like(idx, -1)), dim=2).values
    dup = (srt[:, :, 1:] == srt[:, :, :-1]) & (srt[:, :, 1:] >= 0)
    assert not bool(dup.any())
    full = n_caus > K
    # short rows: exactly every causal slot s0..pos, in order
    short = ~full
    if short.any():
        exp = s0[short, None] + ar[None, :]
        got = idx[short][:, 0, :]
        m = ar[None, :] < n_caus[short, None]
        assert torch.equal(got[m], exp[m])
    # full rows: the local window pos-L+1..pos plus K-L ids drawn before it
    if full.any():
        f = idx[full]                                         # [F, H, K]
        pf = pos[full][:, None, None]
        in_window = (f > pf - L) & (f <= pf)
        assert bool((in_window.sum(dim=2) == L).all())
        before = f <= pf - L
        assert bool((before.sum(dim=2) == K - L).all())
    # order: sorted configs ascend; unsorted ones are not all ascending
    asc = (idx[:, :, 1:] >= idx[:, :, :-1]) | (idx[:, :, 1:] < 0)
    if ordered:
        assert bool(asc.all())
    else:
        assert not bool(asc[full].all())


def test_c3_two_sequences_and_c5_positions():
    w = W.make("c3", device="cpu")
    s0 = w.seq_start.long()
    assert s0[:8192].eq(0).all() and s0[8192:].eq(8192).all()
    w5 = W.make("c5", device="cpu", T=64)
    pos = w5.positions.long()
    assert int(pos[0]) == 131072 - 64 and int(pos[-1]) == 131071
    assert w5.k_cache.shape[0] == 131072 and w5.topk_idx.shape[1] == 2
    # the two KV heads draw independent random parts
    assert not torch.equal(w5.topk_idx[:, 0], w5.topk_idx[:, 1])


def test_decode_lists_stay_in_their_sequence():
    w = W.config_decode(device="cpu", B=4, ctx=4096, heads=(24, 2), topk=1024, local=64)
    idx = w.topk_idx.long()
    for b in range(4):
        lo, hi = b * 4096, (b + 1) * 4096 - 1
        assert int(w.positions[b]) == hi
        assert bool(((idx[b] >= lo) & (idx[b] <= hi)).all())
        for g in range(2):
            row = idx[b, g]
            assert row.unique().numel() == 1024
            assert bool(((row > hi - 64) & (row <= hi)).sum() == 64)


def test_block_lists_name_causal_blocks_with_a_masked_tail():
    w = W.config_c5_block4(device="cpu", T=48, blocks=128, local_blocks=16)
    idx = w.topk_idx.long()
    pos = w.positions.long()
    last_block = pos // 4
    # every entry is a block that starts at or before the token's slot
    assert bool((idx >= 0).all()) and bool((idx <= last_block[:, None, None]).all())
    # the newest block is listed (its slots past the token are masked by last_slot)
    assert bool((idx == last_block[:, None, None]).any(dim=2).all())
    assert torch.equal(w.last_slot.long(), pos)
    for t in range(0, 48, 7):
        for g in range(2):
            assert idx[t, g].unique().numel() == 128
