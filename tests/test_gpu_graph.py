"""Every device-buffer entry point inside a CUDA graph.

The library never allocates, frees or synchronises inside a call and reads
no device value on the host, so a call can be captured into a CUDA graph
and replayed with new contents in the same buffers (the pages' adapter
copies two scalars to the host on every call, which rules that out: page
"Qwen4-Exp QSA llega al Ascend de Huawei", section "Lo que realmente añade
la pull request").  Each test captures the calls once, replays them on two
different inputs written into the captured buffers, and requires the replay
to equal an eager call on the same inputs bit for bit (the kernels have no
order-dependent reductions); the first replay is also held to the oracle.
"""
import numpy as np
import pytest
import torch

from top_sparse_attention_qsa_b200 import workloads as W
from parity import compare, host, run_oracle

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


@pytest.fixture(scope="module")
def C():
    from top_sparse_attention_qsa_b200 import _capi
    return _capi


def _capture(fn):
    """Warm up on a side stream (first-call attribute setting happens there),
    then capture fn() into a graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _refill(dst, src):
    for d, s in zip(dst, src):
        d.copy_(s)


def test_prefill_graph_replays_new_inputs(C):
    w0 = W.make("c2", device=DEV)
    w1 = W.make("c2", device=DEV, seed=991)
    q, k, v, idx, nv = (x.clone() for x in (w0.q, w0.k_cache, w0.v_cache, w0.topk_idx, w0.n_valid))
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
    g = _capture(lambda: C.sparse_prefill_fwd(q, k, v, idx, nv, w0.scale, out=out, lse=lse))
    for i, w in enumerate((w1, w0)):
        _refill((q, k, v, idx, nv), (w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid))
        out.fill_(7.0)
        lse.fill_(7.0)
        g.replay()
        e_out, e_lse = C.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale)
        torch.cuda.synchronize()
        assert torch.equal(out, e_out) and torch.equal(lse, e_lse)
        if i == 0:
            ref_out, ref_lse, _ = run_oracle(w)
            compare(host(out), host(lse), ref_out, ref_lse, "c2 graph replay")


def test_decode_graph_with_workspace(C):
    w0 = W.config_decode(device=DEV, seed=5, B=16, ctx=8192, heads=(24, 2), topk=2048, local=256)
    w1 = W.config_decode(device=DEV, seed=6, B=16, ctx=8192, heads=(24, 2), topk=2048, local=256)
    w1.n_valid[2] = 0
    w1.n_valid[5] = 300
    q, k, v, idx, nv = (x.clone() for x in (w0.q, w0.k_cache, w0.v_cache, w0.topk_idx, w0.n_valid))
    ws = torch.empty(C.decode_workspace_bytes(q, k, idx, 4), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
    g = _capture(lambda: C.sparse_decode_fwd(q, k, v, idx, nv, w0.scale, num_splits=4, workspace=ws,
                                             out=out, lse=lse))
    for i, w in enumerate((w1, w0)):
        _refill((q, k, v, idx, nv), (w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid))
        g.replay()
        e_out, e_lse = C.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                           num_splits=4)
        torch.cuda.synchronize()
        assert torch.equal(out, e_out) and torch.equal(lse, e_lse)
        if i == 0:
            ref_out, ref_lse, _ = run_oracle(w)
            compare(host(out), host(lse), ref_out, ref_lse, "decode graph replay")


def test_fp8_prefill_graph(C):
    w = W.make("c2", device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(13)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, DEV)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, DEV)
    q = w.q.clone()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)
    g = _capture(lambda: C.sparse_prefill_fp8_fwd(q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid,
                                                  scale=w.scale, out=out, lse=lse))
    for seed in (21, 22):
        q.copy_(W.normal_bf16(tuple(q.shape), torch.Generator(device=DEV).manual_seed(seed), DEV))
        g.replay()
        e_out, e_lse = C.sparse_prefill_fp8_fwd(q.clone(), k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid,
                                                scale=w.scale)
        torch.cuda.synchronize()
        assert torch.equal(out, e_out) and torch.equal(lse, e_lse)


def test_indexer_selection_attention_graph(C):
    """The launches of one QSA step (head folding and indexer scores, top-K
    microblocks, microblock attention) captured as one graph; the folded
    query buffer is allocated inside the capture, from the graph's pool."""
    T, S, budget = 64, 4096, 96
    wi = W.config_indexer(device=DEV, seed=51, T=T, S=S, heads=4, seq_starts=[0, 2048])
    gen = torch.Generator(device=DEV).manual_seed(52)
    q = W.normal_bf16((T, 24, 256), gen, DEV)
    k = W.normal_bf16((S, 2, 256), gen, DEV)
    v = W.normal_bf16((S, 2, 256), gen, DEV)
    q_idx = wi.q_idx.clone()
    NB = wi.k_idx.shape[0]
    scores = torch.full((T, (NB + 3) // 4 * 4), float("-inf"), dtype=torch.float32, device=DEV)[:, :NB]
    lists = torch.empty((T, budget + 1), dtype=torch.int32, device=DEV)
    nv = torch.empty((T, 2), dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=DEV)

    def step():
        C.indexer_scores(q_idx, wi.k_idx, wi.positions, wi.seq_start, 4, scores=scores)
        C.topk_select(scores, wi.positions, wi.seq_start, NB, budget, 4, append_tail=True, lists=lists,
                      n_valid=nv, copies=2)
        C.sparse_prefill_block_fwd(q, k, v, lists[:, None, :].expand(T, 2, budget + 1), 4, wi.positions,
                                   nv, 0.0, out=out, lse=lse)

    g = _capture(step)
    for seed in (53, 54):
        q_idx.copy_(W.normal_bf16(tuple(q_idx.shape), torch.Generator(device=DEV).manual_seed(seed), DEV))
        g.replay()
        e_lists, e_nv, _ = C.indexer_select(q_idx.clone(), wi.k_idx, wi.positions, wi.seq_start, budget, 4,
                                            append_tail=True, copies=2)
        e_out, e_lse = C.sparse_prefill_block_fwd(q, k, v, e_lists[:, None, :].expand(T, 2, budget + 1), 4,
                                                  wi.positions, e_nv, 0.0)
        torch.cuda.synchronize()
        assert torch.equal(lists, e_lists) and torch.equal(nv, e_nv)
        assert torch.equal(out, e_out) and torch.equal(lse, e_lse)
        assert not np.array_equal(host(lists).numpy()[:, :8], np.zeros((T, 8), np.int32))
