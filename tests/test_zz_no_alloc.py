"""The allocation-free decode entry point against the ordinary one.

qsa_sparse_decode_fwd_noalloc serves callers that cannot allocate device
memory: it keeps the chunk scratch in a fixed array inside the library
instead of a caller-provided workspace.  These tests call it through the C
ABI and check that it returns what qsa_sparse_decode_fwd returns (with a
workspace the test allocates) on two calls in a row, and that a call too
big for the array is refused.  The file sorts last so that a run stopping at
the first failure has already run every other test; it also passes on its
own in a fresh process.
"""
import numpy as np
import pytest
import torch

from top_sparse_attention_qsa_b200 import workloads as W

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


@pytest.fixture(scope="module")
def C():
    from top_sparse_attention_qsa_b200 import _capi
    return _capi


def _close(a, la, b, lb):
    """The parity tolerance of the other tests: 1e-2 + 1e-2|ref| on out, 1e-3 on lse."""
    r = b.double().cpu().numpy()
    o = a.double().cpu().numpy()
    assert np.all(np.abs(o - r) <= 1e-2 + 1e-2 * np.abs(r))
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isneginf(la), torch.isneginf(lb))
    assert float((la[fin] - lb[fin]).abs().max()) <= 1e-3


def test_noalloc_matches_workspace_entry_point_twice(C):
    for call, seed in enumerate((101, 202)):
        # different inputs on each call: nothing may carry over in the shared array
        w = W.config_decode(device=DEV, seed=seed, B=16, ctx=8192, heads=(24, 2), topk=2048, local=256)
        if call == 1:
            w.n_valid[3] = 0                       # an empty row on the second call
        need = C.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, 4)
        assert 0 < need <= C.NOALLOC_SCRATCH_BYTES
        ref_out, ref_lse = C.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid,
                                               w.scale, num_splits=4)
        out = torch.full_like(w.q, 7.0)
        lse = torch.full(w.q.shape[:2], 7.0, dtype=torch.float32, device=DEV)
        C.sparse_decode_fwd_noalloc(w.q, w.k_cache, w.v_cache, w.topk_idx, out, lse,
                                    n_valid=w.n_valid, scale=w.scale, num_splits=4)
        torch.cuda.synchronize()
        _close(out, lse, ref_out, ref_lse)


def test_noalloc_refuses_oversized_calls(C):
    # 64 tokens x 24 heads x 64 chunks x (1 KB + 4 B) of partials > 16 MiB
    w = W.config_decode(device=DEV, B=64, ctx=8192, heads=(24, 2), topk=8192, local=64)
    assert C.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, 64) > C.NOALLOC_SCRATCH_BYTES
    out = torch.empty_like(w.q)
    with pytest.raises(C.QSAError) as e:
        C.sparse_decode_fwd_noalloc(w.q, w.k_cache, w.v_cache, w.topk_idx, out,
                                    n_valid=w.n_valid, num_splits=64)
    assert e.value.code == C.QSA_ERR_SCRATCH


def _pair(C, w, splits):
    ref_out, ref_lse = C.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                           num_splits=splits)
    out = torch.full_like(w.q, 7.0)
    lse = torch.full(w.q.shape[:2], 7.0, dtype=torch.float32, device=DEV)
    C.sparse_decode_fwd_noalloc(w.q, w.k_cache, w.v_cache, w.topk_idx, out, lse, n_valid=w.n_valid,
                                scale=w.scale, num_splits=splits)
    torch.cuda.synchronize()
    return out, lse, ref_out, ref_lse


def test_noalloc_automatic_and_single_chunk_choices(C):
    # few (token, KV head) units: the automatic choice splits the lists
    w = W.config_decode(device=DEV, seed=303, B=2, ctx=8192, heads=(24, 2), topk=2048, local=256)
    assert C.decode_num_splits(w.q, w.k_cache, w.topk_idx, 0) > 1
    _close(*_pair(C, w, 0))
    # one chunk: no scratch at all, the prefill kernel runs directly
    assert C.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, 1) == 0
    _close(*_pair(C, w, 1))


def test_noalloc_smaller_call_after_larger(C):
    # a large call leaves its partials in the shared array; a smaller one
    # that follows must read only its own
    big = W.config_decode(device=DEV, seed=404, B=16, ctx=8192, heads=(24, 2), topk=2048, local=256)
    small = W.config_decode(device=DEV, seed=505, B=3, ctx=4096, heads=(12, 1), topk=1024, local=128)
    _close(*_pair(C, big, 8))
    _close(*_pair(C, small, 2))


def test_noalloc_allocates_nothing(C):
    w = W.config_decode(device=DEV, seed=606, B=8, ctx=8192, heads=(24, 2), topk=2048, local=256)
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=DEV)
    C.sparse_decode_fwd_noalloc(w.q, w.k_cache, w.v_cache, w.topk_idx, out, lse, n_valid=w.n_valid,
                                scale=w.scale, num_splits=4)                 # warm-up: module loaded
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    for _ in range(3):
        C.sparse_decode_fwd_noalloc(w.q, w.k_cache, w.v_cache, w.topk_idx, out, lse, n_valid=w.n_valid,
                                    scale=w.scale, num_splits=4)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_against_the_oracle(C):
    """The allocation-free path checked on its own against the FP64 oracle,
    not only against the workspace path that shares its kernels."""
    import oracle
    w = W.config_decode(device=DEV, seed=707, B=6, ctx=8192, heads=(16, 2), topk=2048, local=256)
    w.n_valid[2, 1] = 700
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=DEV)
    C.sparse_decode_fwd_noalloc(w.q, w.k_cache, w.v_cache, w.topk_idx, out, lse, n_valid=w.n_valid,
                                scale=w.scale, num_splits=4)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle.sparse_prefill(w.q.cpu(), w.k_cache.cpu(), w.v_cache.cpu(), w.topk_idx.cpu(),
                                                w.n_valid.cpu(), w.scale)
    o = out.double().cpu().numpy()
    assert np.all(np.abs(o - ref_out) <= 1e-2 + 1e-2 * np.abs(ref_out))
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= 1e-3
