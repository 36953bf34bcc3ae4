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
