"""The measurement kernels of libqsa_debug.so on the GPU: the prefill
kernels' gather run alone (the floor the bench reports) and the independent
random-row gather probe that gives the roofline its gather ceiling."""
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


@pytest.fixture(scope="module")
def D():
    from top_sparse_attention_qsa_b200 import _debug
    return _debug


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_gather_only_flags_ids_and_writes_nothing(C, D, cache):
    """The gather-only kernels read the same lists and report out-of-range ids
    like the full kernels, and write no output."""
    w = W.make("c2", device=DEV)
    if cache == "fp8":
        gen = torch.Generator(device=DEV).manual_seed(5)
        k, v = W.normal_fp8(tuple(w.k_cache.shape), gen, DEV), W.normal_fp8(tuple(w.v_cache.shape), gen, DEV)
    else:
        k, v = w.k_cache, w.v_cache
    q_before = w.q.clone()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    D.gather_only(w.q, k, v, w.topk_idx, w.n_valid, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    w.topk_idx[7, 0, 3] = w.k_cache.shape[0] + 11
    D.gather_only(w.q, k, v, w.topk_idx, w.n_valid, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & C.STATUS_OOB_SLOT
    assert torch.equal(w.q, q_before)


@pytest.mark.parametrize("row_bytes", [256, 512])
@pytest.mark.parametrize("method,depth,warps", [("cp_async", 4, 8), ("cp_async", 8, 4), ("ld_v4", 8, 16),
                                                ("ld_v4", 16, 16), ("bulk", 2, 4), ("bulk", 4, 2)])
def test_gather_peak_runs_clean(D, row_bytes, method, depth, warps):
    rows = 1 << 15
    table = torch.randint(0, 255, (rows, 512), dtype=torch.uint8, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(1)
    ids = torch.randint(0, rows, (1 << 20,), generator=gen, device=DEV, dtype=torch.int32)
    ids[::97] = rows + 5                       # out-of-range ids read row 0, never outside the table
    sink = torch.zeros(148 * 8 * 32 * 32, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    D.gather_peak(table, ids, row_bytes, method, depth, warps, 1, sink=sink, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    if method == "ld_v4":
        assert bool((sink != 0).any())


def test_gather_peak_refuses_an_oversized_ring(C, D):
    table = torch.zeros((1024, 512), dtype=torch.uint8, device=DEV)
    ids = torch.zeros(4096, dtype=torch.int32, device=DEV)
    with pytest.raises(C.QSAError) as e:
        D.gather_peak(table, ids, 512, "bulk", 4, 8)     # 8 warps x 4 stages x 16 KB > 227 KB
    assert e.value.code == C.QSA_ERR_UNSUPPORTED
