"""Split-K sparse decode (qsa_sparse_decode_fwd) against the FP64 oracle.

Decode-shaped calls (one query token per sequence, long lists) cut each list
into chunks on separate CTAs and merge the partial results by log-sum-exp
(page "Qwen4-Exp QSA llega al Ascend de Huawei", section "Dónde encaja esto
en el despliegue del servicio de Qwen4Exp": decode context parallelism for
the QSA path).  The merge is exact, so the bar is the prefill bar.
"""
import ctypes

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


def decode(C, w, **kw):
    return C.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale, **kw)


def check(C, w, label, **kw):
    out, lse = decode(C, w, **kw)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = run_oracle(w)
    return compare(host(out), host(lse), ref_out, ref_lse, label)


def test_decode_config_full():
    """64 sequences x 32768 cached tokens, heads (24,2), K=2048, auto chunks."""
    from top_sparse_attention_qsa_b200 import _capi as C
    w = W.make("decode", device=DEV)
    print(check(C, w, "decode"))
    print(check(C, w, "decode_4_chunks", num_splits=4))


def test_decode_few_units_auto_splits():
    """Two sequences, one KV head: units are scarce, so the automatic choice splits."""
    from top_sparse_attention_qsa_b200 import _capi as C
    w = W.config_decode(device=DEV, B=2, ctx=20000, heads=(12, 1), topk=4096, local=128)
    assert C.decode_num_splits(w.q, w.k_cache, w.topk_idx) > 1
    check(C, w, "decode_auto")


@pytest.mark.parametrize("units", [1, 8, 16, 32, 48, 64, 74, 75, 96, 128, 300])
def test_decode_auto_splits_fill_one_wave(C, units):
    """The automatic chunk count: floor(SMs / units) chunks (all chunks in one
    wave of one CTA per SM), never chunks under 256 entries, one chunk once
    the units exceed half the SMs.  Shapes only: nothing is launched."""
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    K = 2048
    q = torch.empty((units, 2, 256), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((16, 1, 256), dtype=torch.bfloat16, device=DEV)
    idx = torch.empty((units, 1, K), dtype=torch.int32, device=DEV)
    want = min(nsm // units, K // 256) if 2 * units <= nsm else 1
    assert C.decode_num_splits(q, k, idx, 0) == max(want, 1)
    assert C.decode_num_splits(q, k, idx, 4) == 4


@pytest.mark.parametrize("splits", [0, 1, 2, 3, 7, 16, 100])
def test_decode_splits(C, splits):
    w = W.config_decode(device=DEV, B=6, ctx=4096, heads=(12, 1), topk=2051, local=64)
    st = check(C, w, f"splits{splits}", num_splits=splits)
    assert st["rows"] == 6 * 12


@pytest.mark.parametrize("heads", W.HEAD_SHAPES)
def test_decode_head_shapes(C, heads):
    w = W.config_decode(device=DEV, B=3, ctx=3000, heads=heads, topk=700, local=32)
    check(C, w, f"decode{heads}", num_splits=4)


def test_decode_ragged_and_empty(C):
    w = W.config_decode(device=DEV, B=8, ctx=2000, heads=(16, 2), topk=640, local=16)
    nv = w.n_valid.clone()
    nv[0] = 0             # empty list: every chunk empty
    nv[1] = 128           # ends exactly at a chunk boundary
    nv[2, 0] = 129        # one entry into the second chunk
    nv[3] = 1
    nv[4, 1] = 383
    w.n_valid = nv
    w.topk_idx[5, :, 100:400] = -1     # a chunk that is entirely interior -1
    st = check(C, w, "ragged", num_splits=5)
    assert st["empty_rows"] >= 16


def test_decode_matches_prefill_kernel(C):
    w = W.config_decode(device=DEV, B=4, ctx=5000, heads=(24, 2), topk=1500, local=64)
    a, la = decode(C, w, num_splits=6)
    b, lb = C.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale)
    torch.cuda.synchronize()
    r = b.double().cpu().numpy()
    assert np.all(np.abs(a.double().cpu().numpy() - r) <= 1e-2 + 1e-2 * np.abs(r))
    assert float((la - lb).abs().max()) <= 1e-3
    # deterministic
    c, lc = decode(C, w, num_splits=6)
    assert torch.equal(a, c) and torch.equal(la, lc)


def test_decode_workspace_checks(C):
    w = W.config_decode(device=DEV, B=2, ctx=3000, heads=(6, 1), topk=1000, local=16)
    need = C.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, 4)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(C.QSAError) as e:
        decode(C, w, num_splits=4, workspace=small)
    assert e.value.code == C.QSA_ERR_SHAPE
    big = torch.empty(need + 512, dtype=torch.uint8, device=DEV)
    with pytest.raises(C.QSAError) as e:
        decode(C, w, num_splits=4, workspace=big[16:])            # not 256-byte aligned
    assert e.value.code == C.QSA_ERR_ALIGN
    out, lse = decode(C, w, num_splits=4, workspace=big)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = run_oracle(w)
    compare(host(out), host(lse), ref_out, ref_lse, "ws")
    # a single chunk needs no workspace
    assert C.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, 1) == 0


def test_decode_oob_status(C):
    w = W.config_decode(device=DEV, B=3, ctx=1000, heads=(3, 1), topk=400, local=8)
    w.topk_idx[1, 0, 300] = w.k_cache.shape[0] + 5
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, lse = decode(C, w, num_splits=3, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & C.STATUS_OOB_SLOT
    ref_out, ref_lse, n = run_oracle(w)
    assert n == 1
    compare(host(out), host(lse), ref_out, ref_lse, "decode_oob")
