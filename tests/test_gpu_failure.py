"""Failure detection without a GPU fault: a stalled pipeline ends with an
error status, never a hang.

Every wait inside the tcgen05 kernel is bounded (2 s of %globaltimer).  The
test hook withholds the producers' signal for the first shared-memory slot of
every CTA, so no stage can complete: the kernel must stop on its own, set
QSA_STATUS_TIMEOUT, release its tensor memory, and leave the CUDA context
usable for the next call.
"""
import time

import pytest
import torch

from top_sparse_attention_qsa_b200 import workloads as W
from parity import compare, host, run_gpu, run_oracle

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def test_stalled_pipeline_reports_timeout_and_context_survives():
    from top_sparse_attention_qsa_b200 import _capi as C
    from top_sparse_attention_qsa_b200 import _debug as D
    w = W.generic_case(T=8, S=2000, Hq=12, Hkv=1, K=300, seed=3, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.time()
    D.run_stalled_pipeline_check(w.q, w.k_cache, w.v_cache, w.topk_idx, status)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert int(status.item()) & C.STATUS_TIMEOUT
    assert elapsed < 30.0
    # the context is intact: a normal call right after is correct
    out, lse = run_gpu(w, "tcgen05")
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = run_oracle(w)
    compare(host(out), host(lse), ref_out, ref_lse, "after_stall")
