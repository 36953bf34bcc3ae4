"""Scores of about +-1000: the online softmax's lazy rescale under stress.

The kernels keep a running maximum per head and raise it (rescaling O and the
partial sums) only when a tile's maximum exceeds it by more than 2^8 in base
2.  These cases drive scores to about +-1100 (page "Qwen4-Exp QSA llega al
Ascend de Huawei", section "Lo que realmente añade la pull request": a
softmax over the selected rows, which must hold for any score range) and
order each list so that the running maximum rises on every tile (ascending
scores), never rises after the first tile (descending), or at random.

The inputs are small integers (Q = c_h * a with c_h a signed power of two and
a in [-4, 4]; K rows m_s * sign(a) + e with m_s in [-4, 4] and e in {-1, 0,
1}), so every product and partial sum of the scores is an integer far below
2^24: FP32 accumulation is exact in any order, and the comparison with the
FP64 oracle at the usual tolerances tests the softmax, not the accumulation
order.  Heads with c_h > 0 see ascending scores while heads with c_h < 0 of
the same list see descending ones.
"""
import pytest
import torch

import oracle
from top_sparse_attention_qsa_b200 import workloads as W
from parity import compare, host

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


def extreme_case(heads, order, T=48, S=4096, K=1024, seed=0):
    Hq, Hkv = heads
    G = Hq // Hkv
    g = torch.Generator().manual_seed(seed)
    a = torch.randint(-4, 5, (256,), generator=g)
    a[a == 0] = 1
    # per query head a signed power of two: 8, -8, 4, -4, 2, -2, 1, -1, ...
    mags = torch.tensor([8, 4, 2, 1], dtype=torch.int64)
    c = torch.stack([mags[(h // 2) % 4] * (1 if h % 2 == 0 else -1) for h in range(G)])
    q = (c[:, None] * a[None, :]).repeat(Hkv, 1)                    # [Hq, 256]
    q = q[None].expand(T, Hq, 256).to(torch.bfloat16).contiguous()
    m = torch.randint(-4, 5, (S, Hkv, 1), generator=g)
    e = torch.randint(-1, 2, (S, Hkv, 256), generator=g)
    k = m * torch.sign(a)[None, None, :] + e                      # |k| <= 5
    v = W.normal_bf16((S, Hkv, 256), torch.Generator().manual_seed(seed + 1), "cpu")
    # integer score of every slot per KV head: <a, k_s> (exact)
    base = (k * a[None, None, :]).sum(-1)                         # [S, Hkv]
    idx = torch.empty((T, Hkv, K), dtype=torch.int64)
    for t in range(T):
        for kv in range(Hkv):
            sel = torch.randperm(S, generator=g)[:K]
            sc = base[sel, kv]
            if order == "ascending":
                sel = sel[torch.argsort(sc, stable=True)]
            elif order == "descending":
                sel = sel[torch.argsort(-sc, stable=True)]
            idx[t, kv] = sel
    w = W.Workload(f"extreme_{order}", q.to(DEV), k.to(torch.bfloat16).to(DEV), v.to(DEV),
                   idx.to(torch.int32).to(DEV), None, 1.0 / 16, torch.zeros(T, dtype=torch.int32, device=DEV),
                   torch.zeros(T, dtype=torch.int32, device=DEV), "integer inputs, scores up to ~1100")
    smax = float((base.abs().max() * c.abs().max()).item()) / 16
    return w, smax


@pytest.mark.parametrize("order", ["ascending", "descending", "random"])
@pytest.mark.parametrize("heads", [(16, 2), (12, 1)])
@pytest.mark.parametrize("kernel", ["tcgen05", "warp_mma"])
def test_extreme_scores(order, heads, kernel):
    from top_sparse_attention_qsa_b200 import _capi
    w, smax = extreme_case(heads, order, seed={"ascending": 1, "descending": 2, "random": 3}[order] + heads[0])
    assert smax > 900                       # the scores really reach about +-1000
    out, lse = _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, None, w.scale, kernel=kernel)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle.sparse_prefill(host(w.q), host(w.k_cache), host(w.v_cache),
                                                host(w.topk_idx), None, w.scale)
    assert float(abs(ref_lse).max()) > 500
    compare(host(out), host(lse), ref_out, ref_lse, f"extreme {order} {heads} {kernel}")


@pytest.mark.parametrize("order", ["ascending", "descending", "random"])
def test_extreme_scores_fp8_cache(order):
    """The same lists over an FP8 E4M3 cache (the integers |k| <= 5 are exact
    in E4M3), through the FP8 kernel."""
    from top_sparse_attention_qsa_b200 import _capi
    w, _ = extreme_case((24, 2), order, seed=7)
    k8 = w.k_cache.float().to(torch.float8_e4m3fn)
    assert torch.equal(k8.float(), w.k_cache.float())
    v8 = w.v_cache.float().to(torch.float8_e4m3fn)
    out, lse = _capi.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 1.0, 1.0, scale=w.scale)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle.sparse_prefill(host(w.q), host(k8), host(v8), host(w.topk_idx), None, w.scale,
                                                k_scale=1.0, v_scale=1.0)
    compare(host(out), host(lse), ref_out, ref_lse, f"extreme fp8 {order}")


def test_extreme_scores_split_decode():
    """Split-K decode over such lists: chunk maxima far apart, merged by lse."""
    from top_sparse_attention_qsa_b200 import _capi
    w, _ = extreme_case((24, 2), "ascending", T=4, K=2048, seed=11)
    out, lse = _capi.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, None, w.scale, num_splits=8)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle.sparse_prefill(host(w.q), host(w.k_cache), host(w.v_cache),
                                                host(w.topk_idx), None, w.scale)
    compare(host(out), host(lse), ref_out, ref_lse, "extreme split decode")
