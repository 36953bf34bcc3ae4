"""The FP64 oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_pages_facts_consistent(pages_facts):
    # the packed-extent cap: 262144 tokens x 2 KV heads x [K,V] = 2*256 BF16
    # columns x 2 bytes is the 512 MiB the page states for C=[K,V]
    cap = pages_facts["packed_extent_cap"]["value"]
    D = pages_facts["head_dim"]["value"]
    assert cap["tokens"] * cap["kv_heads"] * (2 * D) * 2 == cap["mib"] * 2**20
    # every head shape's group pads to the stated power of two
    pad = {int(k): v for k, v in pages_facts["power_of_two_padding"]["value"].items()}
    for hq, hkv in pages_facts["head_shapes"]["value"]:
        g = hq // hkv
        p2 = 1 << (g - 1).bit_length()
        assert p2 == pad.get(g, g)
    # 2051 = 2048 selected microblock slots + a causal tail of 3 at ratio 4
    assert 2051 - 2048 in pages_facts["causal_tail_remainders"]["value"]


def test_oracle_threads_agree(orc):
    from top_sparse_attention_qsa_b200 import workloads as W
    import numpy as np
    w = W.make("tiny")
    a = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale, n_threads=1)
    b = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale, n_threads=8)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    sub = [5, 200, 17]
    c = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale, tokens=sub)
    np.testing.assert_array_equal(c[0], a[0][sub])


def test_oracle_rejects_bad_args(orc):
    from top_sparse_attention_qsa_b200 import workloads as W
    w = W.generic_case(3, 8, 6, 2, 4, 1)
    with pytest.raises(ValueError):
        orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, tokens=[3])
    with pytest.raises(ValueError):
        orc.sparse_prefill(w.q[:, :5], w.k_cache, w.v_cache, w.topk_idx)


def test_oracle_regression_fixture(orc):
    """Drift guard: rows written earlier by tests/golden/make_golden.py."""
    import numpy as np
    from conftest import load_golden
    from top_sparse_attention_qsa_b200 import workloads as W
    doc = load_golden("oracle_tiny_rows.json")
    w = W.make("tiny", device="cpu")
    out, lse, _ = orc.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                     tokens=doc["tokens"])
    want_lse = np.array([[float(x) for x in r] for r in doc["lse"]])
    want_out = np.array([[[float(x) for x in h] for h in r] for r in doc["out_first8"]])
    np.testing.assert_allclose(lse, want_lse, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(out[:, :, :8], want_out, rtol=1e-13, atol=1e-13)
