"""Writes tests/golden/oracle_tiny_rows.json: oracle values for a few rows of
the tiny configuration (CPU-drawn inputs, fixed seed).  Calls only the oracle
and the seeded input generator; the file guards the oracle against drift."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from top_sparse_attention_qsa_b200 import workloads as W  # noqa: E402

TOKENS = [0, 1, 62, 63, 64, 255]


def main():
    w = W.make("tiny", device="cpu")
    out, lse, _ = oracle.sparse_prefill(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid,
                                        w.scale, tokens=TOKENS)
    doc = {
        "what": "Oracle rows of the tiny configuration (T=256, S=256, heads (3,1), K=64, seed 20261001, CPU generator)",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "tokens": TOKENS,
        "lse": [[repr(float(x)) for x in row] for row in lse],
        "out_first8": [[[repr(float(x)) for x in out[i, h, :8]] for h in range(out.shape[1])]
                       for i in range(len(TOKENS))],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_rows.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
