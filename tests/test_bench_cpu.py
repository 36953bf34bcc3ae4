"""The benchmark's accounting, checked on the CPU: the algorithmic bytes and
FLOPs it divides by the measured time, the compulsory bytes, and the DRAM
traffic it reads from the committed ncu summary only while the kernel
sources it was taken on are unchanged."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from top_sparse_attention_qsa_b200 import workloads as W  # noqa: E402


def _case():
    # 3 tokens, 2 KV heads of G = 3, K = 4: hand-placed masks
    w = W.generic_case(T=3, S=50, Hq=6, Hkv=2, K=4, seed=3)
    w.topk_idx = torch.tensor([[[1, 2, 3, 4], [5, -1, 5, 7]],
                               [[9, 9, 60, 1], [0, 1, 2, 3]],
                               [[-1, -1, -1, -1], [4, 3, 2, 1]]], dtype=torch.int32)
    w.n_valid = torch.tensor([[4, 3], [4, 2], [4, 4]], dtype=torch.int32)
    return w


def test_accounting_counts_live_entries():
    w = _case()
    # live: row (0,0) 4; (0,1) first 3 minus one -1 = 2; (1,0) 4 minus the
    # out-of-range 60 = 3; (1,1) first 2 = 2; (2,0) 0; (2,1) 4
    entries = 4 + 2 + 3 + 2 + 0 + 4
    a = bench.workload_accounting(w)
    assert a["entries"] == entries
    D, T, Hq, G = 256, 3, 6, 3
    assert a["gathered_bytes"] == entries * 2 * D * 2
    assert a["algo_bytes"] == entries * 1028 + T * Hq * D * 2 * 2 + T * Hq * 4
    assert a["flops"] == entries * 4 * G * D


def test_compulsory_bytes_counts_each_row_once():
    w = _case()
    # distinct live rows per KV head: head 0 {1,2,3,4,9} (9 twice, 1 twice);
    # head 1 {5,0,1,2,3,4} (5 twice)
    rows = 5 + 6
    live = 4 + 2 + 3 + 2 + 0 + 4
    D, T, Hq = 256, 3, 6
    assert bench.compulsory_bytes(w) == rows * 2 * D * 2 + T * Hq * D * 2 * 2 + T * Hq * 4 + live * 4


def test_profiled_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    # the committed summary is read while its hash matches the sources
    t = bench.profiled_traffic("c5", 16384)
    summary = open(os.path.join(ROOT, "profiles", "traffic_c5.txt")).read()
    if "kernel_source_sha256_16: " + bench.kernel_source_hash() in summary:
        assert t is not None and t > 0
    # a summary taken on other sources, or scaled from fewer units
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic_x.txt").write_text("kernel_source_sha256_16: 0000000000000000\n"
                                        "units_captured: 10\ndram_bytes_per_launch: 1000\n")
    (prof / "traffic_y.txt").write_text(f"kernel_source_sha256_16: {bench.kernel_source_hash()}\n"
                                        "units_captured: 10\ndram_bytes_per_launch: 1000\n")
    csrc = tmp_path / "top_sparse_attention_qsa_b200"
    csrc.symlink_to(os.path.join(ROOT, "top_sparse_attention_qsa_b200"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("x", 40) is None
    assert bench.profiled_traffic("y", 40) == 4000.0
    assert bench.profiled_traffic("missing", 40) is None
