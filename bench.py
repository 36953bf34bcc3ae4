#!/usr/bin/env python
"""QSA sparse-attention prefill benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5] [--impl cuda|reference]

A step is one pass of the whole hot path -- index load/mask, KV gather,
scores, online softmax, PV, epilogue: one launch of the sparse-prefill
kernel -- over one batch of synthetic input already resident in HBM.  The
default workload is the chunked long prefill: 8192 new query tokens at
positions 122880..131071 over a 131072-slot cache, heads (24,2), D=256,
top-K=2048 (256 local + 1792 random earlier slots, unsorted).

value  = query tokens/s over all ranks (each rank runs its own replica; the
         path has no exchange step, so scaling is weak).
e2e    = the same metric through the host-buffer C-ABI entry point: every
         step copies Q, both caches, the lists and n_valid host->device and
         the output and lse device->host inside the timed region.
roofline: algorithmic bytes per launch (1024 B of K+V rows and 4 B of list
         entry per live entry, plus Q and out rows and the lse) over the
         kernel's mean event-timed duration, against the measured HBM copy
         bandwidth.
cpu_baseline: the FP64 oracle on a bounded token sample (rank 0, N=1).
--impl reference: times only the FP64 oracle (the CPU reference arm).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "QSA sparse prefill query-tokens/s and gathered-KV GB/s (% of B200 roofline)"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_NAMES = {"auto": "qsa_prefill_tc_kernel", "tcgen05": "qsa_prefill_tc_kernel",
                "warp_mma": "qsa_prefill_mma_kernel"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="c5",
                    choices=["tiny", "c2", "c3", "c4", "c5", "pages_long"])
    ap.add_argument("--secondary", default="c4",
                    help="second workload reported under 'secondary' ('' to skip)")
    ap.add_argument("--kernel", default="auto", choices=["auto", "tcgen05", "warp_mma"])
    ap.add_argument("--shard", default="replicas", choices=["replicas", "tokens", "heads"],
                    help="N>1: independent replicas (weak scaling) or one workload's tokens split (strong)")
    ap.add_argument("--compare", default="warp_mma",
                    help="second kernel timed on the same workload ('' to skip)")
    ap.add_argument("--decode", default="decode",
                    help="decode workload timed under 'decode' ('' to skip)")
    ap.add_argument("--blocks", default="c5_block4",
                    help="microblock-list workload timed under 'blocks' ('' to skip)")
    ap.add_argument("--fp8", default="c5",
                    help="workload timed with an FP8 E4M3 KV cache under 'fp8' ('' to skip)")
    ap.add_argument("--per-config", default="on", choices=["on", ""],
                    help="also time the five configs (tiny, c2..c5) and report each one's absolute numbers")
    ap.add_argument("--qsa-step", default="on", choices=["on", ""],
                    help="time indexer -> top-K -> microblock attention as one step ('' to skip)")
    ap.add_argument("--indexer", default="indexer",
                    help="indexer + top-K workload timed under 'indexer' ('' to skip)")
    ap.add_argument("--gather-peak", default="on", choices=["on", ""],
                    help="measure the random-row gather rate (the roofline's gather ceiling)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the query-token count of c4/c5 (smaller ncu captures)")
    ap.add_argument("--profile", action="store_true",
                    help="minimal run for ncu: no clocks, e2e, cpu baseline or secondary")
    ap.add_argument("--only", default="", choices=["", "fp8", "indexer", "blocks", "decode", "qsa_step",
                                                    "gather_peak"],
                    help="run one secondary leg alone (--steps / --warmup / --tokens apply), for "
                         "profiling; prints that leg's JSON")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def shard_range(n, world, rank):
    """[start, end) of rank's share of n units (contiguous, sizes differ by at most 1)."""
    base, rem = divmod(n, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def max_over_ranks(x, dist=None, device="cpu"):
    """Max of a host float over all ranks (the identity without a process group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_workload(w, world, rank):
    """The rank's token slice of a workload (views into the same tensors)."""
    t0, t1 = shard_range(w.shape["T"], world, rank)
    import dataclasses
    return dataclasses.replace(
        w, q=w.q[t0:t1], topk_idx=w.topk_idx[t0:t1],
        n_valid=None if w.n_valid is None else w.n_valid[t0:t1],
        positions=w.positions[t0:t1], seq_start=w.seq_start[t0:t1])


def shard_heads(w, world, rank):
    """The rank's share of the KV heads (tensor-parallel split: the rank holds
    only its heads' cache, as a compact copy), or None when the rank has no
    head (more ranks than KV heads)."""
    s = w.shape
    g0, g1 = shard_range(s["Hkv"], world, rank)
    if g1 <= g0:
        return None
    G = s["Hq"] // s["Hkv"]
    import dataclasses
    return dataclasses.replace(
        w, q=w.q[:, g0 * G:g1 * G], k_cache=w.k_cache[:, g0:g1].contiguous(),
        v_cache=w.v_cache[:, g0:g1].contiguous(), topk_idx=w.topk_idx[:, g0:g1],
        n_valid=None if w.n_valid is None else w.n_valid[:, g0:g1].contiguous())


def dataclasses_replace_empty(w):
    """A workload with no query tokens (a rank with nothing to do)."""
    import dataclasses
    return dataclasses.replace(w, q=w.q[:0], topk_idx=w.topk_idx[:0],
                               n_valid=None if w.n_valid is None else w.n_valid[:0],
                               positions=w.positions[:0], seq_start=w.seq_start[:0])


def compulsory_bytes(w):
    """Bytes a launch cannot avoid moving: every cache row named by some list
    once, plus Q, out, lse and the lists (context for the DRAM traffic)."""
    s = w.shape
    idx = w.topk_idx
    live = (idx >= 0) & (idx < s["S"])
    if w.n_valid is not None:
        live &= torch.arange(s["K"], device=idx.device)[None, None, :] < w.n_valid[:, :, None]
    rows = 0
    for g in range(s["Hkv"]):
        ids = idx[:, g][live[:, g]]
        rows += int(torch.unique(ids).numel()) if ids.numel() else 0
    return (rows * 2 * s["D"] * 2 + s["T"] * s["Hq"] * s["D"] * 2 * 2 + s["T"] * s["Hq"] * 4
            + int(live.sum().item()) * 4)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def workload_accounting(w):
    """Live list entries and the algorithmic bytes / FLOPs of one launch."""
    s = w.shape
    idx = w.topk_idx
    live = (idx >= 0) & (idx < s["S"])
    if w.n_valid is not None:
        ar = torch.arange(s["K"], device=idx.device)
        live &= ar[None, None, :] < w.n_valid[:, :, None]
    entries = int(live.sum().item())
    G = s["Hq"] // s["Hkv"]
    gathered = entries * 2 * s["D"] * 2
    algo = gathered + entries * 4 + s["T"] * s["Hq"] * s["D"] * 2 * 2 + s["T"] * s["Hq"] * 4
    flops = entries * 4 * G * s["D"]
    return dict(entries=entries, gathered_bytes=gathered, algo_bytes=algo, flops=flops)


# Device sources of the default sparse-prefill kernel (qsa_prefill_tc_kernel);
# its launch shape (persistent grid of min(units, SMs) CTAs of 512 threads)
# is fixed in qsa_launch.cuh.
PREFILL_SOURCES = ("qsa_prefill_tc.cuh", "qsa_tc_ptx.cuh", "qsa_ptx.cuh")


def kernel_source_hash(files=PREFILL_SOURCES):
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "top_sparse_attention_qsa_b200", "csrc")
    for p in sorted(os.path.join(pkg, f) for f in files):
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, units):
    """DRAM bytes per launch from a committed ncu summary, when it was taken
    on the current kernel sources (else None).  The summary records
    dram bytes for a capture of `units_captured` (token, KV head) units;
    the figure is scaled to `units` when the summary says it scales."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        b = float(kv["dram_bytes_per_launch"])
        cap = float(kv.get("units_captured", units))
    except (KeyError, ValueError):
        return None
    return b * units / cap


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms."""

    FIELDS = ["timestamp", "index", "clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.active", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            sel = str(device_index)
        self.sel = sel

    def start(self):
        try:
            # the raw samples go to $QSA_CLOCKS_DIR (kept) or the temp directory
            d = os.environ.get("QSA_CLOCKS_DIR") or tempfile.gettempdir()
            os.makedirs(d, exist_ok=True)
            self.path = os.path.join(d, f"qsa_clocks_{os.getpid()}.csv")
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0, t1):
        if self.proc is None:
            return {"unavailable": "nvidia-smi could not be started"}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    continue
                rows.append((ts, parts))
        inside = [p for ts, p in rows if t0 - 0.05 <= ts <= t1 + 0.15]
        if not inside:
            inside = [p for _, p in rows[-3:]]
        if not inside:
            return {"unavailable": "no nvidia-smi samples"}
        sm = [float(p[2]) for p in inside if p[2].replace(".", "").isdigit()]
        reasons = []
        for name, col in (("hw_slowdown", 6), ("hw_thermal_slowdown", 7),
                          ("sw_thermal_slowdown", 8), ("sw_power_cap", 9)):
            if any(p[col] == "Active" for p in inside):
                reasons.append(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(inside[0][3]) if inside[0][3].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(inside)}


def time_launches(fn, steps, warmup, barrier, label="timed"):
    for _ in range(warmup):
        fn()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    torch.cuda.nvtx.range_push(label)
    for i in range(steps):
        starts[i].record()
        fn()
        ends[i].record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total = starts[0].elapsed_time(ends[-1])
    return total, per, (t0, t1)


def time_flushed(fn, n=5):
    """Mean and median of n launches, each timed alone (CUDA events) after
    writing a 256 MB buffer that evicts the 126 MB L2."""
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    per = []
    for _ in range(n):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        per.append(a.elapsed_time(b))
    del flush
    return statistics.mean(per), statistics.median(per)


def time_oracle(w, budget_s, min_tokens=1):
    """FP64 oracle over a bounded sample of the workload's tokens (host copies)."""
    import numpy as np

    import oracle
    q, k, v = w.q.cpu(), w.k_cache.cpu(), w.v_cache.cpu()
    idx = w.topk_idx.cpu()
    nv = w.n_valid.cpu() if w.n_valid is not None else None
    T = q.shape[0]
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    probe = np.sort(rng.choice(T, size=min(T, max(cores, min_tokens)), replace=False))
    t = time.perf_counter()
    oracle.sparse_prefill(q, k, v, idx, nv, w.scale, tokens=probe, n_threads=cores)
    dt = time.perf_counter() - t
    per_tok = dt / len(probe)
    n = int(min(T, max(len(probe), budget_s / max(per_tok, 1e-9))))
    sample = np.sort(rng.choice(T, size=n, replace=False))
    t = time.perf_counter()
    oracle.sparse_prefill(q, k, v, idx, nv, w.scale, tokens=sample, n_threads=cores)
    dt = time.perf_counter() - t
    return dict(value=n / dt, unit=UNIT, cores=cores, kind="oracle",
                sample=f"{n} of {T} query tokens (all heads), uniform without replacement, seed 0; "
                       f"{dt:.1f} s on {cores} threads")


def W_make(name, device, **kw):
    from top_sparse_attention_qsa_b200 import workloads as W
    return W.make(name, device=device, **kw)


def make_workload(name, device):
    from top_sparse_attention_qsa_b200 import workloads as W
    return W.make(name, device=device)


def config_of(w, acct):
    s = w.shape
    return {"workload": w.name, "desc": w.description, "T": s["T"], "S": s["S"],
            "heads": [s["Hq"], s["Hkv"]], "head_dim": s["D"], "topk": s["K"],
            "live_entries": acct["entries"],
            "l2": l2_note(w)}


def l2_note(w):
    mb = (w.q.numel() * 2 * 2 + w.k_cache.numel() * 2 * 2 + w.topk_idx.numel() * 4) / 1e6
    if mb > 126:
        return f"no flush: inputs+outputs exceed L2 (126 MB), {mb:.0f} MB resident per rank"
    return f"no flush: {mb:.0f} MB resident per rank fits in L2 (warm-L2 figure)"


# ---------------------------------------------------------------- arms

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = make_workload(args.workload, dev)
    acct = workload_accounting(w)
    import numpy as np

    import oracle
    q, k, v = w.q.cpu(), w.k_cache.cpu(), w.v_cache.cpu()
    idx = w.topk_idx.cpu()
    nv = w.n_valid.cpu() if w.n_valid is not None else None
    T = q.shape[0]
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(1)
    # calibrate the per-step sample so the whole run stays within ~2 minutes
    probe = np.sort(rng.choice(T, size=min(T, cores), replace=False))
    t = time.perf_counter()
    oracle.sparse_prefill(q, k, v, idx, nv, w.scale, tokens=probe, n_threads=cores)
    per_tok = (time.perf_counter() - t) / len(probe)
    step_budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(min(T, max(len(probe), cores * max(1, int(step_budget / max(per_tok * cores, 1e-9))))))
    times = []
    for i in range(args.warmup + args.steps):
        sample = np.sort(rng.choice(T, size=n, replace=False))
        t = time.perf_counter()
        oracle.sparse_prefill(q, k, v, idx, nv, w.scale, tokens=sample, n_threads=cores)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    total = sum(times)
    value = n * len(times) / total
    sample_desc = f"{n} of {T} query tokens per step (all heads), uniform without replacement"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, acct), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample_desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_cuda(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
        # the path has no exchange step: NCCL carries only the barrier and the
        # max-over-ranks timing reduction
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    def max_ranks(x):
        return max_over_ranks(x, pg, dev)

    from top_sparse_attention_qsa_b200 import _capi
    from top_sparse_attention_qsa_b200 import workloads as W

    if args.only:
        hbm, bf16, _ = measured_peaks()
        kw = {"T": args.tokens} if args.tokens else {}
        leg = {"fp8": lambda: run_fp8_bench("c5", dev, barrier, max_ranks, world, hbm, args.steps,
                                            args.warmup, **kw),
               "indexer": lambda: run_indexer_bench(dev, barrier, max_ranks, world, hbm, bf16, args.steps,
                                                    args.warmup, **kw),
               "blocks": lambda: run_blocks_bench("c5_block4", dev, barrier, max_ranks, world, hbm,
                                                  args.steps, args.warmup, **kw),
               "decode": lambda: run_decode_bench("decode", dev, barrier, max_ranks, world, hbm, args.steps,
                                                  args.warmup),
               "qsa_step": lambda: run_qsa_step_bench(dev, barrier, max_ranks, world, hbm, args.steps,
                                                      args.warmup, **kw),
               "gather_peak": lambda: run_gather_peak(dev)}[args.only]()
        if rank == 0:
            print(json.dumps({"leg": args.only, **leg}), flush=True)
        if pg is not None:
            pg.barrier()
            pg.destroy_process_group()
        return 0

    # weak scaling (default): every rank runs its own replica (own seed);
    # strong scaling (--shard tokens): the ranks split one workload's tokens
    seed_off = 1000 * rank if args.shard == "replicas" else 0
    kw = {"seed": W.CONFIG_SEED_BASE + {"tiny": 1, "c2": 2, "c3": 3, "c4": 4, "c5": 5,
                                        "pages_long": 6}[args.workload] + seed_off}
    if args.tokens and args.workload in ("c4", "c5"):
        kw["T"] = args.tokens
    w = W.make(args.workload, device=dev, **kw)
    T_job = w.shape["T"] * (world if args.shard == "replicas" else 1)
    if args.shard == "tokens":
        w = shard_workload(w, world, rank)
    elif args.shard == "heads":
        w_full, w = w, shard_heads(w, world, rank)
        if w is None:                 # more ranks than KV heads: this rank idles
            w = dataclasses_replace_empty(w_full)
    acct = workload_accounting(w)
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                 out=out, lse=lse, status=status, kernel=args.kernel)

    sampler = None
    if not args.profile:
        sampler = ClockSampler(local)
        sampler.start()
        time.sleep(0.3)
    total_ms, per_ms, (t0, t1) = time_launches(step, args.steps, args.warmup, barrier)
    clocks = sampler.stop(t0, t1) if sampler is not None else None
    total_ms = max_ranks(total_ms)
    T = w.shape["T"]
    value = T_job * args.steps / (total_ms / 1e3)
    mean_launch_ms = statistics.mean(per_ms)
    hbm, bf16, peak_src = measured_peaks()
    achieved = acct["algo_bytes"] / (mean_launch_ms / 1e3) / 1e9
    units = T * w.shape["Hkv"]
    traffic = profiled_traffic(args.workload, units)
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic,
            "peak_source": peak_src + " (hbm_gbs, STREAM-style copy)",
            "kernel": KERNEL_NAMES[args.kernel], "algo_bytes_per_launch": acct["algo_bytes"],
            "mean_launch_ms": mean_launch_ms}
    gathered_gbs = acct["gathered_bytes"] / (mean_launch_ms / 1e3) / 1e9
    tflops = acct["flops"] / (mean_launch_ms / 1e3) / 1e12
    roof_time_ms = 1e3 * max(acct["gathered_bytes"] / (hbm * 1e9), acct["flops"] / (bf16 * 1e12))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak" if args.shard == "replicas" else "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": config_of(w, acct),
            "gpu_launches": args.steps,
            "gathered_kv_gbs": gathered_gbs, "effective_tflops": tflops,
            "roofline_time_ms": roof_time_ms, "frac_of_roofline_time": roof_time_ms / mean_launch_ms,
            "roofline": roof, "clocks": clocks}
    if not args.profile:
        fl_mean, fl_median = time_flushed(step)
        line["timing"] = {"mean_launch_ms": mean_launch_ms, "median_launch_ms": statistics.median(per_ms),
                          "l2_flushed_mean_ms": fl_mean, "l2_flushed_median_ms": fl_median,
                          "compulsory_bytes": compulsory_bytes(w)}
    if int(status.item()) != 0:
        line["status_word"] = int(status.item())

    if args.compare and not args.profile and args.compare != args.kernel:
        def step_cmp():
            _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                     out=out, lse=lse, kernel=args.compare)
        cmp_ms, cmp_per, _ = time_launches(step_cmp, min(args.steps, 20), 3, barrier, "compare")
        cmp_ms = max_ranks(cmp_ms)
        n_cmp = min(args.steps, 20)
        line["compare"] = {"kernel": KERNEL_NAMES[args.compare],
                           "tokens_per_s": T * n_cmp * world / (cmp_ms / 1e3),
                           "mean_launch_ms": statistics.mean(cmp_per),
                           "algo_gbs": acct["algo_bytes"] / (statistics.mean(cmp_per) / 1e3) / 1e9}
    if not args.profile and args.kernel in ("auto", "tcgen05"):
        # the same lists through the kernel's gather step alone (measurement
        # kernel of libqsa_debug.so): the floor of the timed kernel here
        from top_sparse_attention_qsa_b200 import _debug

        def step_gather():
            _debug.gather_only(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid)
        n_g = min(args.steps, 20)
        g_ms, g_per, _ = time_launches(step_gather, n_g, 3, barrier, "gather_only")
        g_mean = statistics.mean(g_per)
        line["gather_floor"] = {"kernel": "qsa_gather_only_kernel", "mean_launch_ms": g_mean,
                                "gathered_kv_gbs": acct["gathered_bytes"] / (g_mean / 1e3) / 1e9,
                                "kernel_frac_of_floor": g_mean / mean_launch_ms, "launches": n_g}
    if args.gather_peak and not args.profile:
        # the roofline's gather ceiling: the chip's random-row gather rate
        peak = run_gather_peak(dev)
        line["gather_peak"] = peak
        l2 = peak["best"]["512B_32MB"]
        ws = peak["best"]["512B_134MB"]
        roof["l2_gather_peak"] = {"gbs": l2["gbs"], "method": l2["method"], "table_mb": 32,
                                  "row_bytes": 512}
        roof["gather_peak_working_set"] = {"gbs": ws["gbs"], "method": ws["method"], "table_mb": 134,
                                           "row_bytes": 512,
                                           "note": "table the size of one KV head's K+V rows of c5"}
        roof["frac_gather"] = gathered_gbs / l2["gbs"]
        roof["frac_gather_working_set"] = gathered_gbs / ws["gbs"]
    if traffic is not None:
        roof["frac_dram"] = traffic / (mean_launch_ms / 1e3) / 1e9 / hbm
    if not args.no_e2e and not args.profile:
        line["e2e"] = run_e2e(w, args, barrier, max_ranks, T_job, dev)
    if args.secondary and not args.profile and args.secondary != args.workload:
        line["secondary"] = run_secondary(args.secondary, dev, barrier, max_ranks, world, hbm,
                                          bf16, args.kernel)
    if args.decode and not args.profile:
        line["decode"] = run_decode_bench(args.decode, dev, barrier, max_ranks, world, hbm)
    if args.blocks and not args.profile:
        line["blocks"] = run_blocks_bench(args.blocks, dev, barrier, max_ranks, world, hbm)
    if args.fp8 and not args.profile:
        line["fp8"] = run_fp8_bench(args.fp8, dev, barrier, max_ranks, world, hbm)
    if args.indexer and not args.profile:
        line["indexer"] = run_indexer_bench(dev, barrier, max_ranks, world, hbm, bf16)
    if args.per_config and not args.profile:
        line["per_config"] = run_per_config(dev, barrier, max_ranks, world, hbm, bf16)
    if args.qsa_step and not args.profile:
        line["qsa_step"] = run_qsa_step_bench(dev, barrier, max_ranks, world, hbm)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        line["cpu_baseline"] = time_oracle(w, args.cpu_budget)
    elif not args.profile:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def run_e2e(w, args, barrier, reduce_max, T_job, dev):
    from top_sparse_attention_qsa_b200 import _capi
    hq = w.q.cpu().pin_memory()
    hk = w.k_cache.cpu().pin_memory()
    hv = w.v_cache.cpu().pin_memory()
    hi = w.topk_idx.cpu().pin_memory()
    hn = w.n_valid.cpu().pin_memory() if w.n_valid is not None else None
    ho = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(w.q.shape[:2], dtype=torch.float32).pin_memory()
    bufs = dict(q=torch.empty_like(w.q), k_cache=torch.empty_like(w.k_cache),
                v_cache=torch.empty_like(w.v_cache), topk_idx=torch.empty_like(w.topk_idx),
                n_valid=torch.empty_like(w.n_valid) if hn is not None else None,
                out=torch.empty_like(w.q), lse=torch.empty(w.q.shape[:2], device=dev),
                status=torch.zeros(1, dtype=torch.int32, device=dev))

    def step():
        _capi.sparse_prefill_fwd_host(hq, hk, hv, hi, hn, w.scale, ho, hl, bufs)

    steps = max(1, args.e2e_steps)
    total_ms, _, _ = time_launches(step, steps, 2, barrier, "e2e")
    total_ms = reduce_max(total_ms)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hi) + ((hn,) if hn is not None else ()))
    d2h = ho.numel() * 2 + hl.numel() * 4
    return {"value": T_job * steps / (total_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": total_ms / steps, "steps": steps,
            "api": "qsa_sparse_prefill_fwd_host (pinned host buffers)"}


# (method, depth, warps per CTA, CTAs per SM) of the gather probe, for 512-
# and 256-byte rows: each fills a shared-memory ring of at most 192 KB per SM
# (cp.async, bulk) or keeps 64-256 KB of loads in flight (ld.v4), with at
# most 1024 threads per SM.
PEAK_CONFIGS = {
    512: [("cp_async", 1, 32, 1), ("cp_async", 2, 16, 1), ("cp_async", 1, 16, 2), ("cp_async", 2, 12, 2),
          ("cp_async", 2, 24, 1), ("cp_async", 4, 12, 1), ("cp_async", 8, 6, 1), ("cp_async", 4, 8, 1),
          ("ld_v4", 4, 32, 1), ("ld_v4", 8, 32, 1), ("ld_v4", 16, 16, 1), ("ld_v4", 16, 16, 2),
          ("bulk", 1, 12, 1), ("bulk", 2, 6, 1), ("bulk", 3, 4, 1)],
    256: [("cp_async", 1, 32, 1), ("cp_async", 1, 16, 2), ("cp_async", 2, 24, 1), ("cp_async", 4, 12, 1),
          ("cp_async", 8, 6, 1),
          ("ld_v4", 8, 32, 1), ("ld_v4", 16, 16, 1), ("ld_v4", 16, 16, 2),
          ("bulk", 2, 12, 1), ("bulk", 3, 8, 1), ("bulk", 4, 6, 1)],
}
PEAK_TABLES_MB = (32, 134, 268)


def run_gather_peak(dev, n_ids=1 << 23, launches=5, warmup=2):
    """Random-row gather rate of this GPU, measured with libqsa_debug.so's
    probe kernels (written independently of the prefill's producer code):
    uniform random rows of 512 B (the BF16 cache row) and 256 B (the FP8
    row) from tables of 32 MB (L2-resident), 134 MB (one KV head's K+V rows
    of c5) and 268 MB (both heads), by each method and depth.  Reports every
    configuration's GB/s (row bytes only; the 4-byte ids add 1-2 %) and the
    best per (row size, table)."""
    from top_sparse_attention_qsa_b200 import _debug
    gen = torch.Generator(device=dev).manual_seed(31)
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    sink = torch.zeros(nsm * 2 * 1024, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    res = {"n_ids": n_ids, "launches": launches, "configs": [], "best": {}}
    for mb in PEAK_TABLES_MB:
        table = torch.empty((mb << 20) // 512, 512, dtype=torch.uint8, device=dev)
        table.random_(0, 255, generator=gen)
        for row_bytes in (512, 256):
            view = table.view(-1, row_bytes)
            ids = torch.randint(0, view.shape[0], (n_ids,), generator=gen, device=dev, dtype=torch.int32)
            best = None
            for method, depth, warps, cps in PEAK_CONFIGS[row_bytes]:
                def fn():
                    _debug.gather_peak(view, ids, row_bytes, method, depth, warps, cps, sink=sink, status=status)
                try:
                    for _ in range(warmup):
                        fn()
                except _debug.QSAError as e:
                    res["configs"].append({"table_mb": mb, "row_bytes": row_bytes, "method": method, "depth": depth,
                                           "warps": warps, "ctas_per_sm": cps, "error": str(e)})
                    continue
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                a.record()
                for _ in range(launches):
                    fn()
                b.record()
                torch.cuda.synchronize()
                ms = a.elapsed_time(b) / launches
                gbs = n_ids * row_bytes / (ms / 1e3) / 1e9
                entry = {"table_mb": mb, "row_bytes": row_bytes, "method": method, "depth": depth,
                         "warps": warps, "ctas_per_sm": cps, "ms": ms, "gbs": gbs}
                res["configs"].append(entry)
                if best is None or gbs > best["gbs"]:
                    best = entry
            res["best"][f"{row_bytes}B_{mb}MB"] = best
            del ids
        del table
    res["status_word"] = int(status.item())
    return res


def run_secondary(name, dev, barrier, reduce_max, world, hbm, bf16, kernel="auto"):
    from top_sparse_attention_qsa_b200 import _capi
    w = make_workload(name, dev)
    acct = workload_accounting(w)
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=dev)

    def step():
        _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                 out=out, lse=lse, kernel=kernel)

    steps = 20
    total_ms, per_ms, _ = time_launches(step, steps, 3, barrier, "secondary")
    total_ms = reduce_max(total_ms)
    ms = statistics.mean(per_ms)
    roof_ms = 1e3 * max(acct["gathered_bytes"] / (hbm * 1e9), acct["flops"] / (bf16 * 1e12))
    return {"workload": w.name, "tokens_per_s": w.shape["T"] * steps * world / (total_ms / 1e3),
            "mean_launch_ms": ms, "gathered_kv_gbs": acct["gathered_bytes"] / (ms / 1e3) / 1e9,
            "effective_tflops": acct["flops"] / (ms / 1e3) / 1e12,
            "algo_gbs": acct["algo_bytes"] / (ms / 1e3) / 1e9,
            "frac_of_roofline_time": roof_ms / ms, "steps": steps}


def run_decode_bench(name, dev, barrier, reduce_max, world, hbm, steps=50, warmup=5):
    """Split-K decode (one query token per sequence): two launches per step
    (chunk kernel + merge), workspace allocated once outside the timed loop."""
    from top_sparse_attention_qsa_b200 import _capi
    w = make_workload(name, dev)
    acct = workload_accounting(w)
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=dev)
    splits = _capi.decode_num_splits(w.q, w.k_cache, w.topk_idx, 0)
    need = _capi.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, 0, out, lse)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)

    def step():
        _capi.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                num_splits=0, workspace=ws, out=out, lse=lse)

    total_ms, per_ms, _ = time_launches(step, steps, warmup, barrier, "decode")
    total_ms = reduce_max(total_ms)
    ms = statistics.mean(per_ms)
    algo = acct["algo_bytes"] + need  # partial results are written once and read once by the merge
    # the same decode over an FP8 E4M3 cache (k_scale 0.5, v_scale 2)
    from top_sparse_attention_qsa_b200 import workloads as W
    gen = torch.Generator(device=dev).manual_seed(78)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, dev)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, dev)

    def step8():
        _capi.sparse_decode_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid, scale=w.scale,
                                    num_splits=0, workspace=ws, out=out, lse=lse)

    _, per8, _ = time_launches(step8, steps, warmup, barrier, "decode_fp8")
    ms8 = statistics.mean(per8)
    algo8 = acct["algo_bytes"] - acct["gathered_bytes"] // 2 + need
    del k8, v8
    small = run_decode_small_batch(dev)
    return {"workload": w.name, "desc": w.description, "splits": splits,
            "workspace_bytes": need, "tokens_per_s": w.shape["T"] * steps * world / (total_ms / 1e3),
            "mean_step_ms": ms, "gathered_kv_gbs": acct["gathered_bytes"] / (ms / 1e3) / 1e9,
            "algo_gbs": algo / (ms / 1e3) / 1e9, "frac_of_hbm": algo / (ms / 1e3) / 1e9 / hbm,
            "launches_per_step": 2 if need > 0 else 1, "steps": steps,
            "fp8": {"mean_step_ms": ms8, "tokens_per_s": w.shape["T"] * world / (ms8 / 1e3),
                    "algo_gbs": algo8 / (ms8 / 1e3) / 1e9, "frac_of_hbm": algo8 / (ms8 / 1e3) / 1e9 / hbm},
            "small_batch": small}


def graph_call_us(fn, calls=20, replays=5):
    """Device time of one call, from CUDA-graph replays of `calls` calls (a
    call of a few microseconds is otherwise timed together with the host's
    launch overhead)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) * 1e3 / (calls * replays)


def run_decode_small_batch(dev, B=16):
    """Decode with few (token, KV head) units: 16 sequences x 32 K context,
    heads (24,2), K = 2048 (32 units on the SMs).  The automatic chunk count
    against a single chunk, BF16 and FP8 caches, CUDA-graph timed."""
    from top_sparse_attention_qsa_b200 import _capi
    from top_sparse_attention_qsa_b200 import workloads as W
    w = W.config_decode(device=dev, B=B)
    gen = torch.Generator(device=dev).manual_seed(79)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, dev)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, dev)
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=dev)
    auto = _capi.decode_num_splits(w.q, w.k_cache, w.topk_idx, 0)
    res = {"workload": w.name, "units": w.shape["T"] * w.shape["Hkv"], "auto_splits": auto}
    for splits, key in ((0, "auto"), (1, "one_chunk")):
        need = _capi.decode_workspace_bytes(w.q, w.k_cache, w.topk_idx, splits, out, lse)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        res[key + "_us"] = graph_call_us(
            lambda: _capi.sparse_decode_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale,
                                            num_splits=splits, workspace=ws, out=out, lse=lse))
        res[key + "_fp8_us"] = graph_call_us(
            lambda: _capi.sparse_decode_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid,
                                                scale=w.scale, num_splits=splits, workspace=ws, out=out,
                                                lse=lse))
    return res


def run_blocks_bench(name, dev, barrier, reduce_max, world, hbm, steps=20, warmup=3, **kw):
    """Microblock lists on the c5 shape: the same 2048 keys per (token, KV
    head) as c5, named by 512 blocks of 4 slots."""
    from top_sparse_attention_qsa_b200 import _capi
    w = W_make(name, dev, **kw)
    out = torch.empty_like(w.q)
    lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=dev)
    bs = w.block_size
    # live keys: expand each live entry to its visible slots
    idx = w.topk_idx.to(torch.int64)
    E = idx.shape[2]
    live_e = (idx >= 0) & (torch.arange(E, device=dev)[None, None, :] < w.n_valid[:, :, None])
    slots = idx[..., None] * bs + torch.arange(bs, device=dev)
    vis = live_e[..., None] & (slots < w.shape["S"]) & (slots <= w.last_slot.to(torch.int64)[:, None, None, None])
    keys = int(vis.sum().item())
    s = w.shape
    algo = keys * 1024 + int(live_e.sum().item()) * 4 + s["T"] * s["Hq"] * s["D"] * 4 + s["T"] * s["Hq"] * 4

    def step():
        _capi.sparse_prefill_block_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, bs, w.last_slot,
                                       w.n_valid, w.scale, out=out, lse=lse)

    total_ms, per_ms, _ = time_launches(step, steps, warmup, barrier, "blocks")
    total_ms = reduce_max(total_ms)
    ms = statistics.mean(per_ms)
    return {"workload": w.name, "desc": w.description, "tokens_per_s": s["T"] * steps * world / (total_ms / 1e3),
            "mean_launch_ms": ms, "live_keys": keys, "gathered_kv_gbs": keys * 1024 / (ms / 1e3) / 1e9,
            "algo_gbs": algo / (ms / 1e3) / 1e9, "frac_of_hbm": algo / (ms / 1e3) / 1e9 / hbm,
            "steps": steps}


def run_fp8_bench(name, dev, barrier, reduce_max, world, hbm, steps=20, warmup=3, **kw):
    """The same lists and Q as `name`, with the K and V caches stored as FP8
    E4M3 (k_scale 0.5, v_scale 2): half the gathered bytes per key."""
    from top_sparse_attention_qsa_b200 import _capi
    from top_sparse_attention_qsa_b200 import workloads as W
    w = W_make(name, dev, **kw)
    entries = workload_accounting(w)["entries"]
    gen = torch.Generator(device=dev).manual_seed(77)
    k8 = W.normal_fp8(tuple(w.k_cache.shape), gen, dev)
    v8 = W.normal_fp8(tuple(w.v_cache.shape), gen, dev)
    w.k_cache = w.v_cache = None                   # free the BF16 caches
    T, Hq, D = w.q.shape
    out = torch.empty_like(w.q)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    gathered = entries * 2 * D
    algo = gathered + entries * 4 + T * Hq * D * 2 * 2 + T * Hq * 4

    def step():
        _capi.sparse_prefill_fp8_fwd(w.q, k8, v8, w.topk_idx, 0.5, 2.0, n_valid=w.n_valid, scale=w.scale,
                                     out=out, lse=lse)

    total_ms, per_ms, _ = time_launches(step, steps, warmup, barrier, "fp8")
    total_ms = reduce_max(total_ms)
    ms = statistics.mean(per_ms)

    from top_sparse_attention_qsa_b200 import _debug

    def step_gather():
        _debug.gather_only(w.q, k8, v8, w.topk_idx, w.n_valid)

    _, g_per, _ = time_launches(step_gather, steps, warmup, barrier, "fp8_gather_only")
    g_ms = statistics.mean(g_per)
    return {"workload": w.name + "_fp8e4m3", "tokens_per_s": T * steps * world / (total_ms / 1e3),
            "mean_launch_ms": ms, "live_entries": entries, "algo_bytes": algo,
            "gathered_kv_gbs": gathered / (ms / 1e3) / 1e9,
            "algo_gbs": algo / (ms / 1e3) / 1e9, "frac_of_hbm": algo / (ms / 1e3) / 1e9 / hbm,
            "steps": steps,
            "gather_floor": {"kernel": "qsa_gather_only_f8_kernel", "mean_launch_ms": g_ms,
                             "gathered_kv_gbs": gathered / (g_ms / 1e3) / 1e9,
                             "kernel_frac_of_floor": g_ms / ms}}


def run_indexer_bench(dev, barrier, reduce_max, world, hbm, bf16, steps=20, warmup=3, **kw):
    """Indexer scores (tcgen05) then top-K selection on the c5 size: 8192
    tokens, 32768 block keys, 4 heads x 128, budget 2048 + causal tail.  Each
    kernel is timed on its own (events on the launching stream) and as the
    pair; the scores buffer (1 GiB) is larger than L2."""
    from top_sparse_attention_qsa_b200 import _capi
    from top_sparse_attention_qsa_b200 import workloads as W
    w = W.config_indexer(device=dev, **kw)
    T, H, Dh = w.q_idx.shape
    NB = w.k_idx.shape[0]
    pos = w.positions.to(torch.int64)
    n = ((pos + 1) // w.block_size).clamp(max=NB) - w.seq_start.to(torch.int64) // w.block_size
    cand = int(n.clamp(min=0).sum().item())
    width = w.budget + 1
    scores = torch.empty((T, NB), dtype=torch.float32, device=dev)
    lists = torch.empty((T, width), dtype=torch.int32, device=dev)
    nv = torch.empty((T, 2), dtype=torch.int32, device=dev)
    q2 = torch.empty((T, 2, Dh), dtype=torch.bfloat16, device=dev)

    def s_step():
        # head folding (one small launch) then the score kernel on the folded query
        _capi.indexer_scores(w.q_idx, w.k_idx, w.positions, w.seq_start, w.block_size, scores=scores,
                             q_folded=q2)

    def k_step():
        _capi.topk_select(scores, w.positions, w.seq_start, NB, w.budget, w.block_size, True,
                          lists=lists, n_valid=nv, copies=2)

    def pair():
        s_step()
        k_step()

    _, s_per, _ = time_launches(s_step, steps, warmup, barrier, "indexer_scores")
    _, k_per, _ = time_launches(k_step, steps, warmup, barrier, "topk_select")
    total_ms, p_per, _ = time_launches(pair, steps, warmup, barrier, "indexer_pair")
    total_ms = reduce_max(total_ms)
    s_ms, k_ms = statistics.mean(s_per), statistics.mean(k_per)
    flops = cand * H * Dh * 2
    s_bytes = w.q_idx.numel() * 2 + w.k_idx.numel() * 2 + cand * 4
    k_bytes = cand * 4 + T * width * 4 + T * 2 * 4 + T * 8
    s_roof = 1e3 * max(flops / (bf16 * 1e12), s_bytes / (hbm * 1e9))
    return {"workload": w.name, "desc": w.description, "candidates": cand,
            "tokens_per_s": T * steps * world / (total_ms / 1e3), "mean_pair_ms": statistics.mean(p_per),
            "scores": {"mean_launch_ms": s_ms, "launches": 2, "tflops": flops / (s_ms / 1e3) / 1e12,
                       "algo_gbs": s_bytes / (s_ms / 1e3) / 1e9, "roofline_ms": s_roof,
                       "frac_of_roofline_time": s_roof / s_ms,
                       "bound": "tensor" if flops / (bf16 * 1e12) > s_bytes / (hbm * 1e9) else "hbm"},
            "topk": {"mean_launch_ms": k_ms, "algo_gbs": k_bytes / (k_ms / 1e3) / 1e9,
                     "frac_of_hbm": k_bytes / (k_ms / 1e3) / 1e9 / hbm},
            "launches_per_step": 3, "steps": steps}


def run_per_config(dev, barrier, reduce_max, world, hbm, bf16, steps=20, warmup=3):
    """Every config of the workload table with the default kernel: query
    tokens/s, gathered-KV GB/s, effective TFLOP/s and the fraction of the
    roofline time (gathered bytes at the HBM peak vs FLOPs at the BF16
    peak, the slower of the two)."""
    from top_sparse_attention_qsa_b200 import _capi
    res = {}
    for name in ("tiny", "c2", "c3", "c4", "c5"):
        w = make_workload(name, dev)
        acct = workload_accounting(w)
        out = torch.empty_like(w.q)
        lse = torch.empty(w.q.shape[:2], dtype=torch.float32, device=dev)

        def step():
            _capi.sparse_prefill_fwd(w.q, w.k_cache, w.v_cache, w.topk_idx, w.n_valid, w.scale, out=out, lse=lse)

        total_ms, per_ms, _ = time_launches(step, steps, warmup, barrier, "config_" + name)
        total_ms = reduce_max(total_ms)
        ms = statistics.mean(per_ms)
        roof_ms = 1e3 * max(acct["gathered_bytes"] / (hbm * 1e9), acct["flops"] / (bf16 * 1e12))
        s = w.shape
        res[name] = {"workload": w.name, "T": s["T"], "S": s["S"], "heads": [s["Hq"], s["Hkv"]], "topk": s["K"],
                     "mean_launch_ms": ms, "tokens_per_s": s["T"] * steps * world / (total_ms / 1e3),
                     "gathered_kv_gbs": acct["gathered_bytes"] / (ms / 1e3) / 1e9,
                     "effective_tflops": acct["flops"] / (ms / 1e3) / 1e12,
                     "frac_of_roofline_time": roof_ms / ms}
        del w, out, lse
    return res


def run_qsa_step_bench(dev, barrier, reduce_max, world, hbm, steps=5, warmup=3, T=8192, S=131072,
                       heads=(24, 2)):
    """One whole QSA sparse-attention step on the c5 shape: indexer scores and
    top-K select 2048 microblocks of 4 (+ the causal tail) per query token,
    and the attention reads those 8196 keys per (token, KV head), both KV
    heads sharing the token's list.  Timed with a BF16 and with an FP8 E4M3
    KV cache; three launches per step."""
    from top_sparse_attention_qsa_b200 import _capi
    from top_sparse_attention_qsa_b200 import workloads as W
    wi = W.config_indexer(device=dev, T=T, S=S)
    gen = torch.Generator(device=dev).manual_seed(79)
    Hq, Hkv = heads
    q = W.normal_bf16((T, Hq, 256), gen, dev)
    k = W.normal_bf16((S, Hkv, 256), gen, dev)
    v = W.normal_bf16((S, Hkv, 256), gen, dev)
    k8 = W.normal_fp8((S, Hkv, 256), gen, dev)
    v8 = W.normal_fp8((S, Hkv, 256), gen, dev)
    NB = wi.k_idx.shape[0]
    width = wi.budget + 1
    scores = torch.empty((T, NB), dtype=torch.float32, device=dev)
    lists = torch.empty((T, width), dtype=torch.int32, device=dev)
    nv = torch.empty((T, Hkv), dtype=torch.int32, device=dev)
    idx = lists[:, None, :].expand(T, Hkv, width)
    out = torch.empty_like(q)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    q2 = torch.empty((T, 2, wi.q_idx.shape[2]), dtype=torch.bfloat16, device=dev)

    def select():
        _capi.indexer_scores(wi.q_idx, wi.k_idx, wi.positions, wi.seq_start, 4, scores=scores, q_folded=q2)
        _capi.topk_select(scores, wi.positions, wi.seq_start, NB, wi.budget, 4, True, lists=lists, n_valid=nv,
                          copies=Hkv)

    def step_bf16():
        select()
        _capi.sparse_prefill_block_fwd(q, k, v, idx, 4, wi.positions, nv, 0.0, out=out, lse=lse)

    def step_fp8():
        select()
        _capi.sparse_prefill_fp8_fwd(q, k8, v8, idx, 0.5, 2.0, n_valid=nv, block_size=4, last_slot=wi.positions,
                                     out=out, lse=lse)

    res = {"workload": f"qsa_step_T{T}_S{S}_g{Hq}x{Hkv}_budget{wi.budget}x4",
           "desc": f"indexer ({wi.q_idx.shape[1]}x128, {NB} block keys) + top-{wi.budget} blocks of 4 + tail, "
                   f"then attention over <= {4 * width} keys per (token, KV head)", "launches_per_step": 4}
    for name, fn in (("bf16", step_bf16), ("fp8", step_fp8)):
        total_ms, per_ms, _ = time_launches(fn, steps, warmup, barrier, "qsa_step_" + name)
        total_ms = reduce_max(total_ms)
        res[name] = {"mean_step_ms": statistics.mean(per_ms), "tokens_per_s": T * steps * world / (total_ms / 1e3)}
    res["keys_per_token_head"] = float(nv.float().mean().item()) * 4
    res["steps"] = steps
    return res


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
