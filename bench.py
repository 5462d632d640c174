#!/usr/bin/env python
"""Decode-attention benchmark on B200: microseconds per decode step and achieved HBM
bandwidth, for GQA decode attention over a paged KV cache with split-KV scheduling.

A step is one pass of the whole path on one batch: the planner kernel, the split kernel
and the combine kernel (plan + split + combine). Inputs are seeded synthetic data of the
named workload (``--config``, default "mixed": batch 64, 32 query / 8 KV heads, head_dim 128,
KV lengths log-uniform in [128, 65536], 1% of K rows x8, page size 16, bf16; the largest
single-GPU workload), resident in HBM before timing.

Timing: W untimed warm-up steps, then K timed steps (events at step boundaries only, so the
three kernels keep their programmatic-dependent-launch overlap), then the same K steps again
with events between the kernels for the per-kernel breakdown used by the roofline. Before each step the L2 is flushed
by reading a 256 MiB buffer (a read leaves no dirty lines for the timed kernels to write
back; the KV of every full-size workload is larger than the 126 MB L2 as well) and the GPU is kept busy for a moment so that every launch of the step is queued
before the step starts; CUDA events on the launching stream bracket the planner, the
split kernel and the combine kernel of every step. ``value`` is the mean step time
(max over ranks when run under torchrun: the path does not shard, so each rank runs a
full replica). One JSON line is printed by rank 0.

``--config prefill`` times the causal prefill kernel instead (4 prompts of 2048 tokens; one
kernel per step, reported against the measured bf16 tensor peak).

``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample of the same
workload (rows chosen at random, time scaled to the whole step).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "decode-attention µs/step and achieved HBM GB/s as % of B200 peak, 1 GPU"
PREFILL_METRIC = "prefill-attention µs/step and achieved bf16 TFLOP/s as a fraction of B200 peak, 1 GPU"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FLUSH_BYTES = 256 << 20
SLEEP_CYCLES = 1_000_000  # ~0.5 ms of GPU spin before each step: longer than the host needs to queue it


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="mixed", choices=sorted(W.CONFIGS))
    ap.add_argument("--tile-len", type=int, default=0, help="override the workload's tile length")
    ap.add_argument("--batch", type=int, default=0,
                    help="keep only the first BATCH requests of the workload (smaller profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay figure")
    ap.add_argument("--profile", action="store_true",
                    help="only warm-up + timed steps (for ncu launch lists): no baseline, e2e, graph or clocks")
    ap.add_argument("--json-out", default="", help="also append the JSON line to this file")
    ap.add_argument("--write-traffic", action="store_true",
                    help="write the DRAM-traffic JSON files under profiles/ from the capture tables and exit")
    ap.add_argument("--sparse", type=float, default=0.0,
                    help="block-sparse decode: keep each (request, KV head, tile) with this probability "
                         "(the tile with each request's newest token always kept); 0 = dense")
    ap.add_argument("--mma8", action="store_true",
                    help="FP8 workloads: both products on E4M3 tensor cores (q and P rounded to E4M3; "
                         "its own tolerance)")
    ap.add_argument("--bins", type=int, default=0,
                    help="bins of the plan (0: the library's default, SM count x 4)")
    ap.add_argument("--fp8-kv", action="store_true",
                    help="--config prefill: an E4M3 KV cache with per-(page, KV head) scales "
                         "(dec_attn_prefill_fp8: a widening pass, then the bf16 prefill kernel)")
    ap.add_argument("--append", action="store_true",
                    help="each step starts with the fused pre-processing kernel (rotary embedding of the "
                         "step's new q / k rows and their KV append), and the decode reads the rotated q")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers

def max_over_ranks(vals, dist, device):
    """Element-wise maximum of a list of floats over all ranks (the list itself without a process
    group). Every rank must call it at the same point: it is one collective."""
    if dist is None:
        return [float(x) for x in vals]
    import torch
    t = torch.tensor([float(x) for x in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("split.cu", "split_tc.cu", "walk.cuh", "tc.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "paged_kv_decode_29_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def split_kernel_name(pr) -> str:
    """The split kernel the library runs for this workload: FP8 KV with head_dim 128 and
    G*T <= 16 runs on the tcgen05 kernel, everything else on the warp-MMA kernel."""
    if pr.kv_dtype == "fp8e4m3" and pr.head_dim == 128 and pr.group * pr.q_tokens <= 16:
        return "split_tc_kernel"
    return "split_kernel"


# ---------------------------------------------------------------- DRAM traffic captures
# DRAM bytes (dram__bytes_read.sum, dram__bytes_write.sum) of one launch, from the ncu captures that
# profiles/split_kernel_dram_traffic.md and profiles/prefill_kernel_prefill_b4.md describe.
# `python bench.py --write-traffic` turns them into the JSON files that roofline.traffic reads.
# Split kernels: a smaller case of each workload (its first requests), scaled to a full launch by
# the ratio of algorithmic bytes (reads measured within 0.05% of the algorithmic bytes on every
# captured case, so traffic grows in proportion): workload -> (requests captured, read, write).
SPLIT_TRAFFIC_CAPTURED = {
    "source_hash": "fa4bf76c34d9ec92",  # kernel_source_hash() of the sources these were captured on
    "configs": {
        "uniform": (8, 134365184, 3114752),
        "mixed": (16, 1039181824, 17484288),
        "fp8_spec": (4, 167784448, 4281856),
        "long_b4": (1, 536983040, 6753536),
        "long_b1": (1, 536993792, 16440320),
    },
}
# prefill_kernel on the full prefill workload (read, write): a few hundred MB on the device.
PREFILL_TRAFFIC_CAPTURED = {"source_hash": "3447e365c41c00d8", "read": 109325568, "write": 85145600}


def config_algorithmic_bytes(name: str, batch: int | None = None) -> int:
    """Problem.algorithmic_bytes() of a workload (or its first `batch` requests) without generating
    its data."""
    c = W.CONFIGS[name]
    L = np.asarray(W.config_seq_lens(name), dtype=np.int64)
    if batch is not None:
        L = L[:batch]
    B, d, P, hkv, hq, T = len(L), c["head_dim"], c["page_size"], c["n_kv_heads"], c["n_q_heads"], c["q_tokens"]
    eb = 1 if c["kv_dtype"] == "fp8e4m3" else 2
    pages = int(((L + P - 1) // P).sum())
    return (int(L.sum()) * hkv * d * eb * 2 + B * T * hq * d * 2 + B * T * hq * (d + 1) * 4 + pages * 4 + B * 4
            + (pages * hkv * 2 * 4 if c["kv_dtype"] == "fp8e4m3" else 0))


def prefill_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("prefill.cu", "tc.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "paged_kv_decode_29_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def write_traffic_json():
    """Writes profiles/split_kernel_dram_traffic.json and profiles/prefill_kernel_dram_traffic.json
    from the capture tables above. Each table records the source hash it was captured on; a table
    whose hash is not the current sources' is not written (its figures would describe other code)."""
    wrote = []
    if SPLIT_TRAFFIC_CAPTURED["source_hash"] == kernel_source_hash():
        out = {"source_hash": SPLIT_TRAFFIC_CAPTURED["source_hash"], "configs": {}}
        for name, (nb, rd, wr) in SPLIT_TRAFFIC_CAPTURED["configs"].items():
            small, full = config_algorithmic_bytes(name, nb), config_algorithmic_bytes(name)
            scale = full / small
            out["configs"][f"{name}/tl{W.CONFIGS[name]['tile_len']}"] = {
                "bytes_per_launch": int(round((rd + wr) * scale)),
                "captured_requests": nb, "captured_read": rd, "captured_write": wr,
                "captured_algorithmic": small, "scale": round(scale, 6),
                "read_over_algorithmic": round(rd / small, 5),
            }
        with open(os.path.join(ROOT, "profiles", "split_kernel_dram_traffic.json"), "w") as f:
            json.dump(out, f, indent=1)
        wrote.append("split")
    else:
        log("split-kernel traffic table was captured on other sources: not written")
    if PREFILL_TRAFFIC_CAPTURED["source_hash"] == prefill_source_hash():
        rd, wr = PREFILL_TRAFFIC_CAPTURED["read"], PREFILL_TRAFFIC_CAPTURED["write"]
        pf = {"source_hash": PREFILL_TRAFFIC_CAPTURED["source_hash"],
              "configs": {"prefill": {"bytes_per_launch": rd + wr, "captured_read": rd, "captured_write": wr}}}
        with open(os.path.join(ROOT, "profiles", "prefill_kernel_dram_traffic.json"), "w") as f:
            json.dump(pf, f, indent=1)
        wrote.append("prefill")
    else:
        log("prefill-kernel traffic table was captured on other sources: not written")
    return wrote


def ncu_traffic(config: str, tile_len: int):
    """DRAM bytes per split-kernel launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "split_kernel_dram_traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None
    if d.get("source_hash") != kernel_source_hash():
        return None
    e = d.get("configs", {}).get(f"{config}/tl{tile_len}")
    return None if e is None else float(e["bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = None
        self.err = ""

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd.insert(1, f"--id={self.gpu_id}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except Exception as e:
            self.proc = None
            self.err = str(e)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, self.err = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "error": self.err[-200:]}
        rows = [r for r in csv.reader(io.StringIO(self.out)) if len(r) >= 9]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- oracle timing (CPU)

def oracle_timing(pr, budget_s: float, seed: int = 0):
    """Times the fp64 oracle on a random sample of query rows sized to ~budget_s, and scales the
    time to the whole step by the rows' key counts. Returns (us_per_step, threads, sample text)."""
    import oracle
    B, T, Hq = pr.batch, pr.q_tokens, pr.n_q_heads
    rows = np.array([(b, t, qh) for b in range(B) for t in range(T) for qh in range(Hq)], dtype=np.int32)
    keys = np.maximum(pr.seq_lens[rows[:, 0]].astype(np.int64) - T + 1 + rows[:, 1], 0)
    total_keys = int(keys.sum())
    rng = np.random.default_rng(seed)
    order = rng.permutation(len(rows))
    threads = oracle.max_threads()
    # calibration on a few rows, then a sample sized to the budget
    n0 = min(len(rows), max(threads, 8))
    t0 = time.perf_counter()
    oracle.decode_rows(pr, rows[order[:n0]], nthreads=threads)
    dt0 = max(time.perf_counter() - t0, 1e-4)
    per_key = dt0 / max(int(keys[order[:n0]].sum()), 1)
    want_keys = budget_s / per_key
    csum = np.cumsum(keys[order])
    n = int(np.searchsorted(csum, want_keys)) + 1
    n = max(min(n, len(rows)), 1)
    sel = order[:n]
    t0 = time.perf_counter()
    oracle.decode_rows(pr, rows[sel], nthreads=threads)
    dt = time.perf_counter() - t0
    frac = int(keys[sel].sum()) / max(total_keys, 1)
    us = dt / max(frac, 1e-12) * 1e6
    sample = (f"{n} of {len(rows)} query rows ({100 * frac:.1f}% of the row x key work) of the {pr.name} "
              f"workload, fp64 oracle, time scaled by key count")
    return us, threads, sample


# ---------------------------------------------------------------- reference arm

def make_workload(args):
    kw = dict(W.CONFIGS[args.config])
    if args.tile_len:
        kw["tile_len"] = args.tile_len
    if getattr(args, "fp8_kv", False):
        kw["kv_dtype"] = "fp8e4m3"
    lens = W.config_seq_lens(args.config)
    name = args.config
    if args.batch:
        lens = lens[: args.batch]
        kw["batch"] = len(lens)
        name = f"{args.config}[:{len(lens)}]"
        if "pool_pages" in kw:
            del kw["pool_pages"]
    return W.make_problem(name=name, seq_lens=lens, **kw)


def run_reference(args, rank: int):
    if rank != 0:
        return 0
    pr = make_workload(args)
    import oracle
    oracle.build()
    budget = max(0.5, 90.0 / max(args.steps + args.warmup, 1))
    vals = []
    for i in range(args.warmup + args.steps):
        us, threads, sample = oracle_timing(pr, budget, seed=i)
        if i >= args.warmup:
            vals.append(us)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": PREFILL_METRIC if args.config == "prefill" else METRIC, "value": round(value, 3), "unit": "us/step",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(value / 1e3, 6),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(pr, args.gpus, prefill=args.config == "prefill"),
        "cpu_baseline": {"value": round(value, 3), "unit": "us/step", "cores": threads, "kind": "oracle",
                         "sample": f"each step: {sample}"},
        "e2e": {"value": round(value, 3), "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line, args)
    return 0


# ---------------------------------------------------------------- our arm

def bench_config(pr, world: int, prefill: bool = False):
    """The `config` object of the JSON line, identical on both arms: the workload, its shapes, how
    the L2 is kept from serving the inputs, and the multi-GPU layout."""
    l2 = ("flushed before every step (a reduction reading 256 MiB)" if prefill else
          "flushed before every step (a reduction reading 256 MiB); KV bytes exceed the 126 MB L2")
    return {"workload": pr.name, **workload_desc(pr), "l2": l2,
            "parallelism": "replicas" if world > 1 else "single GPU"}


def workload_desc(pr):
    return {"batch": pr.batch, "n_q_heads": pr.n_q_heads, "n_kv_heads": pr.n_kv_heads, "head_dim": pr.head_dim,
            "q_tokens": pr.q_tokens, "page_size": pr.page_size, "kv_dtype": pr.kv_dtype, "tile_len": pr.tile_len,
            "total_kv_tokens": int(pr.seq_lens.astype(np.int64).sum()),
            "kv_bytes": int(pr.seq_lens.astype(np.int64).sum()) * pr.n_kv_heads * pr.head_dim * 2
            * pr.kv_elem_bytes()}


def emit(line, args):
    s = json.dumps(line)
    print(s, flush=True)
    if args.json_out:
        with open(args.json_out, "a") as f:
            f.write(s + "\n")


def run_ours(args, rank: int, world: int, local_rank: int, dist):
    import torch

    import paged_kv_decode_29_b200 as da
    from paged_kv_decode_29_b200 import build as dbuild

    if not os.path.exists(da.LIB_PATH):
        dbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pr = make_workload(args)
    log(f"[rank {rank}] workload {pr.name}: B={pr.batch} Hq={pr.n_q_heads} Hkv={pr.n_kv_heads} d={pr.head_dim} "
        f"T={pr.q_tokens} P={pr.page_size} kv={pr.kv_dtype} tl={pr.tile_len} tokens={int(pr.seq_lens.sum())}")

    def to_dev(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return t.to(dev) if dt is None else t.view(dt).to(dev)

    q = torch.from_numpy(pr.q.view(np.int16)).view(torch.bfloat16).to(dev)
    if pr.kv_dtype == "bf16":
        k = torch.from_numpy(pr.k_pages.view(np.int16)).view(torch.bfloat16).to(dev)
        v = torch.from_numpy(pr.v_pages.view(np.int16)).view(torch.bfloat16).to(dev)
        sc = None
    else:
        k, v, sc = to_dev(pr.k_pages), to_dev(pr.v_pages), to_dev(pr.kv_scales)
    tab, lens = to_dev(pr.page_table), to_dev(pr.seq_lens)
    total = int(pr.seq_lens.astype(np.int64).sum())
    stream = torch.cuda.current_stream()
    mask_dev = None
    if args.sparse > 0:
        pr.tile_mask = W.make_tile_mask(pr, args.sparse)
        mask_dev = torch.from_numpy(pr.tile_mask.view(np.int32)).to(dev)

    def make_plan(buf=None, stream=None):
        if mask_dev is not None:
            return da.plan_sparse(lens, mask_dev, pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total, buf=buf,
                                  stream=stream, n_bins=args.bins)
        return da.plan(lens, pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total, buf=buf, stream=stream,
                       n_bins=args.bins)

    pl = make_plan()
    shape = da.make_shape(q, k, tab, da.kv_dtype_of(k), pr.sm_scale)
    ws = torch.empty(da.workspace_bytes(shape, pl), dtype=torch.uint8, device=dev)
    out = torch.empty((pr.batch, pr.q_tokens, pr.n_q_heads, pr.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((pr.batch, pr.q_tokens, pr.n_q_heads), dtype=torch.float32, device=dev)
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # one reduction kernel reading 256 MiB (same dtype in and out, so no conversion copy):
        # evicts the KV and leaves only clean lines in L2
        torch.sum(flush, dim=0, out=flush_sink)
    pbuf = pl.buf
    kw = dict(kv_scales=sc, sm_scale=pr.sm_scale, workspace=ws, out=out, lse=lse, mma8=args.mma8)
    q_dec = q
    if args.append:
        # the step's new rows; every step rewrites the same slots with the same values
        if pr.kv_dtype != "bf16":
            raise SystemExit("--append needs a bf16 KV cache")
        qn_h, kn_h, vn_h = W.make_step_inputs(pr)
        q_new, k_new, v_new = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
                               for a in (qn_h, kn_h, vn_h))
        q_dec = torch.empty_like(q_new)
    n_kernels = 4 if args.append else 3

    def enqueue_step(evs):
        """[append +] plan + split + combine; evs: 2 events (step boundaries) or one per kernel
        boundary (which stops the kernels' programmatic overlap -- used for the per-kernel
        breakdown)."""
        brk = len(evs) > 2
        i = 0
        evs[i].record(stream)
        if args.append:
            da.append_rope(q_new, k_new, v_new, tab, lens, k, v, q_out=q_dec)
            if brk:
                i += 1
                evs[i].record(stream)
        make_plan(buf=pbuf)
        if brk:
            i += 1
            evs[i].record(stream)
        da.run(q_dec, k, v, tab, lens, pl, stage="split", **kw)
        if brk:
            i += 1
            evs[i].record(stream)
        da.run(q_dec, k, v, tab, lens, pl, stage="combine", **kw)
        evs[-1].record(stream)

    def one_step(evs):
        flush_l2()
        torch.cuda._sleep(SLEEP_CYCLES)  # keeps the GPU busy while the host queues the step
        enqueue_step(evs)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def new_events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = ""
    # clocks are sampled every 200 ms from before the warm-up to after the last measurement
    # pass; short runs get extra untimed steps so that the samples cover GPU activity
    sampler = ClockSampler(gpu_id) if not args.profile else None
    if sampler:
        sampler.__enter__()
    t_window = time.perf_counter()
    for _ in range(args.warmup):
        one_step(new_events(n_kernels + 1))
    st = da.read_status(pl, ws)
    if st != da.OK:
        raise RuntimeError(f"device status after warm-up: {da.status_string(st)}")
    mean = statistics.mean

    # ---- the timed steps: events at step boundaries only
    evs = [new_events(2) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        one_step(evs[i])
    barrier()
    step_us = [evs[i][0].elapsed_time(evs[i][1]) * 1e3 for i in range(args.steps)]

    # ---- per-kernel breakdown: the same steps with events between the kernels
    bevs = [new_events(n_kernels + 1) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        one_step(bevs[i])
    barrier()
    o = 1 if args.append else 0
    app_us = [bevs[i][0].elapsed_time(bevs[i][1]) * 1e3 for i in range(args.steps)] if args.append else [0.0]
    plan_us = [bevs[i][o].elapsed_time(bevs[i][o + 1]) * 1e3 for i in range(args.steps)]
    split_us = [bevs[i][o + 1].elapsed_time(bevs[i][o + 2]) * 1e3 for i in range(args.steps)]
    comb_us = [bevs[i][o + 2].elapsed_time(bevs[i][o + 3]) * 1e3 for i in range(args.steps)]
    st = da.read_status(pl, ws)
    if st != da.OK:
        raise RuntimeError(f"device status after timing: {da.status_string(st)}")
    local = [mean(step_us), mean(plan_us), mean(split_us), mean(comb_us), mean(app_us)]
    step_m, plan_m, split_m, comb_m, app_m = max_over_ranks(local, dist, dev)

    # CUDA-graph replay of the same step (context figure)
    graph_us = None
    if not args.no_graph and not args.profile:
        g = torch.cuda.CUDAGraph()
        gs = torch.cuda.Stream()
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            with torch.cuda.graph(g, stream=gs):
                if args.append:
                    da.append_rope(q_new, k_new, v_new, tab, lens, k, v, q_out=q_dec, stream=gs)
                make_plan(buf=pbuf, stream=gs)
                da.run(q_dec, k, v, tab, lens, pl, stream=gs, **kw)
        stream.wait_stream(gs)
        gt = []
        for i in range(args.warmup + args.steps):
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush_l2()
            torch.cuda._sleep(SLEEP_CYCLES)
            a.record(stream)
            g.replay()
            b_.record(stream)
            b_.synchronize()
            if i >= args.warmup:
                gt.append(a.elapsed_time(b_) * 1e3)
        graph_us = mean(gt)
        del g

    if sampler:
        while time.perf_counter() - t_window < 1.5:
            one_step(new_events(2))
            torch.cuda.synchronize()
        sampler.__exit__(None, None, None)

    # end to end through the C ABI: inputs of the step from pinned host memory, result back
    e2e = None
    if not args.no_e2e and not args.profile:
        # the step's inputs: q (or, with --append, the new q / k / v rows), page table, seq_lens
        dq = [q_new, k_new, v_new] if args.append else [q]
        hq = [torch.empty(t.shape, dtype=t.dtype).copy_(t.cpu()).pin_memory() for t in dq]
        htab = torch.from_numpy(pr.page_table).pin_memory()
        hlens = torch.from_numpy(pr.seq_lens).pin_memory()
        hout = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        hlse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * 2 for t in hq) + htab.numel() * 4 + hlens.numel() * 4
        d2h = hout.numel() * 4 + hlse.numel() * 4
        et = []
        for i in range(args.warmup + args.steps):
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush_l2()
            torch.cuda._sleep(SLEEP_CYCLES)
            a.record(stream)
            for dt, ht in zip(dq, hq):
                dt.copy_(ht, non_blocking=True)
            tab.copy_(htab, non_blocking=True)
            lens.copy_(hlens, non_blocking=True)
            if args.append:
                da.append_rope(q_new, k_new, v_new, tab, lens, k, v, q_out=q_dec)
            make_plan(buf=pbuf)
            da.run(q_dec, k, v, tab, lens, pl, **kw)
            hout.copy_(out, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)
            b_.record(stream)
            b_.synchronize()
            if i >= args.warmup:
                et.append(a.elapsed_time(b_) * 1e3)
        e2e_local = max_over_ranks([mean(et)], dist, dev)[0]
        e2e = {"value": round(e2e_local, 3), "unit": "us/step", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h),
               "note": ("per step: the new q/k/v rows" if args.append else "per step: q") +
                       ", page table and seq_lens from pinned host memory, " +
                       ("append + " if args.append else "") + "plan + split + combine, "
                       "out and lse back to pinned host memory; the KV cache stays resident in HBM"}

    if rank != 0:
        return 0
    alg = pr.algorithmic_bytes()
    peak, peak_kind = measured_peak()
    split_gbs = alg / (split_m * 1e-6) / 1e9
    step_gbs = alg / (step_m * 1e-6) / 1e9
    sc_gbs = alg / ((split_m + comb_m) * 1e-6) / 1e9  # split + combine, each timed between events
    traffic = None if mask_dev is not None else ncu_traffic(args.config, pr.tile_len)
    line = {
        "metric": METRIC, "value": round(step_m, 3), "unit": "us/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_m / 1e3, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": ("fp8e4m3 (q, P rounded to e4m3)" if args.mma8 else "fp8e4m3 (e4m3 products: q, P as exact e4m3 parts)")
        if pr.kv_dtype == "fp8e4m3" else "bf16",
        "data": "synthetic",
        "config": {**bench_config(pr, world),
                   **({"products": "e4m3 tensor cores (q and P rounded to e4m3)"} if args.mma8 else {})},
        "n_bins": pl.n_bins,
        "breakdown_note": "plan/split/combine: a second pass of the same steps with events between the kernels",
        "plan_us": round(plan_m, 3), "split_us": round(split_m, 3), "combine_us": round(comb_m, 3),
        "graph_step_us": None if graph_us is None else round(graph_us, 3),
        "algorithmic_bytes": int(alg),
        "hbm_gbs_step": round(step_gbs, 1), "pct_of_8tbs_step": round(100 * step_gbs / NOMINAL_HBM_GBS, 2),
        "hbm_gbs_split": round(split_gbs, 1), "pct_of_8tbs_split": round(100 * split_gbs / NOMINAL_HBM_GBS, 2),
        "hbm_gbs_split_combine": round(sc_gbs, 1), "frac_split_combine": round(sc_gbs / peak, 4),
        "roofline": {"bound": "hbm", "kernel": split_kernel_name(pr), "achieved": round(split_gbs, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(split_gbs / peak, 4),
                     "traffic": None if traffic is None else int(traffic)},
        "gpu_launches": n_kernels * args.steps,  # [append,] planner, split, combine kernels per timed step
    }
    if mask_dev is not None:
        nb = (pr.seq_lens.astype(np.int64) + pr.tile_len - 1) // pr.tile_len
        i = np.arange(int(nb.max()) if pr.batch else 0)
        kept = ((pr.tile_mask[:, :, i // 32] >> (i % 32).astype(np.uint32)) & 1).astype(bool) & (i[None, None, :] < nb[:, None, None])
        line["config"]["sparse"] = {"density": args.sparse, "kept_tiles": int(kept.sum()),
                                    "tiles": int(nb.sum()) * pr.n_kv_heads,
                                    "note": "algorithmic bytes count the kept tiles' KV only"}
    if args.append:
        # the fused pre-processing kernel: bytes it must move once (new q/k/v rows in, rotated q
        # and the k/v rows out, seq_lens and one page-table entry per new token)
        rows = pr.batch * pr.q_tokens
        app_bytes = rows * (2 * pr.n_q_heads + 4 * pr.n_kv_heads) * pr.head_dim * 2 + pr.batch * 4 + rows * 4
        line["config"]["fused_append_rope"] = True
        line["append_us"] = round(app_m, 3)
        line["append_roofline"] = {"bound": "latency", "bytes": int(app_bytes),
                                   "achieved_gbs": round(app_bytes / (app_m * 1e-6) / 1e9, 1),
                                   "note": "one block per new token; a few hundred KB per launch, so the "
                                           "launch and one dependent memory round trip set its time"}
    if sampler:
        line["clocks"] = sampler.summary()
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and not args.profile and world == 1:
        import oracle
        oracle.build()
        us, threads, sample = oracle_timing(pr, budget_s=15.0)
        line["cpu_baseline"] = {"value": round(us, 1), "unit": "us/step", "cores": threads, "kind": "oracle",
                                "sample": sample}
    emit(line, args)
    return 0


# ---------------------------------------------------------------- prefill (tensor-bound)

def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(p))["bf16_tflops"]), "measured (cuBLAS bf16, burst)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def prefill_traffic():
    """DRAM bytes per prefill-kernel launch from the committed ncu capture, if it was taken on the
    current kernel source (else None)."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", "prefill_kernel_dram_traffic.json")))
    except Exception:
        return None
    if d.get("source_hash") != prefill_source_hash():
        return None
    return int(d["configs"]["prefill"]["bytes_per_launch"])


def prefill_flops(pr) -> int:
    """Algorithmic FLOPs of causal prefill: row t of request b sees L_b - T + t + 1 keys (none
    when that is <= 0), and each key costs 2 d for q.k and 2 d for p v."""
    T, d = pr.q_tokens, pr.head_dim
    t = np.arange(T, dtype=np.int64)
    vis = np.clip(pr.seq_lens.astype(np.int64)[:, None] - T + 1 + t[None, :], 0, None)
    return int(vis.sum()) * pr.n_q_heads * 4 * d


def run_prefill(args, rank: int, world: int, local_rank: int, dist):
    import torch

    import paged_kv_decode_29_b200 as da
    from paged_kv_decode_29_b200 import build as dbuild

    if not os.path.exists(da.LIB_PATH):
        dbuild.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pr = make_workload(args)
    log(f"[rank {rank}] prefill workload {pr.name}: B={pr.batch} Hq={pr.n_q_heads} Hkv={pr.n_kv_heads} "
        f"d={pr.head_dim} T={pr.q_tokens} P={pr.page_size} tokens={int(pr.seq_lens.sum())}")
    bf = torch.bfloat16
    fp8 = pr.kv_dtype == "fp8e4m3"
    q = torch.from_numpy(pr.q.view(np.int16)).view(bf).to(dev)
    if fp8:
        k = torch.from_numpy(np.ascontiguousarray(pr.k_pages)).to(dev)
        v = torch.from_numpy(np.ascontiguousarray(pr.v_pages)).to(dev)
        sc = torch.from_numpy(np.ascontiguousarray(pr.kv_scales)).to(dev)
    else:
        k = torch.from_numpy(pr.k_pages.view(np.int16)).view(bf).to(dev)
        v = torch.from_numpy(pr.v_pages.view(np.int16)).view(bf).to(dev)
    tab, lens = (torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in (pr.page_table, pr.seq_lens))
    ws = None
    if fp8:
        ws = torch.empty(da.prefill_fp8_workspace_bytes(q.shape, k, tab, pr.q_tokens), dtype=torch.uint8, device=dev)

    def attend():  # one prefill: FP8 KV = the widening pass + the bf16 prefill kernel
        if fp8:
            da.prefill_fp8(q, k, v, sc, tab, lens, sm_scale=pr.sm_scale, workspace=ws, out=out, lse=lse, status=status)
        else:
            da.prefill(q, k, v, tab, lens, sm_scale=pr.sm_scale, out=out, lse=lse, status=status)
    out = torch.empty((pr.batch, pr.q_tokens, pr.n_q_heads, pr.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((pr.batch, pr.q_tokens, pr.n_q_heads), dtype=torch.float32, device=dev)
    status = torch.zeros((), dtype=torch.int32, device=dev)
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def one_step(a, b_):
        torch.sum(flush, dim=0, out=flush_sink)
        torch.cuda._sleep(SLEEP_CYCLES)
        a.record(stream)
        attend()
        b_.record(stream)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def ev():
        return torch.cuda.Event(enable_timing=True)

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = ""
    sampler = ClockSampler(gpu_id) if not args.profile else None
    if sampler:
        sampler.__enter__()
    t_window = time.perf_counter()
    for _ in range(args.warmup):
        one_step(ev(), ev())
    barrier()
    if int(status.item()) != da.OK:
        raise RuntimeError(f"device status after warm-up: {da.status_string(int(status.item()))}")
    evs = [(ev(), ev()) for _ in range(args.steps)]
    barrier()
    for a, b_ in evs:
        one_step(a, b_)
    barrier()
    if int(status.item()) != da.OK:
        raise RuntimeError(f"device status after timing: {da.status_string(int(status.item()))}")
    step_m = statistics.mean(a.elapsed_time(b_) * 1e3 for a, b_ in evs)
    if sampler:
        while time.perf_counter() - t_window < 1.5:
            one_step(ev(), ev())
            torch.cuda.synchronize()
        sampler.__exit__(None, None, None)

    e2e = None
    if not args.no_e2e and not args.profile:
        hq = torch.empty(q.shape, dtype=bf).copy_(q.cpu()).pin_memory()
        htab = torch.from_numpy(pr.page_table).pin_memory()
        hlens = torch.from_numpy(pr.seq_lens).pin_memory()
        hout = torch.empty(out.shape, dtype=torch.float32).pin_memory()
        hlse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        h2d = hq.numel() * 2 + htab.numel() * 4 + hlens.numel() * 4
        d2h = hout.numel() * 4 + hlse.numel() * 4
        et = []
        for i in range(args.warmup + args.steps):
            a, b_ = ev(), ev()
            torch.sum(flush, dim=0, out=flush_sink)
            torch.cuda._sleep(SLEEP_CYCLES)
            a.record(stream)
            q.copy_(hq, non_blocking=True)
            tab.copy_(htab, non_blocking=True)
            lens.copy_(hlens, non_blocking=True)
            attend()
            hout.copy_(out, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)
            b_.record(stream)
            b_.synchronize()
            if i >= args.warmup:
                et.append(a.elapsed_time(b_) * 1e3)
        e2e = {"value": round(max_over_ranks([statistics.mean(et)], dist, dev)[0], 3), "unit": "us/step",
               "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h),
               "note": "per step: q, page table and seq_lens from pinned host memory, prefill, out and lse back "
                       "to pinned host memory; the KV cache stays resident in HBM"}
    step_m = max_over_ranks([step_m], dist, dev)[0]
    if rank != 0:
        return 0
    flops = prefill_flops(pr)
    peak, peak_kind = measured_tensor_peak()
    tflops = flops / (step_m * 1e-6) / 1e12
    line = {
        "metric": PREFILL_METRIC,
        "value": round(step_m, 3), "unit": "us/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_m / 1e3, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (e4m3 KV widened to bf16)" if fp8 else "bf16",
        "data": "synthetic",
        "config": bench_config(pr, world, prefill=True),
        "algorithmic_flops": flops,
        "roofline": {"bound": "tensor", "kernel": "widen_kv_kernel + prefill_kernel" if fp8 else "prefill_kernel",
                     "achieved": round(tflops, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "traffic": prefill_traffic() if pr.name == "prefill" and not fp8 else None},
        "gpu_launches": args.steps * (2 if fp8 else 1),  # per timed step: the prefill kernel (FP8: and the widening)
    }
    if sampler:
        line["clocks"] = sampler.summary()
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline and not args.profile and world == 1:
        import oracle
        oracle.build()
        us, threads, sample = oracle_timing(pr, budget_s=15.0)
        line["cpu_baseline"] = {"value": round(us, 1), "unit": "us/step", "cores": threads, "kind": "oracle",
                                "sample": sample}
    emit(line, args)
    return 0


def main():
    args = parse()
    if args.write_traffic:
        write_traffic_json()
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
    try:
        if args.config == "prefill":
            return run_prefill(args, rank, world, local_rank, dist)
        return run_ours(args, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
