"""Writes split_kernel_dram_traffic.json: DRAM bytes (read + write) per split-kernel launch of each
workload, scaled from an ncu capture of a smaller case of the same workload (its first requests)
by the ratio of algorithmic bytes. Reads measured within 0.05% of the algorithmic bytes on every
captured case, so traffic grows in proportion. The figures below are the captured ncu values
(`dram__bytes_read.sum`, `dram__bytes_write.sum`) of one split-kernel launch of each smaller case (the split kernel that runs for the workload: split_tc_kernel for fp8_spec,
split_kernel for the others).
It also writes prefill_kernel_dram_traffic.json: the prefill kernel's DRAM bytes per launch on
the full prefill workload, captured directly (the workload holds a few hundred MB on the device).
Run from the repository root after the capture: python profiles/make_traffic_json.py"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import workloads as W  # noqa: E402

# workload -> (requests captured, dram read bytes, dram write bytes) of the captured launch
CAPTURED = {
    "uniform": (8, 134362368, 3598080),
    "mixed": (16, 1039144960, 17676288),
    "fp8_spec": (4, 167250432, 6338304),
    "long_b4": (1, 536982272, 5664256),
}


# prefill_kernel on the full prefill workload (dram read bytes, dram write bytes) of the launch
# captured by `ncu --set full` (profiles/prefill_kernel_prefill_b4.md)
PREFILL_CAPTURED = (108316928, 87724800)


def alg_bytes(name, batch=None):
    """Problem.algorithmic_bytes() of the workload (or its first `batch` requests) without
    generating its data."""
    c = W.CONFIGS[name]
    L = np.asarray(W.config_seq_lens(name), dtype=np.int64)
    if batch is not None:
        L = L[:batch]
    B, d, P, hkv, hq, T = len(L), c["head_dim"], c["page_size"], c["n_kv_heads"], c["n_q_heads"], c["q_tokens"]
    eb = 1 if c["kv_dtype"] == "fp8e4m3" else 2
    kv = int(L.sum()) * hkv * d * eb * 2
    q = B * T * hq * d * 2
    out = B * T * hq * (d + 1) * 4
    pages = int(((L + P - 1) // P).sum())
    table = pages * 4 + B * 4
    scales = pages * hkv * 2 * 4 if c["kv_dtype"] == "fp8e4m3" else 0
    return kv + q + out + table + scales


def source_hash():
    h = hashlib.sha256()
    for f in ("split.cu", "split_tc.cu", "walk.cuh", "tc.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "paged_kv_decode_29_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def prefill_source_hash():
    h = hashlib.sha256()
    for f in ("prefill.cu", "tc.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "paged_kv_decode_29_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def main():
    out = {"source_hash": source_hash(), "configs": {}}
    for name, (nb, rd, wr) in CAPTURED.items():
        small, full = alg_bytes(name, nb), alg_bytes(name)
        scale = full / small
        out["configs"][f"{name}/tl{W.CONFIGS[name]['tile_len']}"] = {
            "bytes_per_launch": int(round((rd + wr) * scale)),
            "captured_requests": nb, "captured_read": rd, "captured_write": wr,
            "captured_algorithmic": small, "scale": round(scale, 6),
            "read_over_algorithmic": round(rd / small, 5),
        }
    p = os.path.join(ROOT, "profiles", "split_kernel_dram_traffic.json")
    with open(p, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))
    rd, wr = PREFILL_CAPTURED
    pf = {"source_hash": prefill_source_hash(),
          "configs": {"prefill": {"bytes_per_launch": rd + wr, "captured_read": rd, "captured_write": wr}}}
    with open(os.path.join(ROOT, "profiles", "prefill_kernel_dram_traffic.json"), "w") as f:
        json.dump(pf, f, indent=1)


if __name__ == "__main__":
    main()
