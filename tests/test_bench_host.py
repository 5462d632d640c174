"""bench.py's host-side arithmetic on CPU: the algorithmic FLOPs behind the prefill roofline, which
split kernel a workload runs on, and the rule that an ncu traffic figure is reported only while
the kernel sources hash as they did at the capture."""
import hashlib
import json
import os
import shutil

import numpy as np

import bench
import workloads as W


class _Pr:
    def __init__(self, lens, T, Hq, d=128):
        self.seq_lens = np.asarray(lens, dtype=np.int32)
        self.q_tokens, self.n_q_heads, self.head_dim = T, Hq, d


def test_prefill_flops_closed_forms():
    # T = L: row t sees t + 1 keys, sum = T (T + 1) / 2; each (row, key) costs 4 d per head
    assert bench.prefill_flops(_Pr([2048] * 4, 2048, 32)) == 4 * 32 * 4 * 128 * 2048 * 2049 // 2
    # L > T: row t sees L - T + t + 1 keys
    L, T = 1000, 10
    assert bench.prefill_flops(_Pr([L], T, 1)) == 4 * 128 * sum(L - T + t + 1 for t in range(T))
    # L < T: the first T - L rows see nothing
    assert bench.prefill_flops(_Pr([3], 5, 2)) == 4 * 2 * 128 * (0 + 0 + 1 + 2 + 3)
    # the full prefill workload: 137.5 GFLOP
    pr = _Pr(W.config_seq_lens("prefill"), W.CONFIGS["prefill"]["q_tokens"], W.CONFIGS["prefill"]["n_q_heads"])
    assert abs(bench.prefill_flops(pr) / 1e9 - 137.506062336) < 1e-6


def test_split_kernel_name():
    class P:
        pass

    p = P()
    p.kv_dtype, p.head_dim, p.group, p.q_tokens = "fp8e4m3", 128, 4, 4
    assert bench.split_kernel_name(p) == "split_tc_kernel"
    p.q_tokens = 5  # G*T = 20 > 16
    assert bench.split_kernel_name(p) == "split_kernel"
    p.kv_dtype, p.q_tokens = "bf16", 1
    assert bench.split_kernel_name(p) == "split_kernel"
    p.kv_dtype, p.head_dim = "fp8e4m3", 64
    assert bench.split_kernel_name(p) == "split_kernel"


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    # a copy of the tree whose capture files carry the copy's own source hashes reports the figures;
    # once a kernel source differs by one byte, it reports none
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(bench.ROOT, "profiles"), root / "profiles")
    shutil.copytree(os.path.join(bench.ROOT, "paged_kv_decode_29_b200", "csrc"),
                    root / "paged_kv_decode_29_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(root))
    split_json = root / "profiles" / "split_kernel_dram_traffic.json"
    d = json.load(open(split_json))
    d["source_hash"] = bench.kernel_source_hash()
    split_json.write_text(json.dumps(d))
    h = hashlib.sha256()
    for f in ("prefill.cu", "tc.cuh", "common.cuh"):
        h.update((root / "paged_kv_decode_29_b200" / "csrc" / f).read_bytes())
    pf_json = root / "profiles" / "prefill_kernel_dram_traffic.json"
    d = json.load(open(pf_json))
    d["source_hash"] = h.hexdigest()[:16]
    pf_json.write_text(json.dumps(d))
    assert bench.ncu_traffic("uniform", 256) == json.load(open(split_json))["configs"]["uniform/tl256"]["bytes_per_launch"]
    assert bench.prefill_traffic() == d["configs"]["prefill"]["bytes_per_launch"]
    assert bench.ncu_traffic("uniform", 128) is None  # a tile length that was not captured
    for f in ("split.cu", "prefill.cu"):
        path = root / "paged_kv_decode_29_b200" / "csrc" / f
        path.write_bytes(path.read_bytes() + b"\n")
    assert bench.ncu_traffic("uniform", 256) is None
    assert bench.prefill_traffic() is None


def test_config_algorithmic_bytes_matches_the_generated_workload():
    # the traffic scaling counts a workload's bytes without generating it: same figure as the problem's
    for name, batch in (("tiny", None), ("fp8_spec", 2), ("uniform", 3)):
        pr = W.make_problem(name=name, seq_lens=W.config_seq_lens(name)[:batch] if batch else W.config_seq_lens(name),
                            **{k: v for k, v in W.CONFIGS[name].items() if k not in ("batch", "pool_pages")},
                            batch=batch or W.CONFIGS[name]["batch"])
        assert bench.config_algorithmic_bytes(name, batch) == pr.algorithmic_bytes(), name


def test_write_traffic_refuses_tables_captured_on_other_sources(tmp_path, monkeypatch):
    # the capture tables carry the hash of the sources they were taken on; after a kernel edit
    # --write-traffic must not stamp them with the new hash
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    shutil.copytree(os.path.join(bench.ROOT, "paged_kv_decode_29_b200", "csrc"),
                    root / "paged_kv_decode_29_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(root))
    monkeypatch.setitem(bench.SPLIT_TRAFFIC_CAPTURED, "source_hash", "0" * 16)
    monkeypatch.setitem(bench.PREFILL_TRAFFIC_CAPTURED, "source_hash", "0" * 16)
    assert bench.write_traffic_json() == []
    assert not (root / "profiles" / "split_kernel_dram_traffic.json").exists()
    assert not (root / "profiles" / "prefill_kernel_dram_traffic.json").exists()
    # with the current hashes both tables are written, stamped with the hash they were taken on
    monkeypatch.setitem(bench.SPLIT_TRAFFIC_CAPTURED, "source_hash", bench.kernel_source_hash())
    monkeypatch.setitem(bench.PREFILL_TRAFFIC_CAPTURED, "source_hash", bench.prefill_source_hash())
    assert bench.write_traffic_json() == ["split", "prefill"]
    d = json.load(open(root / "profiles" / "split_kernel_dram_traffic.json"))
    assert d["source_hash"] == bench.kernel_source_hash()
    assert set(d["configs"]) == {f"{n}/tl{W.CONFIGS[n]['tile_len']}" for n in bench.SPLIT_TRAFFIC_CAPTURED["configs"]}


def test_both_arms_report_the_same_config():
    pr = W.make_config("tiny")
    assert bench.bench_config(pr, 1) == bench.bench_config(pr, 1)
    c = bench.bench_config(pr, 1)
    assert c["workload"] == "tiny" and "l2" in c and c["parallelism"] == "single GPU"
    assert "n_bins" not in c


def test_fp8_kv_option_builds_the_same_workload_with_e4m3_pages():
    # --fp8-kv keeps the workload's shape, lengths and seed and only changes the KV cache to E4M3
    # pages with per-(page, head) scales (the prefill entry point then widens them)
    import argparse
    base = argparse.Namespace(config="prefill", tile_len=0, batch=1, fp8_kv=False)
    fp8 = argparse.Namespace(config="prefill", tile_len=0, batch=1, fp8_kv=True)
    a, b = bench.make_workload(base), bench.make_workload(fp8)
    assert a.kv_dtype == "bf16" and b.kv_dtype == "fp8e4m3"
    assert np.array_equal(a.seq_lens, b.seq_lens) and np.array_equal(a.q, b.q)
    assert np.array_equal(a.page_table, b.page_table)
    assert b.k_pages.dtype == np.uint8 and b.kv_scales.shape == (2, b.num_pages, b.n_kv_heads)
    assert bench.bench_config(b, 1, prefill=True)["kv_dtype"] == "fp8e4m3"
