"""Planner kernel vs the oracle's sequential greedy: byte-exact work lists."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_29_b200 as da
import workloads as W

pytestmark = pytest.mark.gpu


def gpu_plan(lens, hkv, tl, n_bins, max_total=None):
    t = torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda")
    total = int(np.asarray(lens, dtype=np.int64).clip(0).sum()) if max_total is None else max_total
    pl = da.plan(t, hkv, tl, max_total_kv_tokens=total, n_bins=n_bins)
    st = da.read_status(pl)
    return pl, st, da.plan_contents(pl, t)


def assert_same(lens, hkv, tl, n_bins):
    pl, st, got = gpu_plan(lens, hkv, tl, n_bins)
    assert st == da.OK, da.status_string(st)
    ref = oracle.plan(lens, hkv, tl, n_bins)
    assert got["n_units"] == ref["n_units"]
    assert np.array_equal(got["bin_off"], ref["bin_off"])
    assert np.array_equal(got["units"], ref["units"]), "work lists differ"
    return got


@pytest.mark.parametrize("name", ["tiny", "uniform", "mixed", "long_b1", "long_b4", "fp8_spec"])
def test_plan_configs_default_bins(name):
    c = W.CONFIGS[name]
    assert_same(W.config_seq_lens(name), c["n_kv_heads"], c["tile_len"], da.default_bins())


@pytest.mark.parametrize("seed", range(6))
def test_plan_random(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.choice([1, 3, 17, 64, 300, 1500]))
    max_len = int(rng.choice([20, 700, 5000, 70000]))
    lens = rng.integers(0, max_len, size=B)
    lens[rng.random(B) < 0.1] = 0
    hkv = int(rng.choice([1, 2, 8]))
    n_bins = int(rng.choice([1, 5, 148, 592, 1184, 4096]))
    # smallest tile (multiple of 16) that keeps the oracle's tiles x bins loop small
    tl = 16
    while hkv * int(((lens + tl - 1) // tl).sum()) * n_bins > 3e8:
        tl *= 2
    assert_same(lens, hkv, tl, n_bins)


@pytest.mark.parametrize("lens,hkv,tl,n_bins", [
    ([0, 0, 0], 2, 64, 8),                # no tiles at all
    ([1], 1, 16, 1),                      # one tile, one bin
    ([1], 8, 16, 592),
    ([4096] * 32, 8, 256, 592),           # full tiles only: round-robin
    (list(range(1, 1200)), 8, 1024, 592), # ~9.6k partial tiles through the sequential pass
    ([65536] * 3 + [17] * 5, 4, 128, 7),
    ([300] * 500, 8, 256, 592),           # 4000 partial tiles of one cost: ties in every round
    (list(range(1, 3000, 7)), 2, 64, 37), # few bins, many rounds of the batched pass
    ([4000 + 37 * i for i in range(80)], 8, 256, 592),  # the first batch leaves a few tiles over
])
def test_plan_edges(lens, hkv, tl, n_bins):
    assert_same(lens, hkv, tl, n_bins)


def test_plan_is_deterministic():
    lens = W.config_seq_lens("mixed")
    a = gpu_plan(lens, 8, 256, 592)[2]
    b = gpu_plan(lens, 8, 256, 592)[2]
    assert all(np.array_equal(a[k], b[k]) for k in ("bin_off", "units"))


def test_plan_capacity_overflow_sets_status():
    lens = [1000, 2000]
    pl, st, got = gpu_plan(lens, 2, 64, 8, max_total=100)
    assert st == da.ECAPACITY
    assert got["n_units"] == -1 and got["status"] == da.ECAPACITY


def test_plan_negative_length_sets_status():
    pl, st, _ = gpu_plan([5, -3, 7], 1, 16, 4, max_total=100)
    assert st == da.EDEVICE
