"""CPU pins of the oracle's block-sparse decode ("HPC-Ops: Tencent's CUDA Kernel Library for LLM
Inference Hot Paths", "How the kernels are organized around specific workload shapes": sparse
attention takes a precomputed block mask and skips the masked-out KV tiles). Each against
something other than the oracle's own code:
  * an all-ones mask is the dense decode and the dense plan, bit for bit;
  * torch SDPA (float64) over the kept keys, gathered densely per (request, KV head);
  * a pair with every tile masked has no visible key (out 0, lse -inf);
  * the sparse plan holds exactly the kept tiles, with the greedy rule replayed step by step.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import _helpers as H


def small(seq_lens, *, Hq=8, Hkv=2, d=64, P=16, T=1, kv="bf16", seed=21, tl=32):
    return W.make_problem(name="sparse", batch=len(seq_lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                          seq_lens=seq_lens, page_size=P, q_tokens=T, kv_dtype=kv, seed=seed, tile_len=tl)


def _kept(mask, b, h, i):
    return bool((int(mask[b, h, i // 32]) >> (i % 32)) & 1)


def test_all_ones_mask_is_dense():
    pr = small([1, 40, 129, 300], Hq=8, Hkv=2, T=2)
    o1, l1 = oracle.decode(pr)
    pl1 = oracle.plan(pr.seq_lens, 2, pr.tile_len, 7)
    pr.tile_mask = np.full((pr.batch, 2, 1), 0xFFFFFFFF, dtype=np.uint32)
    o2, l2 = oracle.decode(pr)
    pl2 = oracle.plan(pr.seq_lens, 2, pr.tile_len, 7, tile_mask=pr.tile_mask)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    for key in ("bin_off", "units", "pair_off"):
        assert np.array_equal(pl1[key], pl2[key])


@pytest.mark.parametrize("case", [
    dict(seq_lens=[1, 40, 129, 300], Hq=8, Hkv=2, d=64, T=1, density=0.5),
    dict(seq_lens=[70, 200], Hq=4, Hkv=4, d=128, T=1, density=0.3),
    dict(seq_lens=[33, 97, 160], Hq=6, Hkv=2, d=64, T=3, density=0.6),
    dict(seq_lens=[64, 190], Hq=4, Hkv=2, d=64, T=2, density=0.4, kv="fp8e4m3"),
])
def test_sparse_oracle_matches_sdpa_on_kept_keys(case):
    density = case.pop("density")
    pr = small(**case)
    pr.tile_mask = W.make_tile_mask(pr, density, keep_last=False)
    out, lse = oracle.decode(pr)
    G, T, tl = pr.group, pr.q_tokens, pr.tile_len
    q = H.q_values(pr)
    for b in range(pr.batch):
        Lb = int(pr.seq_lens[b])
        K, V = H.dense_kv(pr, b, "k"), H.dense_kv(pr, b, "v")  # [Hkv][Lb][d]
        for h in range(pr.n_kv_heads):
            keep = np.array([_kept(pr.tile_mask, b, h, j // tl) for j in range(Lb)], dtype=bool)
            for t in range(T):
                vis = keep & (np.arange(Lb) <= Lb - T + t)
                for g in range(G):
                    qh = h * G + g
                    if not vis.any():
                        assert np.all(out[b, t, qh] == 0) and np.isneginf(lse[b, t, qh])
                        continue
                    Q = torch.from_numpy(q[b, t, qh])[None, None, None]          # [1][1][1][d]
                    Kt = torch.from_numpy(K[h][vis])[None, None]                   # [1][1][n][d]
                    Vt = torch.from_numpy(V[h][vis])[None, None]
                    o = torch.nn.functional.scaled_dot_product_attention(Q, Kt, Vt, scale=pr.sm_scale)
                    s = (Q @ Kt.transpose(-1, -2))[0, 0, 0] * pr.sm_scale
                    np.testing.assert_allclose(out[b, t, qh], o[0, 0, 0].numpy(), rtol=0, atol=1e-12)
                    assert abs(lse[b, t, qh] - torch.logsumexp(s, -1).item()) < 1e-12


def test_fully_masked_pair_has_no_visible_key():
    pr = small([100, 50], Hq=4, Hkv=2, T=1)
    m = np.full((2, 2, 1), 0xFFFFFFFF, dtype=np.uint32)
    m[0, 1, 0] = 0  # request 0, KV head 1: every tile masked
    pr.tile_mask = m
    out, lse = oracle.decode(pr)
    assert np.all(out[0, 0, 2:4] == 0) and np.all(np.isneginf(lse[0, 0, 2:4]))
    assert np.all(np.isfinite(lse[0, 0, 0:2])) and np.all(np.isfinite(lse[1]))


@pytest.mark.parametrize("lens,Hkv,tl,n_bins,density", [
    ([5, 300, 1000, 64], 2, 64, 5, 0.5),
    ([4096] * 6, 4, 256, 7, 0.3),
    ([17, 18, 1, 0, 999], 3, 16, 11, 0.7),
])
def test_sparse_plan_holds_the_kept_tiles_greedily(lens, Hkv, tl, n_bins, density):
    pr = W.make_problem(name="m", batch=len(lens), n_q_heads=Hkv, n_kv_heads=Hkv, head_dim=64, seq_lens=lens,
                        page_size=16, tile_len=tl, seed=5)
    mask = W.make_tile_mask(pr, density, keep_last=False)
    pl = oracle.plan(pr.seq_lens, Hkv, tl, n_bins, tile_mask=mask)
    units, bin_off = pl["units"], pl["bin_off"]
    # coverage: exactly the kept tiles, each once; token ranges and slots by their definition
    want = {(b, h, i) for b in range(len(lens)) for h in range(Hkv) for i in range(-(-lens[b] // tl))
            if _kept(mask, b, h, i)}
    got = [(int(u[0]), int(u[1]), int(u[6])) for u in units]
    assert sorted(got) == sorted(want) and len(got) == len(want)
    for u in units:
        b, h, i = int(u[0]), int(u[1]), int(u[6])
        assert u[2] == i * tl and u[3] == min((i + 1) * tl, lens[b]) and u[4] == lens[b]
        kept_before = sum(_kept(mask, b, h, k) for k in range(i))
        m = sum(_kept(mask, b, h, k) for k in range(-(-lens[b] // tl)))
        assert u[5] == (-1 if m == 1 else pl["pair_off"][b * Hkv + h] + kept_before)
    # the greedy rule replayed: costs in stable descending order, each to the least-loaded bin
    flat = sorted(((b, h, i) for (b, h, i) in want), key=lambda x: (x[0], x[1], x[2]))
    cost = {t: min((t[2] + 1) * tl, lens[t[0]]) - t[2] * tl for t in flat}
    seq = sorted(flat, key=lambda t: -cost[t])  # stable: ties keep (b, h, i) order
    load = [0] * n_bins
    bins = [[] for _ in range(n_bins)]
    for t in seq:
        k = min(range(n_bins), key=lambda x: (load[x], x))
        bins[k].append(t)
        load[k] += cost[t]
    for k in range(n_bins):
        have = [(int(u[0]), int(u[1]), int(u[6])) for u in units[bin_off[k]:bin_off[k + 1]]]
        assert have == bins[k]
