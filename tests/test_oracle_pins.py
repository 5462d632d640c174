"""Pins of the CPU oracle to things other than itself (no GPU needed).

Attention: a library special case (torch SDPA in float64 on gathered dense
K/V), closed forms (one key, q = 0, identical keys), invariants (split-KV +
LSE combine, softmax weights sum to 1, page renumbering, GQA == MHA with
repeated KV heads) and the spec-decode reduction (row t of a T-token query ==
single-token decode over the first Lb - T + 1 + t keys).

FP8: the E4M3 code table against torch.float8_e4m3fn and the OCP anchors; the
generator's encoder against a brute-force nearest-code search.

Planner: a hand-derived worked example, coverage, slots, determinism, the
greedy property replayed step by step, and list scheduling's makespan bound.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import _helpers as H

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small(seq_lens, *, Hq=8, Hkv=2, d=64, P=16, T=1, kv="bf16", seed=11, peaky=0.0, pool=None):
    return W.make_problem(name="small", batch=len(seq_lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                          seq_lens=seq_lens, page_size=P, q_tokens=T, kv_dtype=kv, seed=seed,
                          pool_pages=pool, peaky_frac=peaky)


# ---------------------------------------------------------------- FP8 E4M3 format

def test_e4m3_table_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_format_anchors():
    v = oracle.e4m3_value
    assert v(0x00) == 0.0 and math.copysign(1, v(0x80)) == -1
    assert v(0x01) == 2.0 ** -9          # smallest subnormal
    assert v(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert v(0x08) == 2.0 ** -6          # smallest normal
    assert v(0x38) == 1.0 and v(0x40) == 2.0
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0
    pos = np.array([v(c) for c in range(0x7F)])
    assert np.all(np.diff(pos) > 0)      # monotone in the code
    for c in range(0x7F):
        assert v(c | 0x80) == -v(c)


def _nearest_code(x):
    """Brute force: nearest finite code, ties to the code with even mantissa, saturating."""
    tab = oracle.e4m3_table()
    fin = [c for c in range(256) if not np.isnan(tab[c])]
    xs = min(max(x, -448.0), 448.0)
    best = None
    for c in fin:
        dist = abs(tab[c] - xs)
        key = (dist, c & 1, 0 if (tab[c] != 0 or math.copysign(1, xs) == math.copysign(1, tab[c])) else 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_e4m3_encoder_brute_force():
    tab = oracle.e4m3_table()
    pos = np.sort(tab[:0x7F])
    mids = (pos[1:] + pos[:-1]) / 2                    # exact ties
    rng = np.random.default_rng(5)
    xs = np.concatenate([pos, mids, -mids, rng.normal(0, 60, 2000), rng.uniform(-2 ** -5, 2 ** -5, 500),
                         [449.0, 500.0, 1e4, -1e4, 464.0, 2.0 ** -10, -2.0 ** -10]]).astype(np.float32)
    got = W.e4m3_encode(xs)
    for x, g in zip(xs.tolist(), got.tolist()):
        e = _nearest_code(float(x))
        assert tab[g] == tab[e], (x, g, e)
    # and the library conversion (RNE) where it does not overflow
    small_x = xs[np.abs(xs) <= 448]
    lib = torch.from_numpy(small_x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(tab[lib], tab[W.e4m3_encode(small_x)])


# ---------------------------------------------------------------- attention definition

def _sdpa_rows(pr):
    """torch SDPA (float64, CPU) per request on gathered dense K/V; rows with no visible key -> NaN."""
    G, T, d = pr.group, pr.q_tokens, pr.head_dim
    q = H.q_values(pr)
    outs, lses = [], []
    for b in range(pr.batch):
        Lb = int(pr.seq_lens[b])
        K = torch.from_numpy(H.dense_kv(pr, b, "k")).repeat_interleave(G, 0)   # [Hq][Lb][d]
        V = torch.from_numpy(H.dense_kv(pr, b, "v")).repeat_interleave(G, 0)
        Q = torch.from_numpy(q[b].transpose(1, 0, 2).copy())                  # [Hq][T][d]
        t = torch.arange(T)[:, None]
        j = torch.arange(Lb)[None, :]
        mask = j <= (Lb - T + t)                                               # [T][Lb]
        o = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None], attn_mask=mask,
                                                             scale=pr.sm_scale)[0]
        s = (Q @ K.transpose(1, 2)) * pr.sm_scale
        s = s.masked_fill(~mask, float("-inf"))
        lse = torch.logsumexp(s, dim=-1)                                       # [Hq][T]
        outs.append(o.transpose(0, 1).numpy())
        lses.append(lse.transpose(0, 1).numpy())
    return outs, lses


@pytest.mark.parametrize("case", [
    dict(cfg="tiny"),
    dict(seq_lens=[1, 5, 33, 64], Hq=8, Hkv=2, d=64, P=16, T=1),
    dict(seq_lens=[3, 40, 129], Hq=4, Hkv=4, d=128, P=16, T=1),
    dict(seq_lens=[7, 100], Hq=8, Hkv=1, d=64, P=64, T=3),
    dict(seq_lens=[2, 19, 70], Hq=6, Hkv=2, d=64, P=16, T=4),
    dict(seq_lens=[1, 31, 90], Hq=4, Hkv=2, d=128, P=16, T=2, kv="fp8e4m3"),
    dict(seq_lens=[50, 77], Hq=8, Hkv=2, d=64, P=16, T=1, peaky=0.2),
])
def test_oracle_matches_torch_sdpa(case):
    pr = W.make_config("tiny") if case.get("cfg") == "tiny" else small(**case)
    out, lse = oracle.decode(pr)
    ref_o, ref_l = _sdpa_rows(pr)
    for b in range(pr.batch):
        Lb = int(pr.seq_lens[b])
        for t in range(pr.q_tokens):
            if Lb - pr.q_tokens + t < 0:
                assert np.all(out[b, t] == 0) and np.all(np.isneginf(lse[b, t]))
                continue
            np.testing.assert_allclose(out[b, t], ref_o[b][t], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, t], ref_l[b][t], rtol=0, atol=1e-12)


def test_one_key_closed_form():
    pr = small([1, 1, 1], Hq=4, Hkv=2, d=64)
    out, lse = oracle.decode(pr)
    q = H.q_values(pr)
    for b in range(3):
        K, V = H.dense_kv(pr, b, "k"), H.dense_kv(pr, b, "v")
        for qh in range(4):
            h = qh // 2
            assert np.array_equal(out[b, 0, qh], V[h, 0])                   # out = the V row
            assert lse[b, 0, qh] == pytest.approx(pr.sm_scale * float(q[b, 0, qh] @ K[h, 0]), abs=1e-13)


def test_zero_query_closed_form():
    pr = small([5, 37, 64], Hq=4, Hkv=2, d=64, T=2)
    pr.q = np.zeros_like(pr.q)
    out, lse = oracle.decode(pr)
    for b in range(3):
        Lb = int(pr.seq_lens[b])
        V = H.dense_kv(pr, b, "v")
        for t in range(2):
            n = Lb - 2 + t + 1
            for qh in range(4):
                np.testing.assert_allclose(out[b, t, qh], V[qh // 2, :n].mean(0), atol=1e-13)
                assert lse[b, t, qh] == pytest.approx(math.log(n), abs=1e-13)


def test_identical_keys_closed_form():
    pr = small([9, 40], Hq=4, Hkv=1, d=64)
    k = pr.k_pages.copy()
    k[:, :, :, :] = pr.k_pages[pr.page_table[0, 0], :, 0, :][None, :, None, :]   # every K row := one row
    pr.k_pages = k
    out, lse = oracle.decode(pr)
    q = H.q_values(pr)
    krow = W.bf16_bits_to_f32(k[0, 0, 0]).astype(np.float64)
    for b in range(2):
        Lb = int(pr.seq_lens[b])
        V = H.dense_kv(pr, b, "v")
        for qh in range(4):
            s = pr.sm_scale * float(q[b, 0, qh] @ krow)
            np.testing.assert_allclose(out[b, 0, qh], V[0].mean(0), atol=1e-13)
            assert lse[b, 0, qh] == pytest.approx(s + math.log(Lb), abs=1e-12)


def test_softmax_weights_sum_to_one():
    pr = small([300, 1000], Hq=4, Hkv=2, d=64, peaky=0.05, T=3)
    for b in range(2):
        for t in range(3):
            _, _, n, w = oracle.attend(pr, b, t, 1, weights=True)
            assert n == int(pr.seq_lens[b]) - 3 + t + 1
            assert np.all(w >= 0)
            assert abs(w.sum() - 1.0) < 1e-12


def _lse_combine(parts):
    """Merge (o_i, lse_i) pieces: weights exp(lse_i - max), empty pieces (lse -inf) weigh 0."""
    lses = np.array([p[1] for p in parts])
    M = lses.max()
    if np.isneginf(M):
        return np.zeros_like(parts[0][0]), -np.inf
    w = np.exp(lses - M)
    o = sum(wi * p[0] for wi, p in zip(w, parts)) / w.sum()
    return o, M + math.log(w.sum())


def test_split_partition_invariance():
    pr = small([1, 200, 777], Hq=4, Hkv=2, d=64, T=4, peaky=0.05)
    rng = np.random.default_rng(3)
    for b in range(3):
        Lb = int(pr.seq_lens[b])
        for t in range(4):
            for qh in (0, 3):
                full_o, full_l, _ = oracle.attend(pr, b, t, qh)
                for _ in range(4):
                    cuts = np.sort(rng.integers(0, Lb + 1, size=rng.integers(0, 6)))
                    edges = [0] + cuts.tolist() + [Lb + 3]           # includes empty and past-the-end pieces
                    parts = [oracle.attend(pr, b, t, qh, lo, hi)[:2] for lo, hi in zip(edges[:-1], edges[1:])]
                    o, l = _lse_combine(parts)
                    if np.isneginf(full_l):
                        assert np.isneginf(l) and np.all(o == 0)
                        continue
                    np.testing.assert_allclose(o, full_o, atol=1e-12)
                    assert l == pytest.approx(full_l, abs=1e-12)


@pytest.mark.parametrize("kv", ["bf16", "fp8e4m3"])
def test_page_renumbering_invariance(kv):
    pr = small([17, 95, 160], Hq=4, Hkv=2, d=64, T=2, kv=kv)
    o1, l1 = oracle.decode(pr)
    o2, l2 = oracle.decode(H.repage(pr, 9))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_gqa_equals_mha_with_repeated_kv():
    pr = small([33, 120], Hq=8, Hkv=2, d=64, T=2)
    o1, l1 = oracle.decode(pr)
    o2, l2 = oracle.decode(H.as_mha(pr))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_spec_rows_reduce_to_single_token_decode():
    T = 4
    pr = small([4, 21, 130], Hq=4, Hkv=2, d=64, T=T)
    out, lse = oracle.decode(pr)
    for t in range(T):
        L1 = pr.seq_lens.astype(np.int64) - T + 1 + t
        one = H.with_lens(pr, L1, q_tokens=1, q=pr.q[:, t:t + 1])
        o1, l1 = oracle.decode(one)
        assert np.array_equal(out[:, t], o1[:, 0]) and np.array_equal(lse[:, t], l1[:, 0])


def test_rows_subset_matches_full():
    pr = small([40, 90], Hq=4, Hkv=2, d=64, T=2)
    out, lse = oracle.decode(pr)
    rows = np.array([[1, 1, 3], [0, 0, 0], [1, 0, 2]])
    o, l = oracle.decode_rows(pr, rows)
    for i, (b, t, qh) in enumerate(rows):
        assert np.array_equal(o[i], out[b, t, qh]) and l[i] == lse[b, t, qh]


# ---------------------------------------------------------------- planner

def _bins(pl, n_bins):
    bo, U = pl["bin_off"], pl["units"]
    return [U[bo[k]:bo[k + 1]] for k in range(n_bins)]


def test_plan_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "plan_tiny_worked_example.json")))
    pl = oracle.plan(g["seq_lens"], g["n_kv_heads"], g["tile_len"], g["n_bins"])
    bins = _bins(pl, g["n_bins"])
    for k in range(g["n_bins"]):
        exp = g["expected_bins"].get(str(k), [])
        got = bins[k][:, :7].tolist()
        assert got == exp, (k, got, exp)


def _check_plan(seq_lens, Hkv, tl, n_bins):
    pl = oracle.plan(seq_lens, Hkv, tl, n_bins)
    L = np.asarray(seq_lens, dtype=np.int64)
    nb = (L + tl - 1) // tl
    U = int(Hkv * nb.sum())
    assert pl["n_units"] == U and pl["bin_off"][-1] == U
    units = pl["units"]
    # coverage: every token of every (b, h) exactly once
    cover = {}
    for r in units:
        b, h, beg, end, sl, slot, i, _ = r.tolist()
        assert sl == L[b] and beg == i * tl and end == min((i + 1) * tl, sl) and end > beg
        cover.setdefault((b, h), []).append((beg, end))
        exp_slot = -1 if nb[b] == 1 else pl["pair_off"][b * Hkv + h] + i
        assert slot == exp_slot
    for b in range(len(L)):
        for h in range(Hkv):
            segs = sorted(cover.get((b, h), []))
            pos = 0
            for beg, end in segs:
                assert beg == pos
                pos = end
            assert pos == L[b]
    slots = [r[5] for r in units if r[5] >= 0]
    assert len(slots) == len(set(slots))
    # greedy property, replayed: in assignment order (cost desc, then (b,h,i)), each tile lands on a
    # bin whose load was minimal at that moment, lowest index on ties
    load = np.zeros(n_bins, dtype=np.int64)
    order = []
    for k in range(n_bins):
        for pos, r in enumerate(units[pl["bin_off"][k]:pl["bin_off"][k + 1]]):
            order.append((-(int(r[3]) - int(r[2])), int(r[0]), int(r[1]), int(r[6]), k, pos))
    order.sort()
    seen = np.zeros(n_bins, dtype=np.int64)
    for negc, b, h, i, k, pos in order:
        assert pos == seen[k]
        assert load[k] == load.min() and k == int(np.flatnonzero(load == load.min())[0])
        load[k] += -negc
        seen[k] += 1
    # list-scheduling bound: makespan <= W/N + max cost
    W_ = int(Hkv * L.sum())
    assert load.max() <= W_ / n_bins + min(tl, int(L.max()) if len(L) else 0) + 1e-9
    return pl


@pytest.mark.parametrize("args", [
    ([17, 300], 1, 64, 148),
    ([4096] * 32, 8, 256, 592),
    ([1, 2, 3, 255, 256, 257, 1000], 3, 64, 5),
    ([0, 5, 0, 70], 2, 16, 3),
    (list(np.random.default_rng(1).integers(1, 5000, 40)), 4, 128, 37),
])
def test_plan_invariants(args):
    _check_plan(*args)


def test_plan_equal_costs_round_robin():
    n_bins = 7
    pl = oracle.plan([512] * 5, 2, 64, n_bins)      # 80 equal tiles
    units = pl["units"]
    # k-th tile in (b, h, i) order goes to bin k mod N, position k div N
    for k in range(n_bins):
        got = units[pl["bin_off"][k]:pl["bin_off"][k + 1]]
        lex = [(int(r[0]) * 2 + int(r[1])) * 8 + int(r[6]) for r in got]
        assert lex == list(range(k, 80, n_bins))


def test_plan_deterministic_and_capacity():
    L = W.config_seq_lens("mixed")
    a = oracle.plan(L, 8, 256, 592)
    b = oracle.plan(L, 8, 256, 592)
    assert all(np.array_equal(a[x], b[x]) for x in ("bin_off", "units", "pair_off"))
    assert oracle.plan(L, 8, 256, 592, capacity=a["n_units"] - 1) is None
