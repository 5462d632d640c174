"""FP8-products mode (KV_FP8E4M3_MMA8) on the GPU: E4M3 pages with both products on E4M3 tensor
cores, q rounded to one E4M3 part per row and P rounded to E4M3 (the HPC-Ops article at
sdftguanye.com, section on fine-grained task scheduling and data rearrangement: an FP8 attention
kernel). Judged against the fp64 oracle run on the rounded q
(oracle.round_q_e4m3_rows), with its own tolerance:
  * lse within 1e-4 (the scores use the rounded q exactly; P's rounding does not enter lse);
  * out, per element: P = p * (V page scale) * C is rounded to E4M3, a relative error d_j of at
    most 2^-4 on each weight in E4M3's normal range; the row sums take the rounded weights, so the
    output is sum_j w_j (1 + d_j) v_j / sum_j w_j (1 + d_j) and
    |out - ref| <= (2^-3 / (1 - 2^-4)) * max_j |v_j - ref| over the row's visible keys, plus 1e-3
    for weights in E4M3's subnormal range (below 2^-6 after scaling);
  * out, per row: with a_j = w_j / W the row's softmax weights (from the oracle) and m_j the mean over
    head dims of (v_j - ref)^2, the row's error is sum_j a_j d_j (v_j - ref) / (1 + sum_j a_j d_j);
    random V rows have nearly orthogonal deviations, so its RMS over head dims is about
    2^-4 sqrt(sum_j a_j^2 m_j) at most; the test allows twice that (for the cross terms) plus 2e-4
    (subnormal weights);
  * out, over all elements: RMS error below 4e-3 (independent rounding errors average out; a
    wrong operand layout gives errors of order |v|).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_29_b200 as da
import workloads as W
from tests import _gpu as U
from tests import _helpers as H

pytestmark = pytest.mark.gpu


def _problem(lens, *, Hq, Hkv=2, T=1, seed=13, tl=512):
    return W.make_problem(name="mma8", batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                          seq_lens=lens, page_size=16, q_tokens=T, kv_dtype="fp8e4m3", seed=seed, tile_len=tl)


def _run(pr):
    dev = U.to_device(pr)
    total = int(pr.seq_lens.astype(np.int64).sum())
    pl = da.plan(dev["lens"], pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total)
    out, lse = da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"],
                      sm_scale=pr.sm_scale, mma8=True)
    return out.cpu().numpy(), lse.cpu().numpy(), da.read_status(pl)


def _row_stats(pr, rows, ref_o):
    """Per (b, t, qh) row: max_j |v_j - ref| over the row's visible keys j and all head dims, and
    sqrt(sum_j a_j^2 m_j) with a_j the oracle's softmax weights and m_j = mean_c (v_jc - ref_c)^2.
    The maximum uses running maxima / minima of V over the keys (one pass per (request, KV head))."""
    from concurrent.futures import ThreadPoolExecutor
    vdev = np.zeros(len(rows))
    wdev = np.zeros(len(rows))
    # the oracle's weights of every row, on all cores (the C oracle runs without the GIL)
    with ThreadPoolExecutor(max(1, oracle.max_threads())) as ex:
        weights = list(ex.map(lambda r: oracle.attend(pr, int(r[0]), int(r[1]), int(r[2]), weights=True)[3], rows))
    by_pair = {}
    for i, (b, t, qh) in enumerate(rows):
        by_pair.setdefault((int(b), int(qh) // pr.group), []).append(i)
    cache_b, cache_v = None, None
    for (b, h), idx in sorted(by_pair.items()):
        if b != cache_b:
            cache_b, cache_v = b, H.dense_kv(pr, b, "v")
        V = cache_v[h]                                # [L][d]
        if V.shape[0] == 0:
            continue
        vmax = np.maximum.accumulate(V, axis=0)
        vmin = np.minimum.accumulate(V, axis=0)
        n2 = np.einsum("jc,jc->j", V, V)
        for i in idx:
            _, t, qh = rows[i]
            vis = int(pr.seq_lens[b]) - pr.q_tokens + int(t) + 1
            if vis <= 0:
                continue
            ref = ref_o[i]
            vdev[i] = max(float(np.max(vmax[vis - 1] - ref)), float(np.max(ref - vmin[vis - 1])))
            w = weights[i]
            n = w.shape[0]
            a2 = w * w
            d = pr.head_dim
            # sum_j a_j^2 mean_c (v_jc - ref_c)^2 = sum_j a_j^2 (|v_j|^2 - 2 v_j.ref + |ref|^2) / d
            s = (a2 @ n2[:n] - 2.0 * (a2 @ V[:n]) @ ref + a2.sum() * (ref @ ref)) / d
            wdev[i] = np.sqrt(max(s, 0.0))
    return vdev, wdev


def _check(pr, out, lse, ref_o, ref_l, rows, what):
    """pr: the problem with the rounded q (the oracle's weights are those of the rounded scores)."""
    both_empty = np.isneginf(lse) & np.isneginf(ref_l)
    assert np.all(both_empty | (np.abs(lse - ref_l) <= 1e-4)), what
    vdev, wdev = _row_stats(pr, rows, ref_o)
    bound = 2.0 ** -3 / (1 - 2.0 ** -4) * vdev[:, None] + 1e-3
    err = np.abs(out - ref_o)
    rms = float(np.sqrt(np.mean(err ** 2)))
    row_rms = np.sqrt(np.mean(err ** 2, axis=1))
    row_bound = 2.0 ** -3 * wdev + 2e-4
    print(f"{what}: max err {err.max():.2e}, rms {rms:.2e}, max err / bound {np.max(err / bound):.3f}, "
          f"max row rms / row bound {np.max(row_rms / row_bound):.3f}")
    assert np.all(err <= bound), what
    assert np.all(row_rms <= row_bound), what
    assert rms < 4e-3, what


@pytest.mark.parametrize("G,T", [(1, 1), (4, 1), (8, 1), (16, 1), (4, 4), (2, 3)])
def test_mma8_matches_oracle_on_rounded_q(G, T):
    pr = _problem([1, 40, 300, 1000, 2049, 4100], Hq=2 * G, T=T)
    out, lse, st = _run(pr)
    assert st == da.OK, da.status_string(st)
    pr_q = W.Problem(**{**pr.__dict__, "q": oracle.round_q_e4m3_rows(pr.q)})
    ref_o, ref_l = oracle.decode(pr_q)
    B, Tn, Hq = lse.shape
    rows = [(b, t, qh) for b in range(B) for t in range(Tn) for qh in range(Hq)]
    _check(pr_q, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           f"mma8 G{G} T{T}")


def test_mma8_full_size_fp8_spec_all_rows():
    pr = W.make_config("fp8_spec")
    out, lse, st = _run(pr)
    assert st == da.OK, da.status_string(st)
    pr_q = W.Problem(**{**pr.__dict__, "q": oracle.round_q_e4m3_rows(pr.q)})
    ref_o, ref_l = oracle.decode(pr_q)
    B, Tn, Hq = lse.shape
    rows = [(b, t, qh) for b in range(B) for t in range(Tn) for qh in range(Hq)]
    _check(pr_q, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           "mma8 fp8_spec, every row")


def test_mma8_needs_head_dim_128():
    pr = W.make_problem(name="mma8", batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, seq_lens=[100, 30],
                        page_size=16, q_tokens=1, kv_dtype="fp8e4m3", seed=3, tile_len=64)
    dev = U.to_device(pr)
    pl = da.plan(dev["lens"], 2, 64, max_total_kv_tokens=130)
    with pytest.raises(da.DecAttnError):
        da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"], mma8=True)
