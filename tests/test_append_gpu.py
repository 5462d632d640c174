"""Fused decode pre-processing on the GPU (rotary embedding of the new q / k rows and the append
of the new K/V rows into their pages) against the fp64 oracle, through the C ABI.

Rotated values may differ from the oracle's nearest bf16 by one bf16 unit in the last place (the
kernel rotates in fp32); every other byte of the pools must be untouched, and attention over the
appended cache must meet the decode tolerances (out 2e-3, lse 1e-4).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_29_b200 as da
import workloads as W
from tests import _gpu as U

pytestmark = pytest.mark.gpu


def _problem(seq_lens, *, Hq=8, Hkv=2, d=128, P=16, T=1, seed=5, tl=64, pool=None):
    return W.make_problem(name="append", batch=len(seq_lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                          seq_lens=seq_lens, page_size=P, q_tokens=T, kv_dtype="bf16", seed=seed, tile_len=tl,
                          pool_pages=pool)


def _bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _within_one_ulp(got_bits, want_bits):
    """|got - want| <= one bf16 ulp of want (8 significant bits), elementwise."""
    g, w = _bits_to_f64(got_bits), _bits_to_f64(want_bits)
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(w), 2.0 ** -126))[1] - 8)
    return np.abs(g - w) <= ulp


def _to_dev_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _from_dev_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _run_append(pr, q_new, k_new, v_new, *, in_place=False, status=None, table=None):
    tab = torch.from_numpy(np.ascontiguousarray(pr.page_table if table is None else table)).cuda()
    lens = torch.from_numpy(pr.seq_lens.astype(np.int32)).cuda()
    kp, vp = _to_dev_bits(pr.k_pages), _to_dev_bits(pr.v_pages)
    qn, kn, vn = _to_dev_bits(q_new), _to_dev_bits(k_new), _to_dev_bits(v_new)
    q_out = da.append_rope(qn, kn, vn, tab, lens, kp, vp, q_out=qn if in_place else None, status=status)
    torch.cuda.synchronize()
    return q_out, kp, vp, tab, lens


def _check(pr, T):
    q_new, k_new, v_new = W.make_step_inputs(pr)
    q_out, kp, vp, _, _ = _run_append(pr, q_new, k_new, v_new)
    want_q, want_k, want_v, n = oracle.append_rope(q_new, k_new, v_new, pr.page_table, pr.seq_lens,
                                                   pr.k_pages, pr.v_pages)
    assert n >= 0
    assert _within_one_ulp(_from_dev_bits(q_out), want_q).all()
    got_k, got_v = _from_dev_bits(kp), _from_dev_bits(vp)
    changed = want_k != pr.k_pages  # slots the append rewrites (or the same bits by chance)
    assert _within_one_ulp(got_k, want_k).all()
    assert np.array_equal(got_v, want_v)
    # bytes the append must not touch: every slot except the new tokens' slots
    written = np.zeros(pr.k_pages.shape[:1] + pr.k_pages.shape[2:3], dtype=bool)  # [page][slot]
    for b in range(pr.batch):
        for t in range(T):
            pos = int(pr.seq_lens[b]) - T + t
            if pos >= 0:
                written[pr.page_table[b, pos // pr.page_size], pos % pr.page_size] = True
    keep = ~written[:, None, :, None] & np.ones_like(pr.k_pages, dtype=bool)
    assert np.array_equal(got_k[keep], pr.k_pages[keep])
    assert np.array_equal(got_v[keep], pr.v_pages[keep])
    assert not changed[keep].any()
    return q_out, kp, vp, (want_q, want_k, want_v)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G,T", [(1, 1), (4, 1), (8, 1), (4, 4), (2, 3)])
def test_append_rope_matches_oracle(d, G, T):
    # lengths put the new tokens at page starts, page ends, across a page boundary and in
    # requests shorter than T (tokens at negative positions have no slot)
    lens = [1, T, 16, 17, 31, 33, 300, 1000][: 8]
    pr = _problem(lens, Hq=2 * G, Hkv=2, d=d, T=T)
    _check(pr, T)


def test_append_rope_large_positions():
    # positions near 131072: the angle is formed in fp64, so the rotation stays within one ulp
    pr = _problem([131072, 131071, 65537], Hq=8, Hkv=2, d=128, P=64, T=2)
    _check(pr, 2)


def test_append_rope_in_place_and_status():
    pr = _problem([40, 70, 5], Hq=4, Hkv=2, d=128, T=2)
    q_new, k_new, v_new = W.make_step_inputs(pr)
    q_out, _, _, _, _ = _run_append(pr, q_new, k_new, v_new, in_place=True)
    want_q = oracle.append_rope(q_new, k_new, v_new, pr.page_table, pr.seq_lens, pr.k_pages, pr.v_pages)[0]
    assert _within_one_ulp(_from_dev_bits(q_out), want_q).all()
    # a bad page id: that token's K/V write is skipped and reported, the others land
    bad = pr.page_table.copy()
    bad[1, 4] = pr.num_pages + 3  # request 1 (70 tokens): its tokens 68, 69 sit in logical page 4
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    _, kp, _, _, _ = _run_append(pr, q_new, k_new, v_new, status=st, table=bad)
    assert int(st.item()) == da.EDEVICE
    want_k = oracle.append_rope(q_new, k_new, v_new, pr.page_table, pr.seq_lens, pr.k_pages, pr.v_pages)[1]
    pos = 38  # request 0's second new token
    page, slot = pr.page_table[0, pos // 16], pos % 16
    assert _within_one_ulp(_from_dev_bits(kp)[page, :, slot], want_k[page, :, slot]).all()


def test_decode_after_append_matches_oracle():
    pr = _problem([17, 300, 1000, 64], Hq=16, Hkv=2, d=128, T=2, tl=64)
    q_new, k_new, v_new = W.make_step_inputs(pr)
    q_out, kp, vp, tab, lens = _run_append(pr, q_new, k_new, v_new)
    pl = da.plan(lens, pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=int(pr.seq_lens.sum()))
    out, lse = da.run(q_out, kp, vp, tab, lens, pl, sm_scale=pr.sm_scale)
    assert da.read_status(pl) == da.OK
    want_q, want_k, want_v, _ = oracle.append_rope(q_new, k_new, v_new, pr.page_table, pr.seq_lens,
                                                   pr.k_pages, pr.v_pages)
    pr2 = W.Problem(**{**pr.__dict__, "q": want_q, "k_pages": want_k, "v_pages": want_v})
    ref_o, ref_l = oracle.decode(pr2)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "decode after append")


def test_append_plan_run_in_one_cuda_graph():
    pr = _problem([200, 513, 64], Hq=8, Hkv=2, d=128, T=1, tl=64)
    q_new, k_new, v_new = W.make_step_inputs(pr)
    tab = torch.from_numpy(pr.page_table).cuda()
    lens = torch.from_numpy(pr.seq_lens.astype(np.int32)).cuda()
    kp, vp = _to_dev_bits(pr.k_pages), _to_dev_bits(pr.v_pages)
    qn, kn, vn = _to_dev_bits(q_new), _to_dev_bits(k_new), _to_dev_bits(v_new)
    q_out = torch.empty_like(qn)
    total = int(pr.seq_lens.sum())
    pl = da.plan(lens, pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total)
    shape = da.make_shape(qn, kp, tab, da.KV_BF16)
    ws = torch.empty(da.workspace_bytes(shape, pl), dtype=torch.uint8, device="cuda")
    out = torch.empty(pr.batch, 1, pr.n_q_heads, pr.head_dim, device="cuda")
    lse = torch.empty(pr.batch, 1, pr.n_q_heads, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        da.append_rope(qn, kn, vn, tab, lens, kp, vp, q_out=q_out, stream=s)
        da.plan(lens, pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total, buf=pl.buf, stream=s)
        da.run(q_out, kp, vp, tab, lens, pl, sm_scale=pr.sm_scale, workspace=ws, out=out, lse=lse, stream=s)
    g.replay()
    torch.cuda.synchronize()
    want_q, want_k, want_v, _ = oracle.append_rope(q_new, k_new, v_new, pr.page_table, pr.seq_lens,
                                                   pr.k_pages, pr.v_pages)
    pr2 = W.Problem(**{**pr.__dict__, "q": want_q, "k_pages": want_k, "v_pages": want_v})
    ref_o, ref_l = oracle.decode(pr2)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "graph: append + plan + run")


# ---------------------------------------------------------------- E4M3 pages (dec_attn_append_rope_fp8)

def _fp8_problem(seq_lens, *, Hq=8, Hkv=2, d=128, P=16, T=1, seed=7):
    return W.make_problem(name="append_fp8", batch=len(seq_lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                          seq_lens=seq_lens, page_size=P, q_tokens=T, kv_dtype="fp8e4m3", seed=seed, tile_len=64)


def _run_append_fp8(pr, q_new, k_new, v_new, status=None, table=None):
    tab = torch.from_numpy(np.ascontiguousarray(pr.page_table if table is None else table)).cuda()
    lens = torch.from_numpy(pr.seq_lens.astype(np.int32)).cuda()
    kp = torch.from_numpy(np.ascontiguousarray(pr.k_pages)).cuda()
    vp = torch.from_numpy(np.ascontiguousarray(pr.v_pages)).cuda()
    sc = torch.from_numpy(np.ascontiguousarray(pr.kv_scales)).cuda()
    qn, kn, vn = _to_dev_bits(q_new), _to_dev_bits(k_new), _to_dev_bits(v_new)
    q_out = da.append_rope_fp8(qn, kn, vn, tab, lens, kp, vp, sc, status=status)
    torch.cuda.synchronize()
    return q_out, kp, vp, sc, tab, lens


def _e4m3_step(values, scale):
    """One E4M3 step (3 mantissa bits, subnormal step 2^-9) at each value's magnitude, times scale."""
    m = np.maximum(np.abs(values) / scale, 2.0 ** -6)
    return np.maximum(2.0 ** (np.floor(np.log2(m)) - 3), 2.0 ** -9) * scale


@pytest.mark.parametrize("T,P,d", [(1, 16, 128), (4, 16, 128), (8, 16, 64), (3, 32, 128), (8, 64, 128)])
def test_append_fp8_matches_oracle(T, P, d):
    # requests whose new tokens start a fresh page, continue a page (the scale may grow), span two
    # pages, and sit partly before position 0 (L < T)
    lens = [P * 3, P * 2 + 3, P + T + 5, max(T - 2, 1), 5 * P + P // 2]
    pr = _fp8_problem(lens, T=T, P=P, d=d, seed=T * 10 + P)
    q_new, k_new, v_new = W.make_step_inputs(pr)
    # scale the new rows up for half the requests, so that their pages' scales grow
    big = np.array([1, 0, 1, 0, 1], dtype=bool)[:, None, None, None]
    kf, vf = _bits_to_f64(k_new), _bits_to_f64(v_new)
    k_new = W.bf16_bits_from_f32(np.where(big, kf * 12, kf).astype(np.float32))
    v_new = W.bf16_bits_from_f32(np.where(big, vf * 12, vf).astype(np.float32))
    q_out, kp, vp, sc, tab, lens_d = _run_append_fp8(pr, q_new, k_new, v_new)
    want_q, want_k, want_v, want_sc = oracle.append_rope_fp8(q_new, k_new, v_new, pr.page_table, pr.seq_lens,
                                                             pr.k_pages, pr.v_pages, pr.kv_scales)
    assert np.all(_within_one_ulp(_from_dev_bits(q_out), want_q))
    got_k, got_v, got_sc = kp.cpu().numpy(), vp.cpu().numpy(), sc.cpu().numpy()
    # V: exact inputs, every rounding decision on the same fp32 numbers -> bit-exact codes and scales
    assert np.array_equal(got_v, want_v)
    assert np.array_equal(got_sc[1], want_sc[1])
    # K: rotated in fp32 on the GPU, exactly in the oracle -> scales within an fp32 unit, codes within one
    # E4M3 step (a rounding decision can flip only next to a tie), and almost all codes equal
    assert np.allclose(got_sc[0], want_sc[0], rtol=2.0 ** -22, atol=0)
    tabv = oracle.e4m3_table()
    gk = tabv[got_k] * got_sc[0][:, :, None, None]
    wk = tabv[want_k] * want_sc[0][:, :, None, None]
    assert np.all(np.abs(gk - wk) <= _e4m3_step(wk, want_sc[0][:, :, None, None]) * (1 + 1e-6))
    assert np.mean(got_k != want_k) < 1e-3
    # decode over the appended cache (its own values) meets the decode tolerances
    pr2 = W.Problem(**{**pr.__dict__, "q": _from_dev_bits(q_out), "k_pages": got_k, "v_pages": got_v,
                       "kv_scales": got_sc})
    out, lse, _, st = U.run_problem(pr2)
    assert st == da.OK
    ref_o, ref_l = oracle.decode(pr2)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, f"decode after FP8 append T{T} P{P} d{d}")


def test_append_fp8_bad_page_id_reports_and_skips_the_page():
    pr = _fp8_problem([40, 70], T=2)
    q_new, k_new, v_new = W.make_step_inputs(pr)
    table = pr.page_table.copy()
    table[1, (70 - 2) // 16] = pr.num_pages + 3
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    q_out, kp, vp, sc, _, _ = _run_append_fp8(pr, q_new, k_new, v_new, status=st, table=table)
    assert int(st.item()) == da.EDEVICE
    # request 0's page was written as the oracle writes it; every page of request 1 is unchanged
    _, want_k, _, _ = oracle.append_rope_fp8(q_new, k_new, v_new, pr.page_table, pr.seq_lens, pr.k_pages,
                                             pr.v_pages, pr.kv_scales)
    got_k = kp.cpu().numpy()
    pid0 = int(pr.page_table[0, (40 - 2) // 16])
    assert np.mean(got_k[pid0] != want_k[pid0]) < 1e-3
    for p_ in pr.page_table[1, :(70 + 15) // 16]:
        assert np.array_equal(got_k[p_], pr.k_pages[p_])
