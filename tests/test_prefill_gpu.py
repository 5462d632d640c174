"""Prefill on the GPU (dec_attn_prefill: the T query rows of each request, its last T positions,
over its paged bf16 KV with the bottom-right causal rule; dec_attn_prefill_varlen: a different
number of rows per request, packed; "PaddlePaddle/HALOps" README, Highlights, GQA attention item:
variable-length prefill) against the fp64 oracle, which computes the same attention for any
number of query rows (oracle.decode, oracle.decode_varlen).

Tolerance, derived from the kernel's arithmetic: scores are exact products of bf16 q and K summed
in fp32 (lse within 1e-4); P is rounded once to bf16 for P V (relative error at most 2^-9 per
weight) while the row sums stay in fp32, so out = sum_j w_j (1 + d_j) v_j with |d_j| <= 2^-9 and
|out - ref| <= 2^-9 * max_j |v_j| over the row's visible keys (plus 1e-5 for fp32 accumulation).
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


def _problem(lens, *, T, Hq=4, Hkv=2, P=16, seed=17):
    return W.make_problem(name="prefill", batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                          seq_lens=lens, page_size=P, q_tokens=T, kv_dtype="bf16", seed=seed, tile_len=max(P, 64))


def _run(pr):
    dev = U.to_device(pr)
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    out, lse = da.prefill(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], sm_scale=pr.sm_scale, status=st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy(), int(st.item())


def _vmax(pr, rows, T_of=None):
    """max_j |v_j| over each (b, t, qh) row's visible keys and all head dims (running maxima of
    |V| over the keys, one pass per (request, KV head)). T_of[b]: request b's query rows (default:
    the problem's q_tokens)."""
    res = np.zeros(len(rows))
    by_pair = {}
    for i, (b, t, qh) in enumerate(rows):
        by_pair.setdefault((int(b), int(qh) // pr.group), []).append(i)
    cache_b, cache_v = None, None
    for (b, h), idx in sorted(by_pair.items()):
        if b != cache_b:
            cache_b, cache_v = b, H.dense_kv(pr, b, "v")
        run = np.maximum.accumulate(np.abs(cache_v[h]).max(axis=1)) if cache_v.shape[1] else None
        Tb = pr.q_tokens if T_of is None else int(T_of[b])
        for i in idx:
            vis = int(pr.seq_lens[b]) - Tb + int(rows[i][1]) + 1
            res[i] = run[vis - 1] if vis > 0 else 0.0
    return res


def _check(pr, out, lse, ref_o, ref_l, rows, what, T_of=None):
    both_empty = np.isneginf(lse) & np.isneginf(ref_l)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_l)), what
    assert np.all(both_empty | (np.abs(lse - ref_l) <= 1e-4)), what
    err = np.abs(out - ref_o)
    bound = 2.0 ** -9 * _vmax(pr, rows, T_of)[:, None] + 1e-5
    print(f"{what}: max err {err.max():.2e}, max err / bound {np.max(err / bound):.3f}")
    assert np.all(err <= bound), what


@pytest.mark.parametrize("lens,T,Hq,Hkv,P", [
    ([300, 700], 200, 4, 2, 16),     # two query blocks, partial last one
    ([129, 1000], 1, 8, 2, 16),      # one query row (a decode through the prefill path)
    ([256, 256], 256, 2, 2, 64),     # pure prefill: T = L, two whole blocks
    ([90, 400, 131], 130, 8, 1, 16), # T > L for one request (its first rows see nothing), G = 8
    ([513], 385, 4, 4, 32),          # keys and rows not multiples of the block
    ([700, 333], 300, 6, 2, 16),     # G = 3: adjacent row blocks paired, the last pair's second past T
    ([900, 640], 640, 64, 8, 16),    # 320 tile pairs: more than one per CTA on any current GPU
])
def test_prefill_matches_oracle(lens, T, Hq, Hkv, P):
    pr = _problem(lens, T=T, Hq=Hq, Hkv=Hkv, P=P)
    out, lse, st = _run(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    B = len(lens)
    rows = [(b, t, qh) for b in range(B) for t in range(T) for qh in range(Hq)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           f"prefill L{lens} T{T} G{Hq // Hkv} P{P}")


def test_prefill_full_size_all_rows():
    pr = W.make_config("prefill")
    out, lse, st = _run(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    B, T, Hq = lse.shape
    rows = [(b, t, qh) for b in range(B) for t in range(T) for qh in range(Hq)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           "prefill full size, every row")


def _varlen(lens, q_lens, *, Hq=4, Hkv=2, P=16, seed=23):
    return W.make_varlen_problem(batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128, seq_lens=lens,
                                 q_lens=q_lens, page_size=P, kv_dtype="bf16", seed=seed, tile_len=max(P, 64))


def _run_varlen(pr, guard=0):
    """Runs dec_attn_prefill_varlen with `guard` extra rows after the packed output (canaries)."""
    dev = U.to_device(pr)
    cu = torch.from_numpy(pr.cu_q).cuda()
    total = int(pr.cu_q[-1])
    out_buf = torch.full((total + guard, pr.n_q_heads, 128), 7.0, device="cuda")
    lse_buf = torch.full((total + guard, pr.n_q_heads), 7.0, device="cuda")
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    da.prefill_varlen(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], cu, pr.q_tokens, sm_scale=pr.sm_scale,
                      out=out_buf[:total], lse=lse_buf[:total], status=st)
    torch.cuda.synchronize()
    o, l = out_buf.cpu().numpy(), lse_buf.cpu().numpy()
    assert np.all(o[total:] == 7.0) and np.all(l[total:] == 7.0), "rows past the packed output were written"
    return o[:total], l[:total], int(st.item())


@pytest.mark.parametrize("lens,q_lens,Hq,Hkv,P", [
    ([300, 700, 129, 64], [200, 1, 129, 64], 4, 2, 16),      # ragged blocks, T = 1, T = L
    ([513, 90, 1000], [385, 130, 0], 8, 1, 16),              # T > L for one request, an empty request, G = 8
    ([700, 333, 260, 1], [300, 33, 256, 1], 6, 2, 32),       # G = 3: adjacent row blocks paired
    ([2048, 100, 4096, 640], [31, 100, 257, 640], 16, 2, 64),
])
def test_prefill_varlen_matches_oracle(lens, q_lens, Hq, Hkv, P):
    pr = _varlen(lens, q_lens, Hq=Hq, Hkv=Hkv, P=P)
    out, lse, st = _run_varlen(pr, guard=40)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode_varlen(pr)
    rows = [(b, t, qh) for b in range(pr.batch) for t in range(q_lens[b]) for qh in range(Hq)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           f"prefill varlen L{lens} T{q_lens} G{Hq // Hkv} P{P}", T_of=q_lens)


def test_prefill_varlen_equal_counts_is_the_uniform_kernel_bit_for_bit():
    lens, T = [300, 777, 129], 150
    pr = _varlen(lens, [T] * 3, Hq=8, Hkv=2)
    out_v, lse_v, st = _run_varlen(pr)
    assert st == da.OK
    pr_u = _problem(lens, T=T, Hq=8, Hkv=2, seed=23)
    assert np.array_equal(pr_u.q.reshape(-1, 8, 128), pr.q)
    out_u, lse_u, st_u = _run(pr_u)
    assert st_u == da.OK
    assert np.array_equal(out_u.reshape(-1, 8, 128), out_v) and np.array_equal(lse_u.reshape(-1, 8), lse_v)


def test_prefill_varlen_full_size_mixed_rows_all_rows():
    # the prefill workload's four 2048-token prompts with different numbers of new rows
    q_lens = [2048, 1000, 129, 1777]
    c = W.CONFIGS["prefill"]
    pr = W.make_varlen_problem(name="prefill_varlen", batch=4, n_q_heads=c["n_q_heads"], n_kv_heads=c["n_kv_heads"],
                               head_dim=128, seq_lens=W.config_seq_lens("prefill"), q_lens=q_lens, page_size=16,
                               kv_dtype="bf16", seed=c["seed"], tile_len=256)
    out, lse, st = _run_varlen(pr, guard=8)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode_varlen(pr)
    rows = [(b, t, qh) for b in range(4) for t in range(q_lens[b]) for qh in range(pr.n_q_heads)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           "prefill varlen full size, every row", T_of=q_lens)


def test_prefill_varlen_bad_offsets_are_reported():
    pr = _varlen([300, 200], [100, 50])
    pr.cu_q = np.array([0, 100, 160], dtype=np.int32)   # past the 150 packed rows
    dev = U.to_device(pr)
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    out = torch.zeros((150, 4, 128), device="cuda")
    lse = torch.zeros((150, 4), device="cuda")
    da.prefill_varlen(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], torch.from_numpy(pr.cu_q).cuda(), 100,
                      out=out, lse=lse, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == da.EDEVICE
    assert torch.all(out[100:] == 0)   # the request with bad offsets is not written


def test_prefill_bad_page_id_is_reported():
    pr = _problem([300, 200], T=100)
    tab = pr.page_table.copy()
    tab[1, 3] = pr.num_pages + 5
    pr2 = W.Problem(**{**pr.__dict__, "page_table": tab})
    _, _, st = _run(pr2)
    assert st == da.EDEVICE


def test_prefill_rejects_unsupported_shapes():
    pr = W.make_problem(name="p", batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64, seq_lens=[100], page_size=16,
                        q_tokens=10, kv_dtype="bf16", seed=1, tile_len=64)
    dev = U.to_device(pr)
    with pytest.raises(da.DecAttnError):
        da.prefill(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"])
