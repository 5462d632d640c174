"""Prefill over an FP8 (E4M3) KV cache on the GPU (dec_attn_prefill_fp8: "PaddlePaddle/HALOps"
README, Highlights, GQA attention item: prefill and paged-KV decode across BF16 / FP8 KV caches)
against the fp64 oracle over the dequantised cache, K = code * scale and V likewise
(oracle.decode, oracle.decode_varlen).

Tolerance, derived from the path's arithmetic. The widening pass hands the bf16 prefill kernel
K' = RN_bf16(RN_fp32(k)) and V' likewise: |k' - k| <= e |k| per element with e = 2^-9 (1 + 2^-14).
A score then moves by |ds_j| = sm_scale |sum_i q_i (k'_ji - k_ji)| <= sm_scale e |q|_2 |k_j|_2 (Cauchy-
Schwarz) =: eps over the row's visible keys, so every softmax weight changes by a factor within
e^(+-2 eps) and lse by at most eps. With P rounded once to bf16 (2^-9) and V' (e), a row's output
is sum_j w_j (1 + c_j) v_j with |c_j| <= e^(2 eps) (1 + 2^-9) (1 + e) - 1, so
|out - ref| <= max_j |v_j| (e^(2 eps) (1 + 2^-9)(1 + e) - 1) + 1e-5 and |lse - ref| <= eps + 1e-4.
A second test pins the widening itself: the FP8 path's output equals, bit for bit, the bf16
prefill over a bf16 pool holding RN_bf16(RN_fp32(code * scale)) computed on the host.
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

E = 2.0 ** -9 * (1 + 2.0 ** -14)   # relative error of a widened element


def _problem(lens, *, T, Hq=4, Hkv=2, P=16, seed=31):
    return W.make_problem(name="prefill_fp8", batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                          seq_lens=lens, page_size=P, q_tokens=T, kv_dtype="fp8e4m3", seed=seed,
                          tile_len=max(P, 64))


def _varlen(lens, q_lens, *, Hq=4, Hkv=2, P=16, seed=37):
    return W.make_varlen_problem(batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128, seq_lens=lens,
                                 q_lens=q_lens, page_size=P, kv_dtype="fp8e4m3", seed=seed, tile_len=max(P, 64))


def _run(pr, varlen=False, ws_guard=True):
    dev = U.to_device(pr)
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    cu = torch.from_numpy(pr.cu_q).cuda() if varlen else None
    need = da.prefill_fp8_workspace_bytes(dev["q"].shape, dev["k"], dev["tab"], pr.q_tokens)
    whole, ws = U._guarded(need, "cuda")
    out, lse = da.prefill_fp8(dev["q"], dev["k"], dev["v"], dev["sc"], dev["tab"], dev["lens"], cu_q_lens=cu,
                              max_q_rows=pr.q_tokens, sm_scale=pr.sm_scale, workspace=ws, status=st)
    torch.cuda.synchronize()
    if ws_guard:
        U.check_canaries(whole)
    return out.cpu().numpy(), lse.cpu().numpy(), int(st.item())


def _row_bounds(pr, rows, T_of=None):
    """Per (b, t, qh) row: eps = sm_scale * E * |q|_2 * max |k_j|_2 and max |v_j| over the row's
    visible keys (running maxima over the keys, one pass per (request, KV head))."""
    q = H.q_values(pr).reshape(-1, pr.n_q_heads, pr.head_dim)   # rows packed: (b, t) -> b * T + t, or cu_q
    eps = np.zeros(len(rows))
    vmax = np.zeros(len(rows))
    by_pair = {}
    for i, (b, t, qh) in enumerate(rows):
        by_pair.setdefault((int(b), int(qh) // pr.group), []).append(i)
    cache_b = None
    for (b, h), idx in sorted(by_pair.items()):
        if b != cache_b:
            cache_b, k, v = b, H.dense_kv(pr, b, "k"), H.dense_kv(pr, b, "v")
        kn = np.maximum.accumulate(np.linalg.norm(k[h], axis=1)) if k.shape[1] else None
        vm = np.maximum.accumulate(np.abs(v[h]).max(axis=1)) if v.shape[1] else None
        Tb = pr.q_tokens if T_of is None else int(T_of[b])
        base = int(pr.cu_q[b]) if T_of is not None else b * pr.q_tokens
        for i in idx:
            t, qh = int(rows[i][1]), int(rows[i][2])
            vis = int(pr.seq_lens[b]) - Tb + t + 1
            if vis > 0:
                eps[i] = pr.sm_scale * E * np.linalg.norm(q[base + t, qh]) * kn[vis - 1]
                vmax[i] = vm[vis - 1]
    return eps, vmax


def _check(pr, out, lse, ref_o, ref_l, rows, what, T_of=None):
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_l)), what
    eps, vmax = _row_bounds(pr, rows, T_of)
    fin = ~np.isneginf(ref_l)
    lerr = np.abs(lse[fin] - ref_l[fin])
    assert np.all(lerr <= eps[fin] + 1e-4), what
    err = np.abs(out - ref_o)
    bound = (vmax * (np.exp(2 * eps) * (1 + 2.0 ** -9) * (1 + E) - 1))[:, None] + 1e-5
    print(f"{what}: max err {err.max():.2e}, max err / bound {np.max(err / bound):.3f}, "
          f"max lse err {lerr.max() if lerr.size else 0:.2e}")
    assert np.all(err <= bound), what


@pytest.mark.parametrize("lens,T,Hq,Hkv,P", [
    ([300, 700], 200, 4, 2, 16),     # two query blocks, partial last one
    ([129, 1000], 1, 8, 2, 16),      # one query row
    ([256, 256], 256, 2, 2, 64),     # T = L, two whole blocks
    ([90, 400, 131], 130, 8, 1, 16), # T > L for one request, G = 8
    ([700, 333], 300, 6, 2, 32),     # G = 3
])
def test_prefill_fp8_matches_oracle(lens, T, Hq, Hkv, P):
    pr = _problem(lens, T=T, Hq=Hq, Hkv=Hkv, P=P)
    out, lse, st = _run(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    rows = [(b, t, qh) for b in range(len(lens)) for t in range(T) for qh in range(Hq)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           f"prefill fp8 L{lens} T{T} G{Hq // Hkv} P{P}")


@pytest.mark.parametrize("lens,q_lens,Hq,Hkv,P", [
    ([300, 700, 129, 64], [200, 1, 129, 64], 4, 2, 16),
    ([513, 90, 1000], [385, 130, 0], 8, 1, 16),
])
def test_prefill_fp8_varlen_matches_oracle(lens, q_lens, Hq, Hkv, P):
    pr = _varlen(lens, q_lens, Hq=Hq, Hkv=Hkv, P=P)
    out, lse, st = _run(pr, varlen=True)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode_varlen(pr)
    rows = [(b, t, qh) for b in range(pr.batch) for t in range(q_lens[b]) for qh in range(Hq)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           f"prefill fp8 varlen L{lens} T{q_lens}", T_of=q_lens)


def test_prefill_fp8_full_size_all_rows():
    c = W.CONFIGS["prefill"]
    pr = _problem(W.config_seq_lens("prefill"), T=c["q_tokens"], Hq=c["n_q_heads"], Hkv=c["n_kv_heads"],
                  P=c["page_size"], seed=c["seed"])
    out, lse, st = _run(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    B, T, Hq = lse.shape
    rows = [(b, t, qh) for b in range(B) for t in range(T) for qh in range(Hq)]
    _check(pr, out.reshape(-1, 128), lse.reshape(-1), ref_o.reshape(-1, 128), ref_l.reshape(-1), rows,
           "prefill fp8 full size, every row")


def test_prefill_fp8_is_the_bf16_prefill_over_the_widened_values_bit_for_bit():
    pr = _problem([300, 777, 129], T=150, Hq=8, Hkv=2)
    out8, lse8, st = _run(pr)
    assert st == da.OK
    # the widening on the host: RN_fp32(code * scale), then RN_bf16 (torch's float -> bfloat16 is RNE)
    codes = {w: torch.from_numpy(np.ascontiguousarray(getattr(pr, w))).view(torch.float8_e4m3fn).float()
             for w in ("k_pages", "v_pages")}
    sc = torch.from_numpy(np.ascontiguousarray(pr.kv_scales))     # [2][num_pages][Hkv]
    wide = {w: (codes[w] * sc[i][:, :, None, None]).to(torch.bfloat16) for i, w in enumerate(("k_pages", "v_pages"))}
    dev = U.to_device(pr)
    st16 = torch.zeros((), dtype=torch.int32, device="cuda")
    out16, lse16 = da.prefill(dev["q"], wide["k_pages"].cuda(), wide["v_pages"].cuda(), dev["tab"], dev["lens"],
                              sm_scale=pr.sm_scale, status=st16)
    torch.cuda.synchronize()
    assert int(st16.item()) == da.OK
    assert np.array_equal(out8, out16.cpu().numpy()) and np.array_equal(lse8, lse16.cpu().numpy())


def test_prefill_fp8_bad_page_id_is_reported():
    pr = _problem([300, 200], T=100)
    tab = pr.page_table.copy()
    tab[1, 3] = pr.num_pages + 5
    pr2 = W.Problem(**{**pr.__dict__, "page_table": tab})
    _, _, st = _run(pr2)
    assert st == da.EDEVICE


def test_prefill_fp8_small_workspace_is_refused():
    pr = _problem([300], T=10)
    dev = U.to_device(pr)
    need = da.prefill_fp8_workspace_bytes(dev["q"].shape, dev["k"], dev["tab"], pr.q_tokens)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(da.DecAttnError) as e:
        da.prefill_fp8(dev["q"], dev["k"], dev["v"], dev["sc"], dev["tab"], dev["lens"], workspace=ws)
    assert e.value.code == da.ESMALL
