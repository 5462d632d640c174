"""Pins of the variable-length oracle (oracle.decode_varlen: request b's q_lens[b] query rows are its
last q_lens[b] positions, "PaddlePaddle/HALOps" README, Highlights, GQA attention item: variable-length
prefill), checked against what fixes it independently:
  * torch SDPA in float64 per request on the gathered dense K/V with the bottom-right causal mask,
    the rows taken from the packed q by the offsets;
  * equal row counts: the varlen oracle is the uniform oracle row for row (same arithmetic);
  * a request with no rows contributes nothing; rows before position 0 see no key (out 0, lse -inf).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import _helpers as H


def _varlen(seq_lens, q_lens, *, Hq=4, Hkv=2, d=64, P=16, kv="bf16", seed=5):
    return W.make_varlen_problem(batch=len(seq_lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                                 seq_lens=seq_lens, q_lens=q_lens, page_size=P, kv_dtype=kv, seed=seed, tile_len=64)


def _sdpa_varlen(pr):
    G = pr.group
    q = W.bf16_bits_to_f32(pr.q).astype(np.float64)   # [total][Hq][d]
    outs, lses = [], []
    for b in range(pr.batch):
        lo, hi = int(pr.cu_q[b]), int(pr.cu_q[b + 1])
        Tb, Lb = hi - lo, int(pr.seq_lens[b])
        if Tb == 0:
            continue
        K = torch.from_numpy(H.dense_kv(pr, b, "k")).repeat_interleave(G, 0)   # [Hq][Lb][d]
        V = torch.from_numpy(H.dense_kv(pr, b, "v")).repeat_interleave(G, 0)
        Q = torch.from_numpy(q[lo:hi].transpose(1, 0, 2).copy())             # [Hq][Tb][d]
        mask = torch.arange(Lb)[None, :] <= (Lb - Tb + torch.arange(Tb)[:, None])
        s = (Q @ K.transpose(1, 2)) * pr.sm_scale
        s = s.masked_fill(~mask, float("-inf"))
        lse = torch.logsumexp(s, dim=-1)                                      # [Hq][Tb]
        w = torch.softmax(s, dim=-1).nan_to_num(0.0)
        outs.append((w @ V).transpose(0, 1).numpy())
        lses.append(lse.transpose(0, 1).numpy())
    return np.concatenate(outs), np.concatenate(lses)


@pytest.mark.parametrize("seq_lens,q_lens,kw", [
    ([40, 300, 129, 77], [40, 17, 1, 90], {}),                    # one request with T > L
    ([200, 0, 64, 500], [3, 0, 64, 128], dict(Hq=8, Hkv=2)),      # an empty request, T = L
    ([130, 260], [0, 200], dict(d=128, P=32)),
    ([90, 90, 90], [5, 0, 91], dict(kv="fp8e4m3", d=128)),
])
def test_varlen_oracle_matches_torch_sdpa(seq_lens, q_lens, kw):
    pr = _varlen(seq_lens, q_lens, **kw)
    out, lse = oracle.decode_varlen(pr)
    assert out.shape == (sum(q_lens), pr.n_q_heads, pr.head_dim)
    ref_o, ref_l = _sdpa_varlen(pr)
    empty = np.isneginf(ref_l)
    assert np.array_equal(np.isneginf(lse), empty)
    assert np.all(out[empty] == 0)
    np.testing.assert_allclose(out[~empty], ref_o[~empty], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[~empty], ref_l[~empty], rtol=0, atol=1e-12)


def test_equal_row_counts_reduce_to_the_uniform_oracle():
    seq_lens, T = [33, 200, 129], 9
    pr_v = _varlen(seq_lens, [T] * 3, Hq=8, Hkv=2)
    pr_u = W.make_problem(batch=3, n_q_heads=8, n_kv_heads=2, head_dim=64, seq_lens=seq_lens, q_tokens=T,
                          page_size=16, kv_dtype="bf16", seed=5, tile_len=64)
    assert np.array_equal(pr_v.q, pr_u.q.reshape(-1, 8, 64))   # the same rows, packed
    o_v, l_v = oracle.decode_varlen(pr_v)
    o_u, l_u = oracle.decode(pr_u)
    assert np.array_equal(o_v, o_u.reshape(-1, 8, 64)) and np.array_equal(l_v, l_u.reshape(-1, 8))


def test_rows_before_position_zero_see_nothing():
    pr = _varlen([3, 10], [5, 2])
    out, lse = oracle.decode_varlen(pr)
    # request 0: rows 0, 1 sit at positions -2, -1
    assert np.all(np.isneginf(lse[:2])) and np.all(out[:2] == 0)
    assert np.all(np.isfinite(lse[2:]))
