"""Pins of the FP8 append oracle (oracle.append_rope_fp8: rotary embedding of the new q / k rows and
their append to an E4M3 paged cache whose scale per (page, KV head) covers the page's valid rows),
checked against what fixes it independently:
  * a page that starts with the new rows gets exactly the encoding of the pages' FP8 reading
    (scale = absmax / 448, codes = round-to-nearest-even of x / scale), the workload generator's
    encoder, itself pinned against a brute-force nearest search;
  * old rows keep their codes when the scale need not grow, and move by at most half a step of the
    new scale when it grows; new rows decode to within half a step of their values;
  * q is rotated exactly as the bf16 append oracle rotates it; rows at positions < 0 get no slot.
"""
import numpy as np
import pytest

import oracle
import workloads as W


def _fp8_problem(lens, T, *, Hq=4, Hkv=2, d=64, P=16, seed=41):
    pr = W.make_problem(name="fp8app", batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_lens=lens,
                        page_size=P, q_tokens=T, kv_dtype="fp8e4m3", seed=seed, tile_len=64)
    qn, kn, vn = W.make_step_inputs(pr)
    return pr, qn, kn, vn


def _f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _run(pr, qn, kn, vn):
    return oracle.append_rope_fp8(qn, kn, vn, pr.page_table, pr.seq_lens, pr.k_pages, pr.v_pages, pr.kv_scales)


def test_fresh_pages_get_the_encoding_reading():
    # L - T a multiple of P: every new row starts or continues a page with no older row
    pr2, qn, kn, vn = _fp8_problem([32 + 8, 16 + 8], 8, P=16)
    q_out, kc, vc, sc = _run(pr2, qn, kn, vn)
    for b in range(2):
        L = int(pr2.seq_lens[b])
        pid = int(pr2.page_table[b, (L - 8) // 16])
        for h in range(2):
            x_v = _f64(vn[b, :, h]).astype(np.float32)
            x_k = oracle.rope_rows(_f64(kn[b, :, h]), np.arange(L - 8, L)).astype(np.float32)
            for which, x, codes in ((0, x_k, kc), (1, x_v, vc)):
                s = np.float32(np.abs(x).max()) / np.float32(448)
                assert sc[which, pid, h] == s
                assert np.array_equal(codes[pid, h, :8], W.e4m3_encode(x / s))


@pytest.mark.parametrize("mult", [0.01, 20.0])
def test_old_rows_keep_or_move_within_half_a_step(mult):
    # 3 new tokens land at slots 5..7 of a page that already holds 5 rows
    pr, qn, kn, vn = _fp8_problem([16 + 8, 40 + 8], 3, P=16)
    vn = W.bf16_bits_from_f32((_f64(vn) * mult).astype(np.float32))
    kn = W.bf16_bits_from_f32((_f64(kn) * mult).astype(np.float32))
    q_out, kc, vc, sc = _run(pr, qn, kn, vn)
    tabv = oracle.e4m3_table()
    for b in range(2):
        L = int(pr.seq_lens[b])
        pg = (L - 3) // 16
        pid, s_first = int(pr.page_table[b, pg]), (L - 3) % 16
        for which, old_codes, new_codes, new_rows in ((0, pr.k_pages, kc, kn), (1, pr.v_pages, vc, vn)):
            for h in range(2):
                s_old, s_new = pr.kv_scales[which, pid, h], sc[which, pid, h]
                assert s_new >= s_old
                v_old = tabv[old_codes[pid, h, :s_first]] * s_old
                v_now = tabv[new_codes[pid, h, :s_first]] * s_new
                if mult < 1:
                    assert s_new == s_old and np.array_equal(old_codes[pid, h, :s_first], new_codes[pid, h, :s_first])
                else:
                    assert s_new > s_old
                    # half a step of the new scale's grid at the value (E4M3: 3 mantissa bits; 2^-9 subnormal step)
                    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(v_old) / s_new, 2.0 ** -6))) - 3), 2.0 ** -9)
                    assert np.all(np.abs(v_now - v_old) <= 0.5 * step * s_new * (1 + 1e-6))
                # new rows decode to within half a step of their values
                x = _f64(new_rows[b, :, h])
                if which == 0:
                    x = oracle.rope_rows(x, np.arange(L - 3, L))
                got = tabv[new_codes[pid, h, s_first:s_first + 3]] * s_new
                step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(x) / s_new, 2.0 ** -6))) - 3), 2.0 ** -9)
                assert np.all(np.abs(got - x) <= 0.5 * step * s_new * (1 + 1e-5) + 1e-12)
    # pages other than the ones the new tokens touch are unchanged
    touched = {int(pr.page_table[b, p]) for b in range(2) for p in range((int(pr.seq_lens[b]) - 3) // 16,
                                                                         (int(pr.seq_lens[b]) - 1) // 16 + 1)}
    other = np.array(sorted(set(range(pr.num_pages)) - touched))
    assert np.array_equal(kc[other], pr.k_pages[other]) and np.array_equal(sc[:, other], pr.kv_scales[:, other])


def test_q_path_is_the_bf16_append_and_early_rows_have_no_slot():
    pr, qn, kn, vn = _fp8_problem([2, 40], 4, P=16)   # request 0: positions -2, -1, 0, 1
    q_out, kc, vc, sc = _run(pr, qn, kn, vn)
    bf = W.make_problem(name="bf", batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, seq_lens=[2, 40], page_size=16,
                        q_tokens=4, kv_dtype="bf16", seed=41, tile_len=64)
    q_bf, _, _, _ = oracle.append_rope(qn, kn, vn, bf.page_table, bf.seq_lens, bf.k_pages, bf.v_pages)
    assert np.array_equal(q_out, q_bf)
    # request 0's page 0 holds only its positions 0 and 1 (tokens 2 and 3): slots 0, 1 written, 2.. untouched
    pid = int(pr.page_table[0, 0])
    assert np.array_equal(kc[pid, :, 2:], pr.k_pages[pid, :, 2:])
