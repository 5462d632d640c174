"""CPU pins of the oracle's q rounding for the FP8-products mode (KV_FP8E4M3_MMA8; the HPC-Ops
article at sdftguanye.com, section on fine-grained task scheduling and data rearrangement: an FP8
attention kernel). Each against something other than the function itself:
  * e4m3_round against a brute-force nearest search over all finite codes, ties to the even code;
  * the row scaling lands every row's largest magnitude in [128, 256) before rounding, so each
    row keeps E4M3's 4 significant bits on its largest entries;
  * the rounded rows are bf16 numbers (exact round trip) and a zero row stays zero.
"""
import numpy as np

import oracle


def _brute(x, tab):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    vals = tab[codes]
    out = []
    for v in np.asarray(x, dtype=np.float64).reshape(-1):
        d = np.abs(vals - v)
        best = d.min()
        cand = codes[d == best]
        # ties: the even code (and the one with v's sign when both zeros tie)
        even = cand[cand % 2 == 0]
        pick = even if len(even) else cand
        same_sign = pick[np.signbit(tab[pick]) == np.signbit(v)]
        c = (same_sign if len(same_sign) else pick)[0]
        out.append(tab[c])
    return np.array(out)


def test_e4m3_round_is_the_nearest_value_ties_to_even():
    tab = oracle.e4m3_table()
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 40, 3000), rng.normal(0, 0.01, 1000), rng.uniform(-460, 460, 500),
                        tab[:126] + 0.0,  # every value itself
                        (tab[1:126] + tab[0:125]) / 2])  # every midpoint of neighbouring codes
    got = oracle.e4m3_round(x)
    want = _brute(np.minimum(np.abs(x), 448.0) * np.sign(x), tab)
    assert np.array_equal(np.abs(got), np.abs(want))


def test_rows_are_scaled_into_128_256_and_stay_bf16():
    rng = np.random.default_rng(11)
    rows = rng.normal(0, 1, (64, 128)) * np.exp(rng.uniform(-8, 8, (64, 1)))
    rows[3] = 0.0
    rows[5, :] = 0.0
    rows[5, 17] = 1.0  # largest magnitude exactly a power of two
    qb = oracle.bf16_bits(rows)
    r = oracle.round_q_e4m3_rows(qb)
    v = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    rv = (r.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(rv[3] == 0)
    assert rv[5, 17] == 1.0
    for i in range(64):
        a = np.abs(v[i]).max()
        if a == 0:
            continue
        E = 7 - int(np.floor(np.log2(a)))
        assert 128 <= a * 2.0 ** E < 256
        # the rounded row equals the nearest E4M3 values of the scaled row, scaled back
        want = _brute(v[i] * 2.0 ** E, oracle.e4m3_table()) * 2.0 ** -E
        assert np.array_equal(rv[i], want)
    # bf16 round trip is exact
    assert np.array_equal(oracle.bf16_bits(rv), r)
