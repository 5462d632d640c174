"""CPU pins of the oracle's fused pre-processing (rotary embedding of the new q and k, and the
append of the new K/V rows into their pages), each against something other than the oracle's
own formula:
  * the rotation against the same rotation written as complex multiplication;
  * the defining property of rotary embeddings: scores depend only on the position difference;
  * position 0 is the identity and every (i, i + d/2) pair keeps its norm;
  * bf16 rounding against a brute-force nearest search (ties to even);
  * the append against a dense gather of each request through its page table.
"""
import numpy as np
import pytest

import oracle

BASE = 10000.0


def _complex_rotation(x, pos, base=BASE):
    """The pair (x_i, x_{i+d/2}) as the complex number x_i + 1j x_{i+d/2}, times e^(1j pos theta_i)."""
    d = x.shape[-1]
    h = d // 2
    theta = base ** (-np.arange(h, dtype=np.float64) * 2.0 / d)
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("d", [8, 64, 128])
def test_rope_equals_complex_rotation(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((20, d))
    pos = np.concatenate([[0, 1, 2, 15, 16], rng.integers(0, 200000, 15)]).astype(np.float64)
    got = oracle.rope_rows(x, pos)
    want = _complex_rotation(x, pos)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-9)


def test_rope_scores_depend_only_on_position_difference():
    rng = np.random.default_rng(1)
    d = 64
    for _ in range(20):
        q, k = rng.standard_normal(d), rng.standard_normal(d)
        p, pk, c = (float(v) for v in rng.integers(0, 100000, 3))
        s1 = oracle.rope_rows(q[None], [p])[0] @ oracle.rope_rows(k[None], [pk])[0]
        s2 = oracle.rope_rows(q[None], [p + c])[0] @ oracle.rope_rows(k[None], [pk + c])[0]
        s3 = q @ oracle.rope_rows(k[None], [pk - p])[0]
        assert abs(s1 - s2) < 1e-8 * (1 + abs(s1))
        assert abs(s1 - s3) < 1e-8 * (1 + abs(s1))


def test_rope_identity_at_zero_and_pair_norms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 128))
    assert np.array_equal(oracle.rope_rows(x, [0] * 5), x)
    y = oracle.rope_rows(x, [3, 77, 1000, 65535, 131071])
    np.testing.assert_allclose(x[:, :64] ** 2 + x[:, 64:] ** 2, y[:, :64] ** 2 + y[:, 64:] ** 2, rtol=1e-12)
    # pair 0 has theta = 1: at position 7 it turns by 7 radians
    y7 = oracle.rope_rows(x, [7.0] * 5)
    np.testing.assert_allclose(y7[:, 0], x[:, 0] * np.cos(7.0) - x[:, 64] * np.sin(7.0), atol=1e-12)
    np.testing.assert_allclose(y7[:, 64], x[:, 64] * np.cos(7.0) + x[:, 0] * np.sin(7.0), atol=1e-12)


def _nearest_bf16_brute(v):
    """Nearest bf16 to the double v by trying the neighbours of its binary32 rounding."""
    f = np.float32(v)
    u = int(np.array(f, dtype=np.float32).view(np.uint32)) >> 16
    best = None
    for c in (u - 1, u, u + 1):
        c &= 0xFFFF
        val = float(np.array(c << 16, dtype=np.uint32).view(np.float32))
        if not np.isfinite(val):
            continue
        dist = abs(val - v)
        key = (dist, c & 1)  # ties: the even mantissa wins
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_bf16_rounding_brute_force():
    rng = np.random.default_rng(3)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000))
    # exact ties between neighbouring bf16 values, and values a hair either side of them
    for m in rng.integers(128, 256, 200):
        for e in rng.integers(-100, 100, 2):
            t = (float(m) + 0.5) * 2.0 ** int(e)
            vals += [t, np.nextafter(t, np.inf), np.nextafter(t, -np.inf), -t]
    vals += [2.0 ** -130, 3 * 2.0 ** -133, 1e-40]  # bf16 subnormals
    got = oracle.bf16_bits(np.array(vals))
    for v, g in zip(vals, got):
        assert int(g) == _nearest_bf16_brute(v), (v, hex(int(g)))


def _bf16_value(bits):
    return np.array(np.asarray(bits, dtype=np.uint32) << 16, dtype=np.uint32).view(np.float32).astype(np.float64)


def _rounded(x):
    return np.array([_nearest_bf16_brute(float(v)) for v in x.reshape(-1)], dtype=np.uint16).reshape(x.shape)


def test_append_rope_against_dense_gather():
    rng = np.random.default_rng(4)
    B, T, Hq, Hkv, d, P = 3, 2, 4, 2, 8, 4
    lens = np.array([5, 9, 1], dtype=np.int32)  # request 2 has a token at position -1: no slot
    mpps = 4
    num_pages = B * mpps
    perm = rng.permutation(num_pages).astype(np.int32)
    tab = perm.reshape(B, mpps)

    def bf16(shape):
        return rng.integers(0, 1 << 16, shape, dtype=np.uint16) & 0xBFFF  # finite values, |x| < 2

    q_new, k_new, v_new = bf16((B, T, Hq, d)), bf16((B, T, Hkv, d)), bf16((B, T, Hkv, d))
    k_pages, v_pages = bf16((num_pages, Hkv, P, d)), bf16((num_pages, Hkv, P, d))
    q_out, kp, vp, n = oracle.append_rope(q_new, k_new, v_new, tab, lens, k_pages, v_pages)
    written = set()
    for b in range(B):
        for t in range(T):
            pos = int(lens[b]) - T + t
            want_q = _rounded(_complex_rotation(_bf16_value(q_new[b, t]), [max(pos, 0)] * Hq))
            assert np.array_equal(q_out[b, t], want_q)
            if pos < 0:
                continue
            page, slot = tab[b, pos // P], pos % P
            want_k = _rounded(_complex_rotation(_bf16_value(k_new[b, t]), [pos] * Hkv))
            assert np.array_equal(kp[page, :, slot], want_k)
            assert np.array_equal(vp[page, :, slot], v_new[b, t])
            written.add((page, slot))
    assert n == len(written) * Hkv
    for page in range(num_pages):
        for slot in range(P):
            if (page, slot) not in written:
                assert np.array_equal(kp[page, :, slot], k_pages[page, :, slot])
                assert np.array_equal(vp[page, :, slot], v_pages[page, :, slot])
    bad = tab.copy()
    bad[1, 2] = num_pages  # the page of request 1's positions 8..11 (its new tokens 7 and 8 span pages 1 and 2)
    assert oracle.append_rope(q_new, k_new, v_new, bad, lens, k_pages, v_pages)[3] == -1
