"""Pins of the oracle's 8-bit integer-level layer (oracle.qlinear.int8_levels,
oracle.qlinear.qlinear_int8_levels).

* the integer levels of J. Max's (1960) 4-, 8- and 16-level Gaussian
  quantisers, worked by hand from the published table (tests/golden);
* grid invariants: |l| <= 127 with 127 reached, antisymmetry, order, and
  |l - alpha c| <= 1/2; the same integers for every d (alpha absorbs 1/sqrt(d));
* the layer against a pure-Python triple loop, the equal-code closed form, and
  the exact-level layer (oracle.qlinear) within the levels' rounding bound.
"""

import numpy as np
import pytest

import oracle
from conftest import golden_rows


def test_int8_levels_of_max_1960_table():
    for row in golden_rows("int8_levels_max1960.txt"):
        n = int(row[0])
        want = [int(v) for v in row[1].split()]
        c, _, _ = oracle.lloydmax_unit(int(np.log2(n)))
        l, alpha = oracle.int8_levels(c)
        assert l[n // 2:].tolist() == want
        assert l[: n // 2].tolist() == [-v for v in reversed(want)]


@pytest.mark.parametrize("bits", range(1, 9))
def test_int8_level_grid_invariants(bits):
    c1, _ = oracle.lloydmax_table(64, bits)
    l1, a1 = oracle.int8_levels(c1)
    assert np.max(np.abs(l1)) == 127 and np.all(np.abs(l1) <= 127)
    assert np.array_equal(l1, -l1[::-1])
    assert np.all(np.diff(l1) >= 0)
    assert np.all(np.abs(l1 - a1 * c1) <= 0.5)
    c2, _ = oracle.lloydmax_table(3072, bits)
    l2, a2 = oracle.int8_levels(c2)
    assert np.array_equal(l1, l2)
    assert abs(a2 / a1 - np.sqrt(3072 / 64)) < 1e-12
    # no level sits so close to a half-integer that fp64 rounding, or another
    # solver's table (which agrees to ~3e-11 relative), could round it the
    # other way (the closest is 3.3e-5 away, at 7 bits)
    frac = np.abs(a2 * c2 - np.floor(a2 * c2) - 0.5)
    assert np.all(frac > 1e-6)


def _loop(a_codes, s, la, aa, w_codes, rn, lw, aw):
    M, K = a_codes.shape
    N = w_codes.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0
            for k in range(K):
                acc += int(la[a_codes[m, k]]) * int(lw[w_codes[n, k]])
            y[m, n] = s[m] * rn[n] * acc / (aa * aw)
    return y


def test_layer_against_triple_loop():
    g = np.random.default_rng(7)
    K = 64
    ca, _ = oracle.lloydmax_table(K, 4)
    cw, _ = oracle.lloydmax_table(K, 2)
    p = g.integers(0, 16, (3, K))
    q = g.integers(0, 4, (5, K))
    s = g.uniform(0.5, 2, 3)
    rn = g.uniform(0.5, 2, 5)
    y = oracle.qlinear_int8_levels(p, s, ca, q, rn, cw)
    la, aa = oracle.int8_levels(ca)
    lw, aw = oracle.int8_levels(cw)
    assert np.allclose(y, _loop(p, s, la, aa, q, rn, lw, aw), rtol=1e-14, atol=0)


def test_equal_codes_closed_form():
    K = 256
    ca, _ = oracle.lloydmax_table(K, 3)
    cw, _ = oracle.lloydmax_table(K, 4)
    la, aa = oracle.int8_levels(ca)
    lw, aw = oracle.int8_levels(cw)
    p = np.full((2, K), 5)
    q = np.full((3, K), 12)
    s = np.array([1.5, 0.25])
    rn = np.array([2.0, 1.0, 0.5])
    y = oracle.qlinear_int8_levels(p, s, ca, q, rn, cw)
    want = s[:, None] * rn[None, :] * K * la[5] * lw[12] / (aa * aw)
    assert np.allclose(y, want, rtol=1e-15, atol=0)


@pytest.mark.parametrize("ba,bw", [(4, 4), (4, 2), (3, 3), (6, 4), (8, 8)])
def test_within_rounding_bound_of_exact_levels(ba, bw):
    g = np.random.default_rng(ba * 10 + bw)
    K = 512
    ca, _ = oracle.lloydmax_table(K, ba)
    cw, _ = oracle.lloydmax_table(K, bw)
    p = g.integers(0, 2 ** ba, (6, K))
    q = g.integers(0, 2 ** bw, (7, K))
    s = g.uniform(0.5, 2, 6)
    rn = g.uniform(0.5, 2, 7)
    y8 = oracle.qlinear_int8_levels(p, s, ca, q, rn, cw)
    y = oracle.qlinear(p, s, ca, q, rn, cw)
    la, aa = oracle.int8_levels(ca)
    # C_w C_a - L_w L_a = C_w (C_a - L_a) + L_a (C_w - L_w), |L - C| <= 1/(2 alpha)
    per = np.abs(cw[q])[None, :, :] * 0.5 / aa + np.abs(la[p] / aa)[:, None, :] * 0.5 / oracle.int8_levels(cw)[1]
    bound = s[:, None] * rn[None, :] * per.sum(axis=2)
    assert np.all(np.abs(y8 - y) <= bound * (1 + 1e-12))
    assert np.any(y8 != y)
