"""Pins of the oracle's 8-bit-level layers (oracle.qlinear.int8_levels,
qlinear_int8_levels, e4m3_round, fp8_levels, qlinear_fp8_levels).

* the integer levels of J. Max's (1960) 4-, 8- and 16-level Gaussian
  quantisers, worked by hand from the published table (tests/golden);
* grid invariants: |l| <= 127 with 127 reached, antisymmetry, order, and
  |l - alpha c| <= 1/2; the same integers for every d (alpha absorbs 1/sqrt(d));
* the layer against a pure-Python triple loop, the equal-code closed form, and
  the exact-level layer (oracle.qlinear) within the levels' rounding bound;
* FP8: E4M3 rounding against PyTorch's float8_e4m3fn conversion, the Max
  tables rounded to 3 mantissa bits by hand (tests/golden), the power-of-two
  scale, and the same loop, closed form and rounding bound.
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


# ---- the FP8 (E4M3) form ----------------------------------------------------

def test_e4m3_rounding_matches_library_conversion():
    torch = pytest.importorskip("torch")
    x = np.concatenate([np.linspace(-448, 448, 20001), np.exp2(np.arange(-12, 8.8, 0.01)),
                        -np.exp2(np.arange(-12, 8.8, 0.013)),
                        [0.59375, 2.0 ** -10, 1.5 * 2.0 ** -10, 1.0625, 1.1875, 0.0]])
    lib = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_round(x), lib)


def test_fp8_levels_of_max_1960_table():
    for row in golden_rows("fp8_levels_max1960.txt"):
        n = int(row[0])
        want = np.array([float(v) for v in row[1].split()])
        c, _, _ = oracle.lloydmax_unit(int(np.log2(n)))
        e, beta = oracle.fp8_levels(c)
        assert np.array_equal(e[n // 2:] / beta, want)
        assert np.array_equal(e[: n // 2] / beta, -want[::-1])


@pytest.mark.parametrize("bits", range(1, 9))
def test_fp8_level_scale_and_bound(bits):
    for d in (64, 3072, 12288):
        c, _ = oracle.lloydmax_table(d, bits)
        e, beta = oracle.fp8_levels(c)
        assert beta == 2.0 ** np.round(np.log2(beta))
        assert 128 <= beta * np.max(np.abs(c)) < 256
        assert np.all(np.abs(e / beta - c) <= 2.0 ** -4 * np.abs(c))
        assert np.array_equal(e, -e[::-1])


def test_fp8_layer_against_triple_loop_and_closed_form():
    g = np.random.default_rng(9)
    K = 64
    ca, _ = oracle.lloydmax_table(K, 4)
    cw, _ = oracle.lloydmax_table(K, 3)
    p = g.integers(0, 16, (3, K))
    q = g.integers(0, 8, (4, K))
    s = g.uniform(0.5, 2, 3)
    rn = g.uniform(0.5, 2, 4)
    y = oracle.qlinear_fp8_levels(p, s, ca, q, rn, cw)
    ea, ba = oracle.fp8_levels(ca)
    ew, bw = oracle.fp8_levels(cw)
    assert np.allclose(y, _loop(p, s, ea, ba, q, rn, ew, bw), rtol=1e-14, atol=0)
    pe = np.full((2, K), 11)
    qe = np.full((2, K), 2)
    ye = oracle.qlinear_fp8_levels(pe, s[:2], ca, qe, rn[:2], cw)
    assert np.allclose(ye, s[:2, None] * rn[None, :2] * K * ea[11] * ew[2] / (ba * bw), rtol=1e-15, atol=0)


def test_fp8_layer_within_rounding_bound_of_exact_levels():
    g = np.random.default_rng(10)
    K = 512
    ca, _ = oracle.lloydmax_table(K, 4)
    cw, _ = oracle.lloydmax_table(K, 4)
    p = g.integers(0, 16, (6, K))
    q = g.integers(0, 16, (7, K))
    s = g.uniform(0.5, 2, 6)
    rn = g.uniform(0.5, 2, 7)
    y8 = oracle.qlinear_fp8_levels(p, s, ca, q, rn, cw)
    y = oracle.qlinear(p, s, ca, q, rn, cw)
    # each level within 2^-4 relative, so each product within (1 + 2^-4)^2 - 1
    prod = np.abs(ca[p])[:, None, :] * np.abs(cw[q])[None, :, :]
    bound = s[:, None] * rn[None, :] * prod.sum(axis=2) * ((1 + 2.0 ** -4) ** 2 - 1)
    assert np.all(np.abs(y8 - y) <= bound * (1 + 1e-12))
    assert np.any(y8 != y)
