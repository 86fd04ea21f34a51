"""Pins of the oracle's fused layer (OrbitQuant §6.2: the rotation fused into
the producing matmul): GELU against the normal CDF from scipy.stats and
published values, and the composition against a pure-Python triple loop with
an explicit dense rotation on a tiny case."""

import math

import numpy as np
from scipy.stats import norm

import oracle


def test_gelu_is_y_times_the_normal_cdf():
    y = np.concatenate([np.linspace(-8, 8, 2001), [0.0, -0.0, 1e-300, 40.0, -40.0]])
    assert np.allclose(oracle.gelu(y), y * norm.cdf(y), rtol=1e-13, atol=1e-300)
    # odd-part identity: gelu(y) - gelu(-y) = y (Phi(y) + Phi(-y) = 1)
    assert np.allclose(oracle.gelu(y) - oracle.gelu(-y), y, rtol=1e-14, atol=1e-15)
    # Phi(1) = 0.8413447460685429 (standard normal table), Phi(2) = 0.9772498680518208
    assert math.isclose(oracle.gelu(1.0), 0.8413447460685429, rel_tol=1e-15)
    assert math.isclose(oracle.gelu(2.0), 2 * 0.9772498680518208, rel_tol=1e-15)
    assert oracle.gelu(0.0) == 0.0


def test_fused_layer_against_a_triple_loop_and_dense_rotation():
    g = np.random.default_rng(3)
    M, K, N = 3, 64, 128
    xr = g.standard_normal((M, K))
    q = g.integers(-127, 128, (N, K))
    scale = g.random(N) * 0.01
    perm, signs = oracle.rpbh_draw(N, 9)
    Pi = oracle.rpbh_matrix(perm, signs)
    for act in ("gelu", "none"):
        got = oracle.qlinear_int8_rotate_next(xr, q, scale, Pi, activation=act)
        ref = np.zeros((M, N))
        for m in range(M):
            x = []
            for j in range(N):
                yj = scale[j] * sum(float(q[j, k]) * xr[m, k] for k in range(K))
                x.append(0.5 * yj * (1 + math.erf(yj / math.sqrt(2))) if act == "gelu" else yj)
            for r in range(N):
                ref[m, r] = sum(Pi[r, c] * x[c] for c in range(N))
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_published_erf_approximation_meets_its_bound():
    """The fused kernel's GELU takes the normal CDF from Abramowitz & Stegun
    (1964) formula 7.1.26 (|error| <= 1.5e-7 in erf for x >= 0).  The constants
    as written in the kernel, evaluated here in fp64, meet that bound against
    scipy's erfc; the kernel evaluates them in fp32, and its outputs are checked
    against the oracle's exact GELU by the GPU parity tests."""
    from scipy.special import erfc
    p, a = 0.3275911, (0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429)
    x = np.linspace(0.0, 12.0, 120001)
    t = 1.0 / (1.0 + p * x)
    poly = t * (a[0] + t * (a[1] + t * (a[2] + t * (a[3] + t * a[4]))))
    assert np.max(np.abs(poly * np.exp(-x * x) - erfc(x))) <= 1.5e-7


def test_code_layer_fused_against_a_triple_loop_and_dense_rotation():
    g = np.random.default_rng(4)
    M, K, N, ba, bw = 3, 64, 128, 3, 2
    levels_a, _ = oracle.lloydmax_table(K, ba)
    levels_w, _ = oracle.lloydmax_table(K, bw)
    a = g.integers(0, 2 ** ba, (M, K))
    w = g.integers(0, 2 ** bw, (N, K))
    s = g.random(M) + 0.5
    rn = g.random(N) + 0.5
    perm, signs = oracle.rpbh_draw(N, 10)
    Pi = oracle.rpbh_matrix(perm, signs)
    for act in ("gelu", "none"):
        got = oracle.qlinear_rotate_next(a, s, levels_a, w, rn, levels_w, Pi, activation=act)
        ref = np.zeros((M, N))
        for m in range(M):
            x = []
            for j in range(N):
                yj = s[m] * rn[j] * sum(float(levels_w[w[j, k]]) * float(levels_a[a[m, k]]) for k in range(K))
                x.append(0.5 * yj * (1 + math.erf(yj / math.sqrt(2))) if act == "gelu" else yj)
            for r in range(N):
                ref[m, r] = sum(Pi[r, c] * x[c] for c in range(N))
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_quantize_rotated_is_steps_two_to_four_of_quantize_act():
    """Rotating first and quantising the rotated rows gives exactly what
    quantize_act gives from the unrotated rows (same norms, directions, codes);
    on a tiny case every code is the brute-force nearest level."""
    g = np.random.default_rng(5)
    d, bits = 256, 4
    X = g.standard_normal((9, d)) * np.linspace(0.1, 10, 9)[:, None]
    X[4] = 0.0
    perm, signs = oracle.rpbh_draw(d, 2)
    Pi = oracle.rpbh_matrix(perm, signs)
    levels, bounds = oracle.lloydmax_table(d, bits)
    full = oracle.quantize_act(X, Pi, bounds)
    part = oracle.quantize_rotated(oracle.rpbh_apply(Pi, X), bounds)
    assert np.array_equal(part["codes"], full["codes"])
    assert np.array_equal(part["norms"], full["norms"])
    assert np.array_equal(part["v"], full["v"])
    v = part["v"]
    nearest = np.argmin(np.abs(v[..., None] - levels[None, None, :]), axis=-1)
    tie = np.isclose(np.abs(v[..., None] - levels).min(-1),
                     np.sort(np.abs(v[..., None] - levels), axis=-1)[..., 1], rtol=0, atol=1e-15)
    assert np.array_equal(part["codes"][~tie], nearest[~tie])
    assert np.all(part["codes"][4] == 2 ** (bits - 1))
