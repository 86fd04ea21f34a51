"""Pins of the oracle's Lloyd-Max codebooks.

* closed form at 1 bit: levels +-sqrt(2/pi), MSE 1 - 2/pi;
* J. Max (1960) Table I for 4, 8 and 16 levels (textbook values);
* the centroid condition checked by independent numerical quadrature;
* the midpoint condition, antisymmetry and monotone distortion;
* the Panter-Dite high-resolution limit at 6 and 8 bits;
* the centroid condition and the distortion checked on Gaussian samples
  (random draws and averages only);
* the N(0, 1/d) table checked by quadrature against the N(0, 1/d) density.
"""

import numpy as np
import pytest
from scipy import integrate
from scipy.stats import norm

import oracle
from oracle.lloydmax import lloydmax_distortion_unit
from conftest import golden_rows


def test_one_bit_closed_form():
    c, t, _ = oracle.lloydmax_unit(1)
    assert np.allclose(c, [-np.sqrt(2 / np.pi), np.sqrt(2 / np.pi)], rtol=0, atol=1e-15)
    assert t.tolist() == [0.0]
    assert abs(lloydmax_distortion_unit(c, t) - (1 - 2 / np.pi)) < 1e-15


def test_max_1960_table():
    for row in golden_rows("max1960_gaussian.txt"):
        n = int(row[0])
        xs = [float(v) for v in row[1].split()]
        ys = [float(v) for v in row[2].split()]
        mse = float(row[3])
        c, t, _ = oracle.lloydmax_unit(int(np.log2(n)))
        half = n // 2
        assert np.allclose(c[half:], ys, rtol=5e-4, atol=0)
        assert np.allclose(t[half:], xs, rtol=5e-4, atol=0)
        assert abs(lloydmax_distortion_unit(c, t) / mse - 1) < 1e-3


def _centroid_by_quadrature(lo, hi, pdf):
    num = integrate.quad(lambda x: x * pdf(x), lo, hi, epsabs=0, epsrel=1e-13, limit=200)[0]
    den = integrate.quad(pdf, lo, hi, epsabs=0, epsrel=1e-13, limit=200)[0]
    return num / den


@pytest.mark.parametrize("bits", [2, 3, 4, 6])
def test_centroid_condition_by_quadrature(bits):
    c, t, _ = oracle.lloydmax_unit(bits)
    edges = np.concatenate(([-np.inf], t, [np.inf]))
    half = len(c) // 2
    worst = 0.0
    for j in range(half, len(c)):            # the negative half mirrors it
        lo, hi = edges[j], min(edges[j + 1], 40.0)
        worst = max(worst, abs(_centroid_by_quadrature(lo, hi, norm.pdf) - c[j]))
    assert worst < 1e-11


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 6, 8])
def test_midpoint_and_symmetry(bits):
    c, t, _ = oracle.lloydmax_unit(bits)
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(t, 0.5 * (c[:-1] + c[1:]))
    assert np.array_equal(c, -c[::-1])
    assert t[len(t) // 2] == 0.0


def test_centroid_residual_and_distortion_trend():
    prev = np.inf
    for bits in (1, 2, 3, 4, 5, 6, 7, 8):
        c, t, _ = oracle.lloydmax_unit(bits)
        lo = np.concatenate(([-np.inf], t))
        hi = np.concatenate((t, [np.inf]))
        P = norm.cdf(hi) - norm.cdf(lo)
        cen = (norm.pdf(lo) - norm.pdf(hi)) / np.where(P > 0, P, 1)
        upper = lo >= 0
        Pu = norm.sf(lo) - norm.sf(hi)
        cen = np.where(upper, (norm.pdf(lo) - norm.pdf(hi)) / Pu, cen)
        assert np.max(np.abs(cen - c)) < 1e-12
        D = lloydmax_distortion_unit(c, t)
        assert D < prev
        prev = D


@pytest.mark.parametrize("bits", [6, 8])
def test_panter_dite_limit(bits):
    c, t, _ = oracle.lloydmax_unit(bits)
    D = lloydmax_distortion_unit(c, t)
    pd = np.sqrt(3) * np.pi / 2 * 4.0 ** (-bits)     # (1/12)(int p^(1/3))^3 2^(-2b)
    assert 0.95 < D / pd < 1.0


@pytest.mark.parametrize("bits", [3, 4])
def test_centroid_condition_by_sampling(bits):
    # With the oracle's boundaries held fixed, the sample mean of each cell of a
    # (symmetrised) Gaussian sample must match the oracle's level within 5
    # standard errors, and the sample MSE must match the closed-form distortion.
    # No erf or quadrature is involved: only random draws and averages.
    g = np.random.default_rng(123 + bits)
    half = g.standard_normal(2_000_000)
    x = np.concatenate([half, -half])
    c, t, _ = oracle.lloydmax_unit(bits)
    idx = np.searchsorted(t, x)
    cnt = np.bincount(idx, minlength=len(c))
    mean = np.bincount(idx, weights=x, minlength=len(c)) / cnt
    var = np.bincount(idx, weights=x * x, minlength=len(c)) / cnt - mean ** 2
    se = np.sqrt(var / cnt)
    assert np.all(np.abs(mean - c) < 5 * se)
    err2 = (x - c[idx]) ** 2
    D = lloydmax_distortion_unit(c, t)
    assert abs(np.mean(err2) - D) < 5 * np.std(err2) / np.sqrt(x.size / 2)


def test_table_for_dimension_d_by_quadrature():
    d = 64
    levels, bounds = oracle.lloydmax_table(d, 3)
    sigma = 1 / np.sqrt(d)
    pdf = lambda x: norm.pdf(x, scale=sigma)
    edges = np.concatenate(([-np.inf], bounds, [np.inf]))
    for j in range(4, 8):
        hi = min(edges[j + 1], 40 * sigma)
        assert abs(_centroid_by_quadrature(edges[j], hi, pdf) - levels[j]) < 1e-12
