"""Lloyd-Max codebooks for N(0, 1/d) (oracle side).

OrbitQuant §1 and §4.2: after the RPBH rotation every coordinate of the unit
direction is close to N(0, 1/d), so one Lloyd-Max codebook per input width d
serves every layer, timestep and prompt.  Lloyd-Max means the MSE-optimal
scalar quantiser with 2**b levels; its two necessary conditions are

* midpoint:  each decision boundary is halfway between its two levels,
* centroid:  each level is the conditional mean of the density on its cell,

and for a log-concave density such as the Gaussian they have a single solution
(so any correct solver lands on the same table).  The oracle finds it by the
plain fixed-point iteration that alternates the two conditions, on N(0,1), in
fp64; the N(0, 1/d) table is that table times 1/sqrt(d) (a Gaussian scaled by
sigma has its optimal quantiser scaled by sigma).

Numerics (our reading of "compute in fp64"): a cell probability on the
positive side is taken as Q(a) - Q(b) with Q the upper tail, so that the far
tails keep their relative precision; the iteration runs until the levels stop
moving (below 1e-15, or no new smallest move for 2000 steps: the fp64
rounding floor).  The map contracts slowly for many levels (rate ~0.9999 at 8
bits), which amplifies rounding, so the answer sits within ~1e-11 of the
exact optimum at 8 bits and ~1e-14 at <= 4 bits.  The levels are made
exactly antisymmetric at the end, which puts the middle boundary at 0.
"""

import functools

import numpy as np
from scipy.special import ndtr

_INV_SQRT_2PI = 1.0 / np.sqrt(2.0 * np.pi)


def _pdf(x):
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        out = np.exp(-0.5 * x * x) * _INV_SQRT_2PI
    return np.where(np.isinf(x), 0.0, out)


def _cell_prob(a, b):
    """P(a < X < b) for X ~ N(0,1); upper-tail form when the cell is >= 0."""
    upper = ndtr(-a) - ndtr(-b)
    lower = ndtr(b) - ndtr(a)
    return np.where(a >= 0.0, upper, lower)


def _x_pdf(x):
    """x * pdf(x), taken as 0 at +-inf."""
    x = np.asarray(x, dtype=np.float64)
    safe = np.where(np.isinf(x), 0.0, x)
    return safe * _pdf(safe) * np.where(np.isinf(x), 0.0, 1.0)


@functools.lru_cache(maxsize=None)
def lloydmax_unit(bits, tol=1e-15, stall=2000, max_iter=3_000_000):
    """Lloyd-Max quantiser of N(0,1) with 2**bits levels.

    Returns (levels[2**bits], bounds[2**bits - 1], iterations), increasing,
    levels antisymmetric.  Iteration: levels start uniform on (-4, 4); then
    repeat  t = midpoints(c);  c = centroids(t)  until no level moves by more
    than ``tol``, or until the largest move has not set a new minimum for
    ``stall`` iterations (the map has reached its fp64 rounding floor).
    """
    if not 1 <= bits <= 8:
        raise ValueError("bits must be in 1..8")
    L = 2 ** bits
    c = (np.arange(L) - (L - 1) / 2.0) * (8.0 / L)
    best, since_best = np.inf, 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate(([-np.inf], t))
        hi = np.concatenate((t, [np.inf]))
        c_new = (_pdf(lo) - _pdf(hi)) / _cell_prob(lo, hi)
        step = np.max(np.abs(c_new - c))
        c = c_new
        if step < tol:
            break
        if step < best:
            best, since_best = step, 0
        else:
            since_best += 1
            if since_best >= stall and best < 1e-12:
                break
    else:
        raise RuntimeError(f"Lloyd-Max iteration did not converge at {bits} bits")
    c = 0.5 * (c - c[::-1])
    t = 0.5 * (c[:-1] + c[1:])
    c.setflags(write=False)
    t.setflags(write=False)
    return c, t, it


def lloydmax_table(d, bits):
    """(levels, bounds) of the Lloyd-Max quantiser of N(0, 1/d), fp64."""
    if d < 1:
        raise ValueError("d must be positive")
    c, t, _ = lloydmax_unit(bits)
    sigma = 1.0 / np.sqrt(d)
    return c * sigma, t * sigma


def lloydmax_distortion_unit(levels, bounds):
    """Mean squared error of a scalar quantiser applied to N(0,1).

    Written out per cell from the Gaussian moments on (a, b):
    int (x - c)^2 pdf = P - (b pdf(b) - a pdf(a)) - 2c (pdf(a) - pdf(b)) + c^2 P.
    """
    levels = np.asarray(levels, dtype=np.float64)
    bounds = np.asarray(bounds, dtype=np.float64)
    lo = np.concatenate(([-np.inf], bounds))
    hi = np.concatenate((bounds, [np.inf]))
    P = _cell_prob(lo, hi)
    second = P - (_x_pdf(hi) - _x_pdf(lo))
    first = _pdf(lo) - _pdf(hi)
    return float(np.sum(second - 2.0 * levels * first + levels ** 2 * P))
