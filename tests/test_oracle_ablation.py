"""The transform ablation of OrbitQuant §3.3, checked with the oracle on CPU.

§2.3 gives the reason for the random permutation P_pi: without it, outlier
coordinates that sit together stay concentrated in a few 64-wide blocks; with
it they are scattered over the blocks and every coordinate's variance comes
close to 1/d.  §3.3 reports the outcome: a dense Haar rotation is best in
theory, the block Hadamard transform without the permutation degrades at low
bit widths, and RPBH is close to the dense rotation.  These are statements
about the method (the "why"), not about the CUDA path, so they are tested
here on the oracle: relative quantisation error of the directions for the
three transforms on activations whose outlier channels are contiguous.  The
dense rotation is a seeded Haar-distributed orthogonal matrix (QR of a
Gaussian matrix with the sign of R's diagonal folded in), which makes every
rotated coordinate Gaussian: its error must then match the Lloyd-Max
distortion of N(0, 1), computed in closed form by the oracle.
"""

import numpy as np
import pytest

import oracle


def _haar(d, seed):
    g = np.random.default_rng(seed)
    Q, R = np.linalg.qr(g.standard_normal((d, d)))
    return Q * np.sign(np.diag(R))


def _rel_error(X, Pi, levels, bounds):
    q = oracle.quantize_act(X, Pi, bounds)
    rec = q["norms"][:, None] * levels[q["codes"]]
    return float(np.mean(np.sum((q["xr"] - rec) ** 2, axis=1) / np.sum(q["xr"] ** 2, axis=1)))


@pytest.fixture(scope="module")
def transforms():
    d, T = 1024, 64
    g = np.random.default_rng(0)
    X = g.standard_t(3, (T, d))
    X[:, 200:232] *= 30.0                     # 32 neighbouring outlier channels
    perm, signs = oracle.rpbh_draw(d, 11)
    return d, X, {
        "rpbh": oracle.rpbh_matrix(perm, signs),
        "block_hadamard": oracle.rpbh_matrix(np.arange(d), signs),   # pi = identity
        "haar": _haar(d, 5),
    }


def test_permutation_spreads_neighbouring_outliers(transforms):
    d, X, P = transforms
    share = {}
    for name in ("rpbh", "block_hadamard"):
        Y = oracle.rpbh_apply(P[name], X)
        blocks = np.sum(Y.reshape(len(X), d // 64, 64) ** 2, axis=2)
        # per token, the share of the energy in its fullest block (median over tokens)
        share[name] = float(np.median(np.max(blocks / blocks.sum(axis=1, keepdims=True), axis=1)))
    # without pi the 32 outlier channels fill one of the 16 blocks; with pi
    # they land in many blocks (a heavy-tailed t(3) token can still be
    # dominated by one extreme value, hence the median)
    assert share["block_hadamard"] > 0.9
    assert share["rpbh"] < 0.5


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantisation_error_ordering(transforms, bits):
    d, X, P = transforms
    levels, bounds = oracle.lloydmax_table(d, bits)
    err = {name: _rel_error(X, Pi, levels, bounds) for name, Pi in P.items()}
    # the dense rotation makes the coordinates Gaussian: its error is the
    # Lloyd-Max distortion of N(0, 1) (within sampling error)
    lu, bu = oracle.lloydmax_table(1, bits)
    distortion = oracle.lloydmax_distortion_unit(lu, bu)
    assert abs(err["haar"] / distortion - 1) < 0.05
    # §3.3's ordering: dense Haar <= RPBH, and the permutation matters
    assert err["haar"] <= err["rpbh"]
    assert err["rpbh"] < 0.5 * err["block_hadamard"]
