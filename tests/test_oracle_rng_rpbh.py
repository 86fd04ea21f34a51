"""Pins of the oracle's RNG and RPBH matrix against things other than itself.

* SplitMix64 against its published test vector.
* The Hadamard matrix against scipy.linalg.hadamard (a library routine) and a
  Kronecker-power construction written here.
* The dense Pi against the literal product B @ P, against a recursive fast
  Walsh-Hadamard transform written here, and against orthogonality and the
  cancellation W Pi^T Pi x = W x (OrbitQuant §2.2).
"""

import numpy as np
import pytest
import scipy.linalg

import oracle
from oracle.rpbh import block_part, permutation_matrix
from conftest import golden_path


def _golden_splitmix():
    seeds, cur = {}, None
    for line in open(golden_path("splitmix64.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("seed"):
            cur = int(line.split()[1])
            seeds[cur] = []
        else:
            seeds[cur].append(int(line))
    return seeds


def test_splitmix64_published_vector():
    for seed, outs in _golden_splitmix().items():
        assert oracle.splitmix64(seed, len(outs)) == outs


@pytest.mark.parametrize("d", [1, 2, 64, 256, 3072])
def test_rpbh_draw_is_permutation_and_signs(d):
    perm, signs = oracle.rpbh_draw(d, seed=7)
    assert sorted(perm.tolist()) == list(range(d))
    assert set(np.unique(signs).tolist()) <= {-1, 1}
    p2, s2 = oracle.rpbh_draw(d, seed=7)
    assert np.array_equal(perm, p2) and np.array_equal(signs, s2)


def test_rpbh_draw_small_case_by_hand():
    # d = 2: one swap step with u0, then two sign draws u1, u2.
    u = oracle.splitmix64(5, 3)
    perm, signs = oracle.rpbh_draw(2, seed=5)
    j = (u[0] * 2) >> 64
    expect = [1, 0] if j == 0 else [0, 1]
    assert perm.tolist() == expect
    assert signs.tolist() == [-1 if (x >> 63) else 1 for x in u[1:]]


def test_rpbh_draw_statistics():
    # Sign balance at d = 16384 and first-position uniformity over seeds.
    _, signs = oracle.rpbh_draw(16384, seed=3)
    frac = np.mean(signs < 0)
    assert abs(frac - 0.5) < 5 * 0.5 / np.sqrt(16384)
    counts = np.zeros(8)
    for seed in range(2000):
        perm, _ = oracle.rpbh_draw(8, seed)
        counts[perm[0]] += 1
    chi2 = np.sum((counts - 250.0) ** 2 / 250.0)
    assert chi2 < 30.0   # 7 dof; p ~ 1e-4


def test_hadamard_matches_library_and_kronecker():
    for h in (1, 2, 4, 16, 64):
        H = oracle.hadamard(h)
        assert np.array_equal(H * np.sqrt(h), scipy.linalg.hadamard(h).astype(float))
        K = np.array([[1.0]])
        for _ in range(int(np.log2(h))):
            K = np.kron(K, np.array([[1.0, 1.0], [1.0, -1.0]]))
        assert np.allclose(H, K / np.sqrt(h), atol=0, rtol=0)
        assert np.allclose(H @ H.T, np.eye(h), atol=1e-15)


def test_rpbh_matrix_equals_literal_product():
    perm, signs = oracle.rpbh_draw(256, seed=11)
    Pi = oracle.rpbh_matrix(perm, signs)
    literal = block_part(signs) @ permutation_matrix(perm)
    assert np.array_equal(Pi, literal)


def test_chunked_application_equals_dense():
    d = 1024
    perm, signs = oracle.rpbh_draw(d, seed=6)
    x = np.random.default_rng(3).standard_normal((4, d))
    dense = oracle.rpbh_apply(oracle.rpbh_matrix(perm, signs), x)
    assert np.array_equal(oracle.rpbh_apply((perm, signs), x, chunk=192), dense) or \
        np.allclose(oracle.rpbh_apply((perm, signs), x, chunk=192), dense, rtol=0, atol=1e-14)


def test_rpbh_identity_case_is_textbook_hadamard():
    Pi = oracle.rpbh_matrix(np.arange(64), np.ones(64, dtype=int))
    assert np.array_equal(Pi * 8.0, scipy.linalg.hadamard(64).astype(float))


def _fwht(v):
    """Recursive fast Walsh-Hadamard transform, unnormalised (test-local)."""
    n = v.shape[-1]
    if n == 1:
        return v.copy()
    a, b = v[..., : n // 2], v[..., n // 2:]
    return np.concatenate([_fwht(a + b), _fwht(a - b)], axis=-1)


def test_rpbh_matrix_equals_gather_sign_fwht():
    d = 1024
    perm, signs = oracle.rpbh_draw(d, seed=2)
    Pi = oracle.rpbh_matrix(perm, signs)
    x = np.random.default_rng(0).standard_normal((5, d))
    y = x[:, perm] * signs[None, :]
    fast = _fwht(y.reshape(5, d // 64, 64)).reshape(5, d) / 8.0
    assert np.allclose(oracle.rpbh_apply(Pi, x), fast, rtol=0, atol=1e-13)


@pytest.mark.parametrize("d", [256, 3072])
def test_rpbh_orthogonal_and_norm_preserving(d):
    perm, signs = oracle.rpbh_draw(d, seed=1)
    Pi = oracle.rpbh_matrix(perm, signs)
    assert np.max(np.abs(Pi @ Pi.T - np.eye(d))) < 1e-12
    x = np.random.default_rng(1).standard_normal((8, d))
    n0 = np.linalg.norm(x, axis=1)
    n1 = np.linalg.norm(oracle.rpbh_apply(Pi, x), axis=1)
    assert np.max(np.abs(n1 / n0 - 1)) < 1e-13
    # each output coordinate reads exactly the 64 inputs of its permuted block
    for k in (0, 63, 64, d - 1):
        b = k // 64
        cols = np.nonzero(Pi[k])[0]
        assert sorted(cols.tolist()) == sorted(perm[64 * b: 64 * b + 64].tolist())


def test_rotation_cancels_in_the_linear():
    d = 512
    perm, signs = oracle.rpbh_draw(d, seed=4)
    Pi = oracle.rpbh_matrix(perm, signs)
    g = np.random.default_rng(2)
    W = g.standard_normal((96, d))
    x = g.standard_t(3, size=(7, d))
    Wr = oracle.rpbh_apply(Pi, W)            # W' = W Pi^T (rows w'_i = Pi w_i)
    xr = oracle.rpbh_apply(Pi, x)            # x' = Pi x
    ref = x @ W.T
    rel = np.linalg.norm(xr @ Wr.T - ref) / np.linalg.norm(ref)
    assert rel < 1e-12
