"""The RPBH rotation as an explicit dense matrix (oracle side).

OrbitQuant §2.3: Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) · P_pi, with H_h the
h x h Walsh-Hadamard matrix (h = 64 in practice), D_i diagonal +-1 and P_pi a
permutation.  The page does not say which Hadamard ordering or scaling; the
reading taken here is the Sylvester (natural) order scaled by 1/sqrt(h), so
that H_h is orthonormal and Pi_d is orthogonal -- which the cancellation in
§2.2 (W Pi^T · Pi x = W x) and the N(0, 1/d) target of §1 both require.

The oracle multiplies by the dense d x d matrix; it never uses a fast
transform.
"""

import numpy as np


def _popcount(a):
    a = np.asarray(a, dtype=np.int64)
    c = np.zeros_like(a)
    while np.any(a):
        c += a & 1
        a = a >> 1
    return c


def hadamard(h):
    """Orthonormal Sylvester-order Walsh-Hadamard matrix:
    H[r, c] = (-1)**popcount(r & c) / sqrt(h)."""
    if h < 1 or (h & (h - 1)):
        raise ValueError("h must be a power of two")
    r = np.arange(h)
    parity = _popcount(r[:, None] & r[None, :]) % 2
    return np.where(parity == 0, 1.0, -1.0) / np.sqrt(h)


def block_part(signs, h=64):
    """B = blkdiag(H_h D_1, ..., H_h D_{d/h}) as a dense d x d matrix."""
    signs = np.asarray(signs, dtype=np.float64)
    d = signs.shape[0]
    if d % h:
        raise ValueError("d must be a multiple of h")
    H = hadamard(h)
    B = np.zeros((d, d))
    for b in range(d // h):
        sl = slice(b * h, (b + 1) * h)
        B[sl, sl] = H @ np.diag(signs[sl])
    return B


def permutation_matrix(perm):
    """P with (P x)_k = x_{perm[k]}: one 1 per row, at column perm[k]."""
    d = len(perm)
    P = np.zeros((d, d))
    P[np.arange(d), perm] = 1.0
    return P


def rpbh_matrix(perm, signs, h=64):
    """Dense Pi_d = B · P_pi.

    Row k of P_pi selects input coordinate perm[k], so the product B · P_pi
    is B with column m moved to column perm[m].  That column move is what is
    computed here (a d^3 matmul at d = 12288 would take hours); the test-suite
    checks it against the literal product B @ P at small d.
    """
    B = block_part(signs, h)
    Pi = np.empty_like(B)
    Pi[:, np.asarray(perm)] = B
    return Pi


def rpbh_apply(Pi, X):
    """x' = Pi x for each row x of X (OrbitQuant §2.2 step 1)."""
    return np.asarray(X, dtype=np.float64) @ Pi.T
