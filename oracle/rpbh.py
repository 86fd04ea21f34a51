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


def rpbh_rows(perm, signs, r0, r1, h=64):
    """Rows r0 .. r1-1 of the dense Pi_d = B · P_pi (r0, r1 multiples of h).

    Row k of P_pi selects input coordinate perm[k], so the product B · P_pi
    is B with column m moved to column perm[m]; within output block b that
    places the 64 x 64 piece H_h D_b at the columns perm[64b .. 64b+63].  (A
    d^3 matmul at d = 12288 would take hours; the test-suite checks this
    column move against the literal product B @ P at small d.)
    """
    perm = np.asarray(perm)
    signs = np.asarray(signs, dtype=np.float64)
    d = perm.shape[0]
    if d % h or r0 % h or r1 % h or not 0 <= r0 <= r1 <= d:
        raise ValueError("rows must be whole blocks of h")
    H = hadamard(h)
    out = np.zeros((r1 - r0, d))
    for b in range(r0 // h, r1 // h):
        sl = slice(b * h, (b + 1) * h)
        out[b * h - r0: (b + 1) * h - r0, perm[sl]] = H @ np.diag(signs[sl])
    return out


def rpbh_matrix(perm, signs, h=64):
    """The dense d x d Pi_d = B · P_pi."""
    return rpbh_rows(perm, signs, 0, len(perm), h)


def rpbh_apply(Pi, X, chunk=2048):
    """x' = Pi x for each row x of X (OrbitQuant §2.2 step 1).

    ``Pi`` is the dense matrix, or a (perm, signs) pair for widths whose dense
    matrix is too large to hold: then Pi is built and applied ``chunk`` rows
    at a time -- the same dense product, in pieces.
    """
    X = np.asarray(X, dtype=np.float64)
    if isinstance(Pi, tuple):
        perm, signs = Pi
        d = len(perm)
        out = np.empty((X.shape[0], d))
        for r0 in range(0, d, chunk):
            r1 = min(d, r0 + chunk)
            out[:, r0:r1] = X @ rpbh_rows(perm, signs, r0, r1).T
        return out
    return X @ Pi.T
