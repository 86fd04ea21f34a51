"""Quantised linear layers (oracle side), fp64.

OrbitQuant §2.2 (the last paragraph): the weights absorbed Pi^T and the
activations get Pi, so W^' x^' ~= W Pi^T Pi x = W x with no inverse rotation.
With w^'_n = r'_n · C_w[q_n] (§2.1 step 4) and x^' = s · C_a[p] (§2.2 step 5)
the layer output is

    y[m, n] = s_m · r'_n · sum_k C_w[q_nk] · C_a[p_mk].

INT8 path (INT8-convrot §4: "load W_int8, dequantise or use an INT8 operator"):

    y[m, n] = scale_n · sum_k q_nk · x'_mk,   x' = bf16(Pi x).

Both are plain definitions; the oracle evaluates them with one fp64 matmul.
"""

import numpy as np


def qlinear(a_codes, s, levels_a, w_codes, rnorm, levels_w):
    A = np.asarray(levels_a, dtype=np.float64)[np.asarray(a_codes)]
    B = np.asarray(levels_w, dtype=np.float64)[np.asarray(w_codes)]
    s = np.asarray(s, dtype=np.float64)
    r = np.asarray(rnorm, dtype=np.float64)
    return (A @ B.T) * s[:, None] * r[None, :]


def qlinear_int8(xr, q, scale):
    xr = np.asarray(xr, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    return (xr @ q.T) * np.asarray(scale, dtype=np.float64)[None, :]


def qlinear_int8_asym(xr, q, scale, z):
    """y = scale_n * sum_k (q_nk - z_n) x'_mk in fp64 (asymmetric INT8 layer)."""
    xr = np.asarray(xr, dtype=np.float64)
    qz = np.asarray(q, dtype=np.float64) - np.asarray(z, dtype=np.float64)[:, None]
    return (xr @ qz.T) * np.asarray(scale, dtype=np.float64)[None, :]
