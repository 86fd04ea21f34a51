"""Quantised linear layers (oracle side), fp64.

OrbitQuant §2.2 (the last paragraph): the weights absorbed Pi^T and the
activations get Pi, so W^' x^' ~= W Pi^T Pi x = W x with no inverse rotation.
With w^'_n = r'_n · C_w[q_n] (§2.1 step 4) and x^' = s · C_a[p] (§2.2 step 5)
the layer output is

    y[m, n] = s_m · r'_n · sum_k C_w[q_nk] · C_a[p_mk].

INT8 path (INT8-convrot §4: "load W_int8, dequantise or use an INT8 operator"):

    y[m, n] = scale_n · sum_k q_nk · x'_mk,   x' = bf16(Pi x).

8-bit integer-level variant (a deployment form of the first layer for INT8
tensor cores, in the spirit of OrbitQuant §4.2-§4.4: start from W8A8, lower
the widths; the pages do not define it, so its definition is ours): every
codebook's levels c_j are put on a signed 8-bit grid,

    alpha = 127 / max_j |c_j|,   l_j = round_half_even(alpha · c_j),

and y[m, n] = s_m · r'_n · (sum_k l_w[q_nk] · l_a[p_mk]) / (alpha_w · alpha_a),
the sum an exact integer.

FP8 variant (the same, for FP8 tensor cores): beta = 2^(7 - floor(log2 max|c|))
(a power of two, so beta·max|c| lies in [128, 256)), e_j = E4M3(beta · c_j)
rounded to nearest even (OCP E4M3FN: 3 mantissa bits, exponent bias 7,
subnormals below 2^-6, largest finite 448), and
y[m, n] = s_m · r'_n · (sum_k e_w[q_nk] · e_a[p_mk]) / (beta_w · beta_a).

All are plain definitions; the oracle evaluates them with one matmul.
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


def int8_levels(levels):
    """(l int64[L], alpha): levels on the signed 8-bit grid, l = RNE(alpha c)
    with alpha = 127 / max |c| (np.rint rounds halves to even); fp64 throughout."""
    c = np.asarray(levels, dtype=np.float64)
    alpha = 127.0 / np.max(np.abs(c))
    return np.rint(alpha * c).astype(np.int64), alpha


def qlinear_int8_levels(a_codes, s, levels_a, w_codes, rnorm, levels_w):
    """y = s_m r'_n (sum_k l_w[q_nk] l_a[p_mk]) / (alpha_w alpha_a); the integer
    sum is exact (int64), the scaling fp64."""
    la, alpha_a = int8_levels(levels_a)
    lw, alpha_w = int8_levels(levels_w)
    acc = la[np.asarray(a_codes)] @ lw[np.asarray(w_codes)].T
    s = np.asarray(s, dtype=np.float64)
    r = np.asarray(rnorm, dtype=np.float64)
    return acc.astype(np.float64) * s[:, None] * r[None, :] / (alpha_a * alpha_w)


def e4m3_round(x):
    """Round fp64 values to the nearest FP8 E4M3FN value (ties to even);
    magnitudes beyond 448 saturate to 448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    out = np.zeros_like(a)
    nz = a > 0
    e = np.floor(np.log2(a[nz]))
    e = np.maximum(e, -6.0)                  # below 2^-6 the spacing stays 2^-9 (subnormals)
    step = np.exp2(e - 3.0)                  # 3 mantissa bits
    out[nz] = np.rint(a[nz] / step) * step   # np.rint: round half to even
    out = np.minimum(out, 448.0)
    return np.copysign(out, x)


def fp8_levels(levels):
    """(e float64[L], beta): E4M3 values of beta·c, beta = 2^(7 - floor(log2 max|c|))."""
    c = np.asarray(levels, dtype=np.float64)
    beta = np.exp2(7.0 - np.floor(np.log2(np.max(np.abs(c)))))
    return e4m3_round(beta * c), beta


def qlinear_fp8_levels(a_codes, s, levels_a, w_codes, rnorm, levels_w):
    """y = s_m r'_n (sum_k e_w[q_nk] e_a[p_mk]) / (beta_w beta_a) in fp64 (the
    E4M3 products are exact in fp64, so this is the exact sum)."""
    ea, beta_a = fp8_levels(levels_a)
    ew, beta_w = fp8_levels(levels_w)
    acc = ea[np.asarray(a_codes)] @ ew[np.asarray(w_codes)].T
    s = np.asarray(s, dtype=np.float64)
    r = np.asarray(rnorm, dtype=np.float64)
    return acc * s[:, None] * r[None, :] / (beta_a * beta_w)
