"""The rotation fused into the producing matmul (oracle side), fp64.

OrbitQuant §6.2 ("performance below expectations") suggests fusing the
rotation with the matrix-multiply kernels.  What the fused layer computes has a
plain definition -- the producing W8A16 layer (INT8-convrot §4), an
element-wise activation, then the next layer's rotation (OrbitQuant §2.2 step
1) -- so the oracle is that composition written out, on the weights in their
ORIGINAL row order (the fused kernel's reordering of the rows by the next
layer's permutation is what the parity test checks):

    y       = qlinear_int8(x', q, scale)          y[m, j] = scale_j sum_k q_jk x'_mk
    x_next  = act(y)                               act = identity or GELU
    x'_next = Pi_next x_next                       (rotate_only, before BF16 rounding)

The same with the code layer of OrbitQuant §2.2 as the producer (y = s_m r'_n
sum_k C_w[q_nk] C_a[p_mk]), whose output the next layer then quantises from
x'_next with steps 2-4 only (quant.quantize_rotated).

GELU is the exact one (the page's synthetic MLP inputs are "GELU-shaped"; no
page fixes a variant): gelu(y) = y Phi(y) = 0.5 y (1 + erf(y / sqrt 2)),
evaluated as 0.5 y erfc(-y / sqrt 2), which has no cancellation for negative y.
"""

import math

import numpy as np
from scipy.special import erfc

from .qlinear import qlinear, qlinear_int8
from .quant import rotate_only


def gelu(y):
    """y Phi(y) = 0.5 y erfc(-y / sqrt 2) in fp64."""
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * erfc(-y / math.sqrt(2.0))


def qlinear_int8_rotate_next(xr, q, scale, Pi_next, activation="gelu"):
    """x'_next = Pi_next act(qlinear_int8(x', q, scale)) in fp64 (unrounded)."""
    y = qlinear_int8(xr, q, scale)
    x = gelu(y) if activation == "gelu" else y
    return rotate_only(x, Pi_next)["xr"]


def qlinear_rotate_next(a_codes, s, levels_a, w_codes, rnorm, levels_w, Pi_next, activation="gelu"):
    """x'_next = Pi_next act(qlinear(codes...)) in fp64 (unrounded)."""
    y = qlinear(a_codes, s, levels_a, w_codes, rnorm, levels_w)
    x = gelu(y) if activation == "gelu" else y
    return rotate_only(x, Pi_next)["xr"]
