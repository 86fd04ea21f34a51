"""Round fp64 values to the nearest bfloat16 (oracle side).

bfloat16 keeps 8 significant bits and fp32's exponent range.  This rounds the
exact fp64 value once, to nearest with ties to even, in the normal range; it is
used where the method stores a quantity as BF16 (OrbitQuant §2.1: the row norms
r') and for the rotate-only BF16 output of the INT8 path.
"""

import numpy as np

_BF16_MIN_NORMAL = 2.0 ** -126


def round_to_bf16(x):
    x = np.asarray(x, dtype=np.float64)
    nz = x != 0
    if np.any(np.abs(x[nz]) < _BF16_MIN_NORMAL) or not np.all(np.isfinite(x)):
        raise ValueError("round_to_bf16 handles finite normal-range values only")
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # np.rint: ties to even
