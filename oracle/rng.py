"""Random draws of the RPBH transform (oracle side).

OrbitQuant §2.3 defines Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) · P_pi with
Rademacher signs D_i and a random permutation P_pi, and §6.3 asks that the
permutation be reproducible across platforms.  The pages name no generator,
this oracle fixes one (a reading; the pages cannot pin the choice):

* generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): a Weyl sequence with
  increment 0x9E3779B97F4A7C15 followed by the 64-bit finaliser
  z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27; z *= 0x94D049BB133111EB;
  z ^= z>>31.  The state starts at ``seed``.
* permutation: Fisher-Yates on the identity, i = d-1 down to 1, swapping
  entries i and j = floor(u * (i+1) / 2**64) where u is the next output
  (multiply-high range reduction, D. Lemire 2019, without the rejection step).
* signs: the following d outputs; D_k = -1 when the top bit of output k is set.

The oracle writes this from the published definition; the C++ side writes it
again on its own.  Pure Python integers keep every step exact.
"""

import numpy as np

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def splitmix64(seed, n):
    """First ``n`` outputs of SplitMix64 started at ``seed`` (list of ints)."""
    s = seed & _M64
    out = []
    for _ in range(n):
        s = (s + _GAMMA) & _M64
        z = s
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
        out.append(z ^ (z >> 31))
    return out


def rpbh_draw(d, seed):
    """Permutation pi (int64[d]) and signs D (int64[d], values +-1) for Pi_d.

    Convention: (P_pi x)_k = x_{pi[k]}; D_k multiplies coordinate k of the
    permuted vector, matching the factor order blkdiag(H D_i) · P_pi.
    """
    if d < 1:
        raise ValueError("d must be positive")
    u = splitmix64(seed, (d - 1) + d)
    perm = list(range(d))
    for n, i in enumerate(range(d - 1, 0, -1)):
        j = (u[n] * (i + 1)) >> 64
        perm[i], perm[j] = perm[j], perm[i]
    signs = [-1 if (x >> 63) else 1 for x in u[d - 1:]]
    return np.array(perm, dtype=np.int64), np.array(signs, dtype=np.int64)
