"""Rotate-then-quantise steps (oracle side).

OrbitQuant §2.2 (online activations), per token x:
  1. x' = Pi_d x
  2. s  = ||x'||_2
  3. x~ = x' / (s + eps)
  4. codes = Q_b(x~) with the Lloyd-Max codebook of N(0, 1/d)
  5. (reconstruction x^ = s · C[codes] -- used by the quantised linear)
OrbitQuant §2.1 (offline weights), per output row w_i: the same steps on
w'_i = Pi_d w_i with the norm r'_i kept in BF16.
INT8-convrot §4 / rotated-model explainer §4 / INT8 image-text model: rotate,
compute a scale, q = round(W_rot / s).

Readings where the pages are silent (each also listed in the design notes):
* eps = 1e-12 (§2.2 names eps without a value); the weight rows use the same
  guard, which only matters for an all-zero row.
* the code of a coordinate v is #{j : t_j <= v} over the sorted boundaries t
  (nearest level, ties to the upper cell).
* the norm s is stored as fp32; r' as BF16 (§2.1), rounded from the exact norm.
* INT8: symmetric per output channel, scale = max|w'|/127 stored as fp32,
  q = clamp(round-half-even(w'/scale), -127, 127); an all-zero row has scale 0
  and q = 0.
* packing: code j of a row occupies bits [j*b, j*b + b) of the row's
  little-endian bitstream (LSB first); the row pitch is d*b/8 bytes.
"""

import numpy as np

from .bf16 import round_to_bf16
from .rpbh import rpbh_apply

EPS = 1e-12


def assign_codes(v, bounds):
    """Code of each coordinate: the number of boundaries t_j <= v."""
    return np.searchsorted(np.asarray(bounds), np.asarray(v), side="right").astype(np.int64)


def pack_codes(codes, bits):
    """Pack int codes [R, d] (values < 2**bits) into uint8 [R, d*bits/8]."""
    codes = np.asarray(codes, dtype=np.int64)
    R, d = codes.shape
    if (d * bits) % 8:
        raise ValueError("d*bits must be a multiple of 8")
    if np.any(codes < 0) or np.any(codes >= (1 << bits)):
        raise ValueError("code out of range")
    planes = (codes[:, :, None] >> np.arange(bits)) & 1          # LSB first
    return np.packbits(planes.reshape(R, d * bits).astype(np.uint8),
                       axis=1, bitorder="little")


def unpack_codes(packed, bits, d):
    """Inverse of pack_codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    R = packed.shape[0]
    flat = np.unpackbits(packed, axis=1, bitorder="little")[:, : d * bits]
    planes = flat.reshape(R, d, bits).astype(np.int64)
    return np.sum(planes << np.arange(bits), axis=2)


def _direction_quantise(Xr, bounds, eps):
    norms = np.sqrt(np.sum(Xr * Xr, axis=1))
    V = Xr / (norms + eps)[:, None]
    return assign_codes(V, bounds), norms, V


def quantize_rotated(Xr, bounds, eps=EPS):
    """OrbitQuant §2.2 steps 2-4 on rows that are already rotated (x' = Pi x
    computed elsewhere, e.g. by the producing layer): s = ||x'||, codes of
    x'/(s + eps).

    Returns dict(codes int64[T,d], norms fp64[T], v fp64[T,d]).
    """
    Xr = np.asarray(Xr, dtype=np.float64)
    codes, norms, V = _direction_quantise(Xr, bounds, eps)
    return {"codes": codes, "norms": norms, "v": V}


def quantize_act(X, Pi, bounds, eps=EPS):
    """OrbitQuant §2.2 steps 1-4 on each row of X.

    Returns dict(codes int64[T,d], norms fp64[T], v fp64[T,d], xr fp64[T,d]);
    the stored norm is fp32(norms).
    """
    Xr = rpbh_apply(Pi, X)
    codes, norms, V = _direction_quantise(Xr, bounds, eps)
    return {"codes": codes, "norms": norms, "v": V, "xr": Xr}


def quantize_weights_lloydmax(W, Pi, bounds, eps=EPS):
    """OrbitQuant §2.1 steps 1-3 on each output row of W (W' = W Pi^T).

    Returns dict(codes, rnorm (exact fp64), rnorm_bf16, v, wr).
    """
    Wr = rpbh_apply(Pi, W)
    codes, norms, V = _direction_quantise(Wr, bounds, eps)
    return {"codes": codes, "rnorm": norms, "rnorm_bf16": round_to_bf16(norms),
            "v": V, "wr": Wr}


def quantize_weights_int8(W, Pi=None, per_tensor=False):
    """Symmetric INT8 of the rotated rows (Pi=None: naive), one scale per
    output channel (INT8-convrot §4), or with per_tensor=True one scale for
    the whole tensor (INT8 image-text model page, "how it works"), repeated
    per row.

    Returns dict(q int64[N,d], scale fp32-valued fp64[N], ratio w'/scale, wr).
    """
    Wr = np.asarray(W, dtype=np.float64) if Pi is None else rpbh_apply(Pi, W)
    amax = np.max(np.abs(Wr), axis=1)
    if per_tensor:
        amax = np.full_like(amax, np.max(amax))
    scale = (amax / 127.0).astype(np.float32).astype(np.float64)
    safe = np.where(scale > 0, scale, 1.0)
    ratio = Wr / safe[:, None]
    q = np.clip(np.rint(ratio), -127, 127).astype(np.int64)
    q[scale == 0] = 0
    ratio[scale == 0] = 0.0
    return {"q": q, "scale": scale, "ratio": ratio, "wr": Wr}


def quantize_weights_int8_asym(W, Pi=None):
    """Asymmetric per-output-channel INT8 with a zero point (INT8-convrot,
    "the quantized model file": a scale and a zero point per channel).  The
    row's range is widened to contain 0 and cut into 255 steps:
    scale = (hi - lo)/255, z = clip(round(-lo/scale), 0, 255),
    q = clip(round(w'/scale) + z, 0, 255), w' ~ scale (q - z).

    Returns dict(q int64[N,d] in 0..255, scale fp32-valued fp64[N], z int64[N],
    ratio w'/scale, zratio -lo/scale, wr).
    """
    Wr = np.asarray(W, dtype=np.float64) if Pi is None else rpbh_apply(Pi, W)
    hi = np.maximum(np.max(Wr, axis=1), 0.0)
    lo = np.minimum(np.min(Wr, axis=1), 0.0)
    scale = ((hi - lo) / 255.0).astype(np.float32).astype(np.float64)
    safe = np.where(scale > 0, scale, 1.0)
    zratio = np.where(scale > 0, -lo / safe, 0.0)
    z = np.clip(np.rint(zratio), 0, 255).astype(np.int64)
    ratio = np.where(scale[:, None] > 0, Wr / safe[:, None], 0.0)
    q = np.clip(np.rint(ratio) + z[:, None], 0, 255).astype(np.int64)
    q[scale == 0] = 0
    return {"q": q, "scale": scale, "z": z, "ratio": ratio, "zratio": zratio, "wr": Wr}


def rotate_only(X, Pi):
    """x' = Pi x rounded to BF16: the activation operand of the INT8 path
    (INT8-convrot §3/§4: the transform information is used at inference)."""
    xr = rpbh_apply(Pi, X)
    return {"xr": xr, "xr_bf16": round_to_bf16(xr)}
