"""Seeded synthetic inputs shaped like the source pages' DiT workloads.

This module only draws random tensors; it holds none of the method's
arithmetic, so both the oracle and the CUDA path can be fed from it.  Every
tensor is drawn in fp32 from numpy's PCG64, keyed by a SeedSequence of
integers, and (for BF16 workloads) rounded to bfloat16 with
round-to-nearest-even on the fp32 bit pattern.

Workloads (OrbitQuant §3 evaluates FLUX.1 / Z-Image-Turbo image DiTs and Wan
2.1 video DiTs; INT8-convrot §2 describes a 7B, 32-layer single-stream DiT):

* tiny        d_in = d_out = 256, 64 tokens, fp32; X ~ N(0,1) with 4 channels
              x20; W ~ N(0, 0.02^2) with 1% of entries x10.
* attn_proj   d = 3072, 4608 tokens (64x64 latent patches + 512 text), BF16;
              X Student-t(3) per element with 1% of channels x30;
              W ~ N(0, 0.02^2).
* mlp         up 3072 -> 12288 and down 12288 -> 3072, 4608 tokens, BF16;
              X = GELU(N(0,1)) with 1% of channels x30.
* int8_dit    32 blocks of {q,k,v,o 4096x4096, up 16384x4096, down
              4096x16384}; W ~ N(0, 0.02^2) with 1% of entries x10; X ~ N(0,1)
              BF16, 4096 tokens.
* video       d = 1536 / 8960, 32760 tokens = 21 frames x 1560 patches, BF16;
              Student-t(3) times a per-frame scale ~ U(0.5, 4); generated frame
              by frame so a subset of frames can be drawn alone.
"""

import math

import numpy as np
from scipy.special import erf

# --------------------------------------------------------------------------
# bfloat16 helpers (storage format only)
# --------------------------------------------------------------------------


def bf16_bits(x):
    """fp32 array -> uint16 bfloat16 bit patterns, round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(bits):
    """uint16 bfloat16 bit patterns -> exact fp32 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def to_bf16(x):
    """Round an fp32 array to bfloat16 values (returned as fp32)."""
    return bf16_to_f32(bf16_bits(x))


def rng(*keys):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(keys))))


def _outlier_channels(g, d, frac=0.01):
    n = max(1, math.ceil(frac * d))
    return np.sort(g.choice(d, size=n, replace=False))


def _outlier_entries(g, shape, frac=0.01):
    n = int(round(frac * shape[0] * shape[1]))
    return g.choice(shape[0] * shape[1], size=n, replace=False)


def gaussian_weights(g, n_out, d_in, std=0.02, outlier_frac=0.0, outlier_mult=10.0):
    W = (g.standard_normal((n_out, d_in)) * std).astype(np.float32)
    if outlier_frac > 0:
        idx = _outlier_entries(g, W.shape, outlier_frac)
        W.reshape(-1)[idx] *= np.float32(outlier_mult)
    return W


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

TINY = dict(name="tiny", T=64, d=256, n_out=256, bits_w=4, bits_a=4, seed=0, dtype="f32")
ATTN = dict(name="attn_proj", T=4608, d=3072, n_out=3072, bits_w=4, bits_a=4, seed=0, dtype="bf16")


def tiny(seed=0):
    """64 x 256 fp32 activations (4 channels x20) and a 256 x 256 weight."""
    g = rng(1, seed)
    X = g.standard_normal((64, 256)).astype(np.float32)
    ch = np.sort(g.choice(256, size=4, replace=False))
    X[:, ch] *= np.float32(20.0)
    W = gaussian_weights(g, 256, 256, outlier_frac=0.01, outlier_mult=10.0)
    return {"X": X, "W": W, "outlier_channels": ch}


def student_t_act(T, d, seed, nu=3.0, outlier_frac=0.01, outlier_mult=30.0, key=2):
    g = rng(key, seed, T, d)
    X = g.standard_t(nu, size=(T, d)).astype(np.float32)
    ch = _outlier_channels(g, d, outlier_frac)
    X[:, ch] *= np.float32(outlier_mult)
    return to_bf16(X), ch


def gelu_act(T, d, seed, outlier_frac=0.01, outlier_mult=30.0):
    g = rng(3, seed, T, d)
    Z = g.standard_normal((T, d))
    X = (0.5 * Z * (1.0 + erf(Z / math.sqrt(2.0)))).astype(np.float32)
    ch = _outlier_channels(g, d, outlier_frac)
    X[:, ch] *= np.float32(outlier_mult)
    return to_bf16(X), ch


def attn_proj(seed=0, T=4608, d=3072):
    """Attention-projection shape: Student-t(3) activations, Gaussian weights."""
    X, ch = student_t_act(T, d, seed)
    W = to_bf16(gaussian_weights(rng(4, seed, d), d, d))
    return {"X": X, "W": W, "outlier_channels": ch}


def mlp(seed=0, T=4608, d=3072, d_ff=12288):
    X_up, _ = gelu_act(T, d, seed)
    X_dn, _ = gelu_act(T, d_ff, seed + 1)
    W_up = to_bf16(gaussian_weights(rng(5, seed, d_ff, d), d_ff, d))
    W_dn = to_bf16(gaussian_weights(rng(6, seed, d, d_ff), d, d_ff))
    return {"X_up": X_up, "X_dn": X_dn, "W_up": W_up, "W_dn": W_dn}


INT8_DIT_SHAPES = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096),
                   ("o", 4096, 4096), ("up", 16384, 4096), ("down", 4096, 16384)]


def int8_dit_weight(block, name, seed=0):
    """One weight of the 32-block, 7B single-stream DiT (BF16 values)."""
    shapes = {n: (o, i) for n, o, i in INT8_DIT_SHAPES}
    n_out, d_in = shapes[name]
    key = [n for n, _, _ in INT8_DIT_SHAPES].index(name)
    W = gaussian_weights(rng(7, seed, block, key), n_out, d_in,
                         outlier_frac=0.01, outlier_mult=10.0)
    return to_bf16(W)


def int8_dit_act(d_in, seed=0, T=4096):
    return to_bf16(rng(8, seed, d_in).standard_normal((T, d_in)).astype(np.float32))


VIDEO_FRAMES = 21
VIDEO_PATCHES = 30 * 52


def video_act(d, layer, frames=None, seed=0):
    """Video-DiT activations for the given frames (default: all 21)."""
    frames = range(VIDEO_FRAMES) if frames is None else frames
    out = []
    for f in frames:
        g = rng(9, seed, layer, d, f)
        scale = np.float32(g.uniform(0.5, 4.0))
        out.append(g.standard_t(3.0, size=(VIDEO_PATCHES, d)).astype(np.float32) * scale)
    return to_bf16(np.concatenate(out, axis=0))


def video_weight(n_out, d_in, layer, seed=0):
    return to_bf16(gaussian_weights(rng(10, seed, layer, n_out, d_in), n_out, d_in))
