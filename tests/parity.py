"""Comparison rules between the CUDA path and the oracle (test helpers).

Where floating point decides an integer the two sides decide in different
precisions (the kernel in fp32, the oracle in fp64), so exact agreement is
required everywhere except inside a narrow band around each decision point:

* codes: a coordinate may differ only if its oracle value v lies within
  1e-6 * max(|t_j|, sigma) of a boundary t_j (sigma = 1/sqrt(d)); the two
  codes must then be neighbours;
* INT8: only where w'/scale lies within 1e-6 * max(|k + 1/2|, 1) of a
  half-integer, by one step;
* BF16 roundings (rotate-only output, BF16 row norms): only where the exact
  value lies within 1e-6 relative of a rounding midpoint, by one BF16 ulp.

Every mismatch inside the band is counted and returned so tests can report it.
"""

import numpy as np

import oracle
import synth

BAND = 1e-6


def torch_bf16(x_f32, device="cuda"):
    import torch
    bits = synth.bf16_bits(x_f32)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)


def bf16_to_numpy(t):
    import torch
    return synth.bf16_to_f32(t.detach().view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def near_boundary(v, bounds, sigma, rel=BAND):
    bounds = np.asarray(bounds)
    idx = np.searchsorted(bounds, v)
    near = np.zeros(v.shape, dtype=bool)
    for j in (idx - 1, idx):
        jj = np.clip(j, 0, len(bounds) - 1)
        t = bounds[jj]
        near |= (j >= 0) & (j < len(bounds)) & (np.abs(v - t) <= rel * np.maximum(np.abs(t), sigma))
    return near


def check_codes(gpu_codes, ora_codes, v, bounds, d):
    """Assert the band rule; return (n_mismatch, n_in_band)."""
    gpu_codes = np.asarray(gpu_codes)
    mism = gpu_codes != ora_codes
    near = near_boundary(v, bounds, 1.0 / np.sqrt(d))
    bad = mism & ~near
    if np.any(bad):
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{int(bad.sum())} code mismatches outside the band; first at {tuple(i)}: gpu "
            f"{gpu_codes[tuple(i)]} oracle {ora_codes[tuple(i)]} v {v[tuple(i)]!r}")
    assert np.all(np.abs(gpu_codes[mism].astype(np.int64) - ora_codes[mism]) == 1)
    return int(mism.sum()), int(near.sum())


def check_rel(gpu, ref, rtol, what):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-300)
    worst = float(np.max(err)) if err.size else 0.0
    assert worst <= rtol, f"{what}: worst relative error {worst:.3e} > {rtol:.1e}"
    return worst


def _bf16_midpoint_near(x, rel=BAND):
    """True where fp64 x lies within rel of a BF16 rounding midpoint."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    scaled = np.ldexp(m, 8)                 # 8 significant bits before the point
    frac = scaled - np.floor(scaled)
    return np.abs(frac - 0.5) <= rel * np.abs(scaled)


def check_bf16_rounding(gpu_vals, exact, what):
    """gpu_vals: BF16 values from the kernel; exact: fp64 values it rounds."""
    ref = oracle.round_to_bf16(exact)
    mism = gpu_vals != ref
    near = _bf16_midpoint_near(exact)
    bad = mism & ~near
    assert not np.any(bad), f"{what}: {int(bad.sum())} BF16 roundings differ outside the band"
    ulp = np.ldexp(1.0, np.frexp(ref)[1] - 8)
    assert np.all(np.abs(gpu_vals[mism] - ref[mism]) <= ulp[mism] * 1.0001)
    return int(mism.sum())


def check_int8(gpu_q, gpu_scale, ora):
    """INT8 rows: scales to 1e-6 relative, q with the half-integer band."""
    scale_ref = ora["scale"]
    assert np.all((gpu_scale == 0) == (scale_ref == 0))
    check_rel(gpu_scale[scale_ref > 0], scale_ref[scale_ref > 0], 1e-6, "int8 scale")
    q_ref = ora["q"]
    mism = gpu_q != q_ref
    ratio = ora["ratio"]
    k = np.floor(ratio)
    near = np.abs(ratio - (k + 0.5)) <= BAND * np.maximum(np.abs(k + 0.5), 1.0)
    bad = mism & ~near
    assert not np.any(bad), f"{int(bad.sum())} int8 values differ outside the band"
    assert np.all(np.abs(gpu_q[mism].astype(np.int64) - q_ref[mism]) == 1)
    return int(mism.sum())


def check_int8_asym(gpu_q, gpu_scale, gpu_z, ora):
    """Asymmetric INT8 rows: scales to 1e-6 relative; the zero point and every
    code exact except where the deciding ratio (-lo/scale, w'/scale) lies within
    the half-integer band, by one step (a row whose zero point moved is then
    allowed to move as a whole)."""
    scale_ref, z_ref = ora["scale"], ora["z"]
    assert np.all((gpu_scale == 0) == (scale_ref == 0))
    check_rel(gpu_scale[scale_ref > 0], scale_ref[scale_ref > 0], 1e-6, "int8 asym scale")
    zr = ora["zratio"]
    zk = np.floor(zr)
    z_near = np.abs(zr - (zk + 0.5)) <= BAND * np.maximum(np.abs(zk + 0.5), 1.0)
    zmis = gpu_z != z_ref
    assert not np.any(zmis & ~z_near), "zero points differ outside the band"
    assert np.all(np.abs(gpu_z[zmis].astype(np.int64) - z_ref[zmis]) <= 1)
    q_ref = ora["q"] + (gpu_z.astype(np.int64) - z_ref)[:, None]
    q_ref = np.clip(q_ref, 0, 255)
    mism = gpu_q != q_ref
    ratio = ora["ratio"]
    k = np.floor(ratio)
    near = np.abs(ratio - (k + 0.5)) <= BAND * np.maximum(np.abs(k + 0.5), 1.0)
    bad = mism & ~near
    assert not np.any(bad), f"{int(bad.sum())} asymmetric int8 values differ outside the band"
    assert np.all(np.abs(gpu_q[mism].astype(np.int64) - q_ref[mism]) == 1)
    return int(mism.sum())


def rel_frobenius(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


# --------------------------------------------------------------------------
# poisoned output buffers: every output the kernels are asked to write starts
# as a value they never produce (0xAB bytes for codes and int8, NaN for BF16
# and fp32), so a row or tile a kernel leaves unwritten fails its comparison
# instead of passing on whatever stale bytes the allocator returned
# --------------------------------------------------------------------------

POISON_BYTE = 0xAB


def poison(shape, dtype, device="cuda"):
    import torch
    if dtype in (torch.uint8, torch.int8):
        t = torch.empty(shape, dtype=torch.uint8, device=device).fill_(POISON_BYTE)
        return t if dtype == torch.uint8 else t.view(torch.int8)
    if dtype in (torch.float32, torch.bfloat16, torch.float16):
        return torch.full(shape, float("nan"), dtype=dtype, device=device)
    if dtype == torch.int32:
        return torch.full(shape, -0x54545455, dtype=dtype, device=device)
    raise TypeError(f"no poison for {dtype}")
