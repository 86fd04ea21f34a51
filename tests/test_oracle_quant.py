"""Pins of the oracle's quantisation steps and the quantised linear layers.

* codes against a brute-force nearest-level search (ties to the upper level);
* the packed bit layout against a hand-made fixture, and pack/unpack round trip;
* norm/direction identities, the zero row, INT8 bounds;
* the qualitative claims of the pages: rotation spreads outliers so the
  coordinates look N(0, 1/d) (OrbitQuant §1, §2.3) and rotated INT8 has lower
  error than naive INT8 on outlier weights (INT8-convrot §2);
* qlinear against a pure-Python triple loop and a closed-form special case.
"""

import numpy as np
import pytest
from scipy import stats

import oracle
import synth
from conftest import golden_rows


def _brute_force_codes(v, levels):
    out = np.empty(v.shape, dtype=np.int64)
    for idx, x in np.ndenumerate(v):
        best, best_d = 0, np.inf
        for j, c in enumerate(levels):
            dist = abs(x - c)
            if dist <= best_d:          # '<=' keeps the upper index on a tie
                best, best_d = j, dist
        out[idx] = best
    return out


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codes_equal_brute_force_nearest_level(bits):
    levels, bounds = oracle.lloydmax_table(16, bits)
    g = np.random.default_rng(bits)
    v = np.concatenate([g.standard_normal(400) * 0.25, levels, [0.0]])
    v = v[np.min(np.abs(v[:, None] - bounds[None, :]), axis=1) > 1e-12]
    assert np.array_equal(oracle.assign_codes(v, bounds), _brute_force_codes(v, levels))
    # On a boundary the two neighbours are equally near (up to the rounding of
    # the fp64 midpoint); the boundary count takes the upper one.
    on = oracle.assign_codes(bounds, bounds)
    assert np.array_equal(on, np.arange(1, len(levels)))
    bf = _brute_force_codes(bounds, levels)
    assert np.all((bf == on) | (bf == on - 1))


def test_pack_layout_fixture():
    for row in golden_rows("pack_layout.txt"):
        bits = int(row[0])
        codes = np.array([[int(v) for v in row[1].split()]])
        expect = np.array([[int(v, 16) for v in row[2].split()]], dtype=np.uint8)
        assert np.array_equal(oracle.pack_codes(codes, bits), expect)
        assert np.array_equal(oracle.unpack_codes(expect, bits, codes.shape[1]), codes)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_pack_roundtrip(bits):
    g = np.random.default_rng(bits)
    codes = g.integers(0, 2 ** bits, size=(3, 128))
    packed = oracle.pack_codes(codes, bits)
    assert packed.shape == (3, 128 * bits // 8)
    assert np.array_equal(oracle.unpack_codes(packed, bits, 128), codes)
    # independent packer: one big Python integer per row
    for r in range(3):
        acc = 0
        for j, c in enumerate(codes[r]):
            acc |= int(c) << (j * bits)
        assert bytes(packed[r]) == acc.to_bytes(128 * bits // 8, "little")


def _tiny_setup(bits=4, seed=0):
    data = synth.tiny()
    perm, signs = oracle.rpbh_draw(256, seed)
    Pi = oracle.rpbh_matrix(perm, signs)
    levels, bounds = oracle.lloydmax_table(256, bits)
    return data, Pi, levels, bounds


def test_quantize_act_identities_and_zero_row():
    data, Pi, levels, bounds = _tiny_setup()
    X = data["X"].astype(np.float64).copy()
    X[5] = 0.0
    out = oracle.quantize_act(X, Pi, bounds)
    n = np.linalg.norm(X, axis=1)
    assert np.allclose(out["norms"], n, rtol=1e-13, atol=0)       # ||Pi x|| = ||x||
    assert np.allclose(out["v"] * (out["norms"] + oracle.EPS)[:, None], out["xr"], rtol=1e-14, atol=1e-300)
    assert out["norms"][5] == 0.0 and np.all(out["codes"][5] == 8)
    # reconstruction error of s * C[codes] at 4 bits is near the Lloyd-Max distortion
    rec = levels[out["codes"]] * out["norms"][:, None]
    keep = np.arange(64) != 5
    err = np.sum((rec[keep] - out["xr"][keep]) ** 2, axis=1) / n[keep] ** 2
    assert np.all(err < 0.03)


def test_rotation_spreads_outliers():
    # OrbitQuant §2.3: the block Hadamard spreads an outlier over its block of
    # 64 (peak down by ~sqrt(64)), and over random permutations every output
    # coordinate has variance ~1/d.  §1: without outlier channels the rotated
    # coordinates look Gaussian (kurtosis ~3).  Statistical checks of the why.
    d, T = 512, 16
    X, _ = synth.student_t_act(T, d, seed=0)
    raw = X / np.linalg.norm(X, axis=1, keepdims=True)
    bounds = oracle.lloydmax_table(d, 4)[1]
    acc = np.zeros(d)
    for seed in range(60):
        perm, signs = oracle.rpbh_draw(d, seed)
        v = oracle.quantize_act(X, oracle.rpbh_matrix(perm, signs), bounds)["v"]
        if seed == 0:
            assert np.max(np.abs(v)) < np.max(np.abs(raw)) / 4
        acc += np.mean(v * v, axis=0)
    per_coord = acc / 60 * d
    assert abs(np.mean(per_coord) - 1) < 1e-9
    assert np.all(np.abs(per_coord - 1) < 0.5)
    g = np.random.default_rng(0)
    Y = g.standard_normal((64, 3072)) * g.uniform(0.5, 4, (64, 1))
    perm, signs = oracle.rpbh_draw(3072, 0)
    vy = oracle.quantize_act(Y, oracle.rpbh_matrix(perm, signs), oracle.lloydmax_table(3072, 4)[1])["v"]
    assert abs(stats.kurtosis(vy.ravel(), fisher=False) - 3) < 0.1


def test_int8_per_tensor_bounds():
    # one scale for the tensor: exactly one |q| = 127 in the row holding the
    # tensor's largest |w'|, the dequantisation error bound, and the scale
    # equals the largest per-row scale (max commutes with the monotone /127)
    data, Pi, _, _ = _tiny_setup()
    W = data["W"].astype(np.float64)
    W[3] = 0.0
    t = oracle.quantize_weights_int8(W, Pi, per_tensor=True)
    c = oracle.quantize_weights_int8(W, Pi)
    q, scale, wr = t["q"], t["scale"], t["wr"]
    assert np.all(scale == scale[0]) and scale[0] == np.max(c["scale"])
    assert np.all(np.abs(q) <= 127)
    i, _ = np.unravel_index(np.argmax(np.abs(wr)), wr.shape)
    assert np.max(np.abs(q[i])) == 127
    assert np.all(q[3] == 0)
    assert np.all(np.abs(wr - scale[0] * q) <= scale[0] * (0.5 + 1e-6))
    # with a coarser grid the per-tensor error is at least the per-channel one
    assert np.linalg.norm(wr - scale[0] * q) >= np.linalg.norm(wr - c["scale"][:, None] * c["q"])


def test_int8_asymmetric_zero_point_pins():
    # the range [min, max] (widened to hold 0) is cut into 255 steps: codes
    # stay in 0..255, 0 maps to exactly the zero point, every value is within
    # half a step (one step where the top code clips), and on rows whose
    # values are mostly positive the zero point beats the symmetric scheme
    data, Pi, _, _ = _tiny_setup()
    W = data["W"].astype(np.float64)
    W[3] = 0.0
    a = oracle.quantize_weights_int8_asym(W, Pi)
    q, scale, z, wr = a["q"], a["scale"], a["z"], a["wr"]
    assert q.min() >= 0 and q.max() <= 255
    assert np.all(q[3] == 0) and scale[3] == 0 and z[3] == 0
    nz = scale > 0
    deq = scale[:, None] * (q - z[:, None])
    err = np.abs(wr - deq)
    inner = (q > 0) & (q < 255)
    half = 0.5 * scale[:, None] * (1 + 1e-9)
    assert np.all((err <= half)[nz & inner.any(axis=1)][inner[nz & inner.any(axis=1)]])
    assert np.all(err[nz] <= 2 * half[nz])
    # zero is representable: the code of 0 is z
    zero_codes = np.clip(np.rint(0.0 / np.where(scale > 0, scale, 1.0)) + z, 0, 255)
    assert np.array_equal(zero_codes, z)
    # skewed rows (shifted up): the zero point uses the whole range
    Ws = oracle.rpbh_apply(Pi.T, np.abs(oracle.rpbh_apply(Pi, W)) + 0.01)   # rotated rows all positive
    asym = oracle.quantize_weights_int8_asym(Ws, Pi)
    sym = oracle.quantize_weights_int8(Ws, Pi)
    e_asym = np.linalg.norm(asym["wr"] - asym["scale"][:, None] * (asym["q"] - asym["z"][:, None]))
    e_sym = np.linalg.norm(sym["wr"] - sym["scale"][:, None] * sym["q"])
    assert e_asym < 0.6 * e_sym


def test_int8_bounds_and_rotation_helps():
    data, Pi, _, _ = _tiny_setup()
    W = data["W"].astype(np.float64)
    W[3] = 0.0
    out = oracle.quantize_weights_int8(W, Pi)
    q, scale, wr = out["q"], out["scale"], out["wr"]
    assert np.all(np.abs(q) <= 127)
    nz = scale > 0
    assert np.all(np.max(np.abs(q[nz]), axis=1) == 127)
    assert np.all(q[3] == 0) and scale[3] == 0
    assert np.all(np.abs(wr - scale[:, None] * q) <= scale[:, None] * (0.5 + 1e-6) + 1e-300)
    naive = oracle.quantize_weights_int8(W)
    x = data["X"].astype(np.float64)
    ref = x @ W.T
    y_rot = oracle.qlinear_int8(oracle.rpbh_apply(Pi, x), q, scale)
    y_naive = oracle.qlinear_int8(x, naive["q"], naive["scale"])
    e_rot = np.linalg.norm(y_rot - ref) / np.linalg.norm(ref)
    e_naive = np.linalg.norm(y_naive - ref) / np.linalg.norm(ref)
    assert e_rot < 0.6 * e_naive


def test_weights_lloydmax_norms_bf16():
    data, Pi, _, bounds = _tiny_setup()
    out = oracle.quantize_weights_lloydmax(data["W"], Pi, bounds)
    r = out["rnorm"]
    assert np.allclose(r, np.linalg.norm(data["W"].astype(np.float64), axis=1), rtol=1e-13)
    rb = out["rnorm_bf16"]
    assert np.all(np.abs(rb - r) <= np.abs(r) * 2.0 ** -8)   # half an ulp of an 8-bit significand
    assert np.array_equal(rb, synth.to_bf16(rb.astype(np.float32)).astype(np.float64))


def test_round_to_bf16_matches_bit_rounding():
    g = np.random.default_rng(9)
    x = (g.standard_normal(10000) * 10.0 ** g.integers(-5, 5, 10000)).astype(np.float32)
    assert np.array_equal(oracle.round_to_bf16(x.astype(np.float64)),
                          synth.to_bf16(x).astype(np.float64))


def test_qlinear_triple_loop_and_closed_form():
    g = np.random.default_rng(5)
    la, _ = oracle.lloydmax_table(64, 3)
    lw, _ = oracle.lloydmax_table(64, 2)
    M, N, K = 3, 4, 64
    pa = g.integers(0, 8, (M, K))
    pw = g.integers(0, 4, (N, K))
    s = g.uniform(0.5, 2, M)
    r = g.uniform(0.5, 2, N)
    y = oracle.qlinear(pa, s, la, pw, r, lw)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += lw[pw[n, k]] * la[pa[m, k]]
            assert abs(y[m, n] - s[m] * r[n] * acc) < 1e-12
    yc = oracle.qlinear(np.full((1, K), 5), [2.0], la, np.full((1, K), 1), [3.0], lw)
    assert abs(yc[0, 0] - 2.0 * 3.0 * K * la[5] * lw[1]) < 1e-12


def test_qlinear_approximates_dense_linear():
    data, Pi, _, _ = _tiny_setup()
    X, W = data["X"].astype(np.float64), data["W"].astype(np.float64)
    ref = X @ W.T
    for bits, tol in ((4, 0.2), (8, 0.01)):
        lv, bd = oracle.lloydmax_table(256, bits)
        a = oracle.quantize_act(X, Pi, bd)
        w = oracle.quantize_weights_lloydmax(W, Pi, bd)
        y = oracle.qlinear(a["codes"], a["norms"], lv, w["codes"], w["rnorm_bf16"], lv)
        assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < tol
