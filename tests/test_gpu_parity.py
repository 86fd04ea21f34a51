"""CUDA path vs oracle, element by element, through the C ABI (needs a B200).

Small cases run the oracle on every row; the full-size workloads run the
kernel on the whole batch and compare sampled rows (the oracle multiplies by
the dense d x d rotation, so it computes sampled tokens one by one).  The
comparison rules (exact outside a 1e-6 band around each decision point) are
in tests/parity.py.
"""

import numpy as np
import pytest

import oracle
import synth
from parity import (bf16_to_numpy, check_bf16_rounding, check_codes, check_int8, check_int8_asym, check_rel,
                    poison, rel_frobenius, torch_bf16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_bit_ptq_b200 as rbq  # noqa: E402

NORM_RTOL = 1e-5          # fp32 norm vs fp64 (the stated norm tolerance)
QLINEAR_RTOL = 4e-3       # rel. Frobenius, fp16 operands + BF16 output (bar: 2e-2)
QLINEAR8_RTOL = 3e-3      # rel. Frobenius, exact operands + BF16 output (bar: 2e-2)


def _dense(x, dtype):
    if dtype == "bf16":
        return torch_bf16(x)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _rpbh(d, seed):
    """Library handle plus the oracle's Pi (dense matrix, or (perm, signs) for
    widths whose dense matrix is applied in row chunks)."""
    perm, signs = oracle.rpbh_draw(d, seed)
    Pi = oracle.rpbh_matrix(perm, signs) if d <= 4096 else (perm, signs)
    return rbq.RPBH(d, seed), Pi


def _unpack(t, bits, d):
    return oracle.unpack_codes(t.cpu().numpy(), bits, d)


# Library calls with poisoned outputs (see parity.poison): every element the
# comparison reads must have been written by the kernel.

def rq_act(r, X, bits):
    T, d = X.shape
    return rbq.rotate_quantize_act(r, X, bits, codes=poison((T, d * bits // 8), torch.uint8),
                                   norms=poison((T,), torch.float32))


def rot_act(r, X, norms=None):
    return rbq.rotate_act(r, X, out=poison(tuple(X.shape), torch.bfloat16), norms=norms)


def qweights(r, W, bits, mode="lloydmax"):
    N, d = W.shape
    if mode == "lloydmax":
        return rbq.quantize_weights(r, W, bits, mode, out=poison((N, d * bits // 8), torch.uint8),
                                    aux=poison((N,), torch.bfloat16))
    return rbq.quantize_weights(r, W, bits, mode, out=poison((N, d), torch.int8), aux=poison((N,), torch.float32))


def _layer(fn, a_codes, s, ba, w_codes, rn, bw, K):
    return fn(a_codes, s, ba, w_codes, rn, bw, K,
              out=poison((a_codes.shape[0], w_codes.shape[0]), torch.bfloat16))


def qlin(a_codes, s, ba, w_codes, rn, bw, K):
    return _layer(rbq.qlinear, a_codes, s, ba, w_codes, rn, bw, K)


def qlin_i8(a_codes, s, ba, w_codes, rn, bw, K):
    return _layer(rbq.qlinear_int8_levels, a_codes, s, ba, w_codes, rn, bw, K)


def qlin_fp8(a_codes, s, ba, w_codes, rn, bw, K):
    return _layer(rbq.qlinear_fp8_levels, a_codes, s, ba, w_codes, rn, bw, K)


def qlin_int8(xr, q, sc):
    return rbq.qlinear_int8(xr, q, sc, out=poison((xr.shape[0], q.shape[0]), torch.bfloat16))


def _act_parity(X, d, bits, seed=0, dtype="bf16", rows=None, Pi=None, r=None):
    """Run the kernel on all of X; compare rows `rows` (default all) with the oracle."""
    if r is None:
        r, Pi = _rpbh(d, seed)
    xt = _dense(X, dtype)
    codes, norms = rq_act(r, xt, bits)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    levels, bounds = oracle.lloydmax_table(d, bits)
    ora = oracle.quantize_act(X[rows].astype(np.float64), Pi, bounds)
    g_codes = _unpack(codes[torch.as_tensor(rows).cuda()], bits, d)
    n_mis, n_band = check_codes(g_codes, ora["codes"], ora["v"], bounds, d)
    check_rel(norms.cpu().numpy()[rows], ora["norms"], NORM_RTOL, "norms")
    return codes, norms, n_mis, n_band


# --------------------------------------------------------------------------
# rotate_quantize_act
# --------------------------------------------------------------------------

def test_tiny_w4a4_activations():
    data = synth.tiny()
    _act_parity(data["X"], 256, 4, dtype="f32")


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_all_bit_widths_ragged_tokens(bits, dtype):
    X, _ = synth.student_t_act(257, 512, seed=bits)      # 257: ragged against any grouping
    _act_parity(X, 512, bits, seed=3, dtype=dtype)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_fast_path_all_bit_widths(bits):
    # d = 1088 (17 blocks, not a multiple of 256) takes the register-staged
    # kernel (4 tokens per CTA); 257 tokens leave a ragged last group
    X, _ = synth.student_t_act(257, 1088, seed=10 + bits)
    _act_parity(X, 1088, bits, seed=bits)


@pytest.mark.parametrize("d,T,bits", [(4160, 37, 3), (8896, 9, 5), (16320, 5, 7), (1088, 1, 4),
                                      (2112, 4099, 2)])
def test_fast_path_widths(d, T, bits):
    # widths that are multiples of 64 but not of 256 take the register-staged
    # kernel: 4160 = 65 blocks (4 tokens per CTA, padded lanes); 8896 = 139
    # blocks (2 tokens per CTA); 16320: 1 token per CTA; 4099 tokens: many
    # groups per CTA
    X, _ = synth.student_t_act(T, d, seed=d + T)
    rows = None if T < 600 else np.random.default_rng(0).choice(T, 64, replace=False)
    _act_parity(X, d, bits, seed=d, rows=rows)


@pytest.mark.parametrize("d,T", [(64, 1), (64, 130), (128, 3), (1536, 33), (8960, 5), (32768, 2)])
def test_widths_from_one_block_to_maximum(d, T):
    X, _ = synth.student_t_act(T, d, seed=d)
    _act_parity(X, d, 4, seed=1)


def test_zero_and_degenerate_rows():
    d = 256
    X = synth.tiny()["X"][:8].copy()
    X[0] = 0.0                       # zero row: s = 0, every code is 2^(b-1)
    X[1] = 1.0                       # constant row
    X[2, :] = 0.0
    X[2, 17] = -3.0                  # one-hot row
    X[3] = -0.0
    codes, norms, _, _ = _act_parity(X, d, 4, dtype="f32")
    g = _unpack(codes, 4, d)
    assert np.all(g[0] == 8) and np.all(g[3] == 8)
    assert norms[0].item() == 0.0


@pytest.mark.parametrize("d,bits,dtype", [(3072, 4, "bf16"), (1280, 6, "bf16"),     # token-pair kernel, 8 pairs
                                          (4096, 5, "bf16"), (12288, 8, "bf16"),   # token-pair kernel, 4 / 1 pairs
                                          (4160, 5, "bf16"),                       # register-staged, [-1,1] grid
                                          (4160, 8, "bf16"),                       # register-staged, clamped grid
                                          (512, 3, "f32")])                        # general kernel
def test_non_finite_rows_encode_as_the_zero_vector(d, bits, dtype):
    """A row holding NaN or +-Inf has no finite norm; the kernels encode it as
    the zero vector (every code 2^(b-1)) and the other rows are unaffected."""
    X, _ = synth.student_t_act(40, d, seed=d + bits)
    X = X.copy()
    X[3, 7] = np.nan
    X[17, d - 1] = np.inf
    X[18, 0] = -np.inf
    X[38, :] = np.nan
    bad = np.array([3, 17, 18, 38])
    good = np.setdiff1d(np.arange(40), bad)
    r, Pi = _rpbh(d, 11)
    codes, norms = rq_act(r, _dense(X, dtype), bits)
    w_codes, rn = qweights(r, _dense(X, dtype), bits)          # the same rows as weights
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    for c in (codes, w_codes):
        g = _unpack(c, bits, d)
        assert np.all(g[bad] == 2 ** (bits - 1))
    _, bounds = oracle.lloydmax_table(d, bits)
    ora = oracle.quantize_act(X[good].astype(np.float64), Pi, bounds)
    check_codes(_unpack(codes, bits, d)[good], ora["codes"], ora["v"], bounds, d)
    check_rel(norms.cpu().numpy()[good], ora["norms"], NORM_RTOL, "norms")
    assert not np.any(np.isfinite(norms.cpu().numpy()[bad]))


def test_attention_projection_full_size_sampled():
    data = synth.attn_proj()
    X = data["X"]
    rows = np.unique(np.concatenate([[0, 1, X.shape[0] - 1], np.random.default_rng(0).choice(X.shape[0], 61)]))
    _, _, n_mis, n_band = _act_parity(X, 3072, 4, rows=rows)
    print(f"attn_proj A4: {n_mis} in-band mismatches, {n_band} coordinates in band")


@pytest.mark.parametrize("bits", [4, 3])
def test_mlp_down_input_full_size_sampled(bits):
    X, _ = synth.gelu_act(4608, 12288, seed=1)
    rows = np.random.default_rng(1).choice(4608, 24, replace=False)
    _act_parity(X, 12288, bits, seed=5, rows=rows)


@pytest.mark.parametrize("d", [1536, 8960])
def test_video_w4a6_activations_sampled_frames(d):
    X = synth.video_act(d, layer=3, frames=[0, 20])        # two frames, different scales
    rows = np.random.default_rng(d).choice(X.shape[0], 32, replace=False)
    _act_parity(X, d, 6, seed=1000 + 3, rows=rows)


# --------------------------------------------------------------------------
# token-pair kernel (BF16, d = 1024..3072 in steps of 256): every mode, ragged
# tiles of 16 tokens, and enough tiles per CTA to wrap its ring of slots and
# its norm barriers several times
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_pair_kernel_all_bit_widths(bits):
    # d = 1280: 5 warps per CTA; 37 tokens = 2 full tiles + 5 rows
    X, _ = synth.student_t_act(37, 1280, seed=40 + bits)
    _act_parity(X, 1280, bits, seed=bits)


@pytest.mark.parametrize("d,T,bits", [(3072, 1, 4), (3072, 17, 6), (3072, 33, 8), (1024, 16, 2), (2816, 31, 3)])
def test_pair_kernel_shapes(d, T, bits):
    X, _ = synth.student_t_act(T, d, seed=d + T)
    _act_parity(X, d, bits, seed=d)


@pytest.mark.parametrize("d,T,bits", [(1024, 148 * 16 * 14 + 5, 4), (3072, 148 * 16 * 6 + 9, 4)])
def test_pair_kernel_many_tiles_per_cta(d, T, bits):
    X, _ = synth.student_t_act(T, d, seed=7)
    rows = np.unique(np.concatenate([[0, 15, 16, T - 1, T - 6],
                                     np.random.default_rng(d).choice(T, 60, replace=False)]))
    _act_parity(X, d, bits, seed=3, rows=rows)


@pytest.mark.parametrize("d", [1280, 3072])
def test_pair_kernel_rotate_only(d):
    X, _ = synth.student_t_act(41, d, seed=d)
    r, Pi = _rpbh(d, 6)
    nr = torch.empty((41,), dtype=torch.float32, device="cuda")
    xr = rot_act(r, torch_bf16(X), norms=nr)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.rotate_only(X.astype(np.float64), Pi)
    check_bf16_rounding(bf16_to_numpy(xr), ora["xr"], "rotate-only")
    check_rel(nr.cpu().numpy(), np.linalg.norm(ora["xr"], axis=1), NORM_RTOL, "rotate-only norms")


# Wider rows: tiles of 8, 4 or 2 rows (4, 2 or 1 token pairs per tile), as
# many as keep two ring slots next to the gather table; 12288 (and 11520 at 8
# bits, whose code grid is larger) take 4-row tiles with the 16-bit gather
# table.  3328, 8960 and 11520 leave the CTA's
# last warp with lanes past the last block; the long cases wrap the ring of
# slots and the norm barriers several times per CTA.
@pytest.mark.parametrize("d,T,bits", [(4096, 8 * 148 * 3 + 5, 4), (3328, 45, 6), (5120, 19, 5), (8960, 37, 2),
                                      (8960, 4 * 148 * 2 + 3, 6), (12288, 4 * 148 * 3 + 1, 4), (12288, 21, 7),
                                      (11520, 37, 8), (11520, 29, 5), (16384, 19, 3), (16384, 7, 8)])
def test_pair_kernel_wide_rows(d, T, bits):
    X, _ = synth.student_t_act(T, d, seed=d + bits)
    rows = None
    if T > 64:
        rows = np.unique(np.concatenate([[0, 1, 7, 8, T - 1, T - 2],
                                         np.random.default_rng(d).choice(T, 40, replace=False)]))
    _act_parity(X, d, bits, seed=d + 1, rows=rows)


@pytest.mark.parametrize("d,n,bits", [(4096, 21, 4), (8960, 13, 3), (16384, 9, 2)])
def test_pair_kernel_wide_rows_weights(d, n, bits):
    W = synth.to_bf16(synth.gaussian_weights(synth.rng(15, d), n, d, outlier_frac=0.01).astype(np.float32))
    W[1] = 0.0
    r, Pi = _rpbh(d, 14)
    codes, rn = qweights(r, torch_bf16(W), bits)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    _, bounds = oracle.lloydmax_table(d, bits)
    ora = oracle.quantize_weights_lloydmax(W.astype(np.float64), Pi, bounds)
    check_codes(_unpack(codes, bits, d), ora["codes"], ora["v"], bounds, d)
    check_bf16_rounding(bf16_to_numpy(rn), ora["rnorm"], "row norms")


@pytest.mark.parametrize("d,n", [(4096, 37), (12288, 11), (8960, 5)])
def test_pair_kernel_wide_rows_int8(d, n):
    W = synth.to_bf16(synth.gaussian_weights(synth.rng(16, d), n, d, outlier_frac=0.01).astype(np.float32))
    W[2] = 0.0
    r, Pi = _rpbh(d, 15)
    q, sc = qweights(r, torch_bf16(W), 8, mode="int8")
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.quantize_weights_int8(W.astype(np.float64), Pi)
    check_int8(q.cpu().numpy().astype(np.int64), sc.cpu().numpy().astype(np.float64), ora)


@pytest.mark.parametrize("d,T", [(4096, 45), (8960, 11), (16384, 6)])
def test_pair_kernel_wide_rows_rotate_only(d, T):
    X, _ = synth.student_t_act(T, d, seed=d)
    r, Pi = _rpbh(d, 16)
    nr = torch.empty((T,), dtype=torch.float32, device="cuda")
    xr = rot_act(r, torch_bf16(X), norms=nr)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.rotate_only(X.astype(np.float64), Pi)
    check_bf16_rounding(bf16_to_numpy(xr), ora["xr"], "rotate-only")
    check_rel(nr.cpu().numpy(), np.linalg.norm(ora["xr"], axis=1), NORM_RTOL, "rotate-only norms")


@pytest.mark.parametrize("d,n", [(1024, 33), (3072, 50)])
def test_pair_kernel_weights_int8(d, n):
    W = synth.to_bf16(synth.gaussian_weights(synth.rng(12, d), n, d, outlier_frac=0.01).astype(np.float32))
    W[3] = 0.0
    r, Pi = _rpbh(d, 9)
    q, sc = qweights(r, torch_bf16(W), 8, mode="int8")
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.quantize_weights_int8(W.astype(np.float64), Pi)
    check_int8(q.cpu().numpy().astype(np.int64), sc.cpu().numpy().astype(np.float64), ora)


@pytest.mark.parametrize("d,n,dtype", [(1024, 40, "bf16"), (3072, 56, "bf16"),    # token-pair kernel
                                       (4096, 40, "bf16"),                         # token-pair kernel, 4 pairs
                                       (4160, 40, "bf16"),                         # register-staged kernel
                                       (512, 37, "f32")])                          # general kernel
def test_weights_int8_per_tensor(d, n, dtype):
    W = synth.to_bf16(synth.gaussian_weights(synth.rng(13, d), n, d, outlier_frac=0.01).astype(np.float32))
    W[4] = 0.0
    r, Pi = _rpbh(d, 10)
    q, sc = qweights(r, _dense(W, dtype), 8, mode="int8_tensor")
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.quantize_weights_int8(W.astype(np.float64), Pi, per_tensor=True)
    check_int8(q.cpu().numpy().astype(np.int64), sc.cpu().numpy().astype(np.float64), ora)
    # and the layer runs unchanged on it
    X = synth.to_bf16(np.random.default_rng(d).standard_normal((20, d)).astype(np.float32))
    xr = rot_act(r, torch_bf16(X)) if dtype == "bf16" else None
    if xr is not None:
        y = qlin_int8(xr, q, sc)
        torch.cuda.synchronize()
        ref = oracle.qlinear_int8(bf16_to_numpy(xr), q.cpu().numpy().astype(np.float64),
                                  sc.cpu().numpy().astype(np.float64))
        assert rel_frobenius(bf16_to_numpy(y), ref) < QLINEAR8_RTOL


@pytest.mark.parametrize("d,n,dtype", [(1024, 40, "bf16"), (3072, 37, "bf16"), (4096, 24, "bf16"),
                                       (8960, 13, "bf16"), (12288, 9, "bf16"),   # token-pair kernel
                                       (4160, 11, "bf16"), (512, 37, "f32")])   # general kernel
def test_weights_int8_asymmetric(d, n, dtype):
    W = synth.gaussian_weights(synth.rng(14, d), n, d, outlier_frac=0.01).astype(np.float32)
    W[: n // 2] += 0.01                      # some rows skewed, so zero points vary
    W = synth.to_bf16(W)
    W[2] = 0.0
    r, Pi = _rpbh(d, 12)
    q, sc, z = rbq.quantize_weights_int8_asym(r, _dense(W, dtype), q=poison((n, d), torch.uint8),
                                              scale=poison((n,), torch.float32),
                                              zero_point=poison((n,), torch.uint8))
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.quantize_weights_int8_asym(W.astype(np.float64), Pi)
    check_int8_asym(q.cpu().numpy().astype(np.int64), sc.cpu().numpy().astype(np.float64),
                    z.cpu().numpy().astype(np.int64), ora)
    if n % 8 == 0 and dtype == "bf16":
        X = synth.to_bf16(np.random.default_rng(d + 1).standard_normal((24, d)).astype(np.float32))
        xr = rot_act(r, torch_bf16(X))
        y = rbq.qlinear_int8_asym(xr, q, sc, z, out=poison((24, n), torch.bfloat16))
        torch.cuda.synchronize()
        assert rbq.device_error() == 0
        ref = oracle.qlinear_int8_asym(bf16_to_numpy(xr), q.cpu().numpy(), sc.cpu().numpy().astype(np.float64),
                                       z.cpu().numpy())
        assert rel_frobenius(bf16_to_numpy(y), ref) < QLINEAR8_RTOL


@pytest.mark.parametrize("bits", [6, 8])
def test_pair_kernel_weights_wide_codebooks(bits):
    d = 3072
    W = synth.attn_proj()["W"][:40].copy()
    W[2] = 0.0
    r, Pi = _rpbh(d, 0)
    codes, rn = qweights(r, torch_bf16(W), bits)
    torch.cuda.synchronize()
    _, bounds = oracle.lloydmax_table(d, bits)
    ora = oracle.quantize_weights_lloydmax(W.astype(np.float64), Pi, bounds)
    check_codes(_unpack(codes, bits, d), ora["codes"], ora["v"], bounds, d)
    check_bf16_rounding(bf16_to_numpy(rn), ora["rnorm"], "row norms")


# --------------------------------------------------------------------------
# ablation handles (OrbitQuant §3.3): block Hadamard without the permutation,
# and without the signs; the same kernels, checked against the oracle's
# dense matrix built from the same pi and D
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d,T,bits,permute,signs", [(3072, 37, 4, False, True), (1024, 20, 2, False, True),
                                                    (3072, 19, 3, True, False), (512, 33, 4, False, False),
                                                    (12288, 9, 4, False, True), (8960, 11, 3, True, False)])
def test_ablation_handles_quantize(d, T, bits, permute, signs):
    X, _ = synth.student_t_act(T, d, seed=d + bits)
    r = rbq.RPBH(d, 21, permute=permute, signs=signs)
    perm, sg = r.export()
    op, os_ = oracle.rpbh_draw(d, 21)
    assert np.array_equal(perm, np.arange(d) if not permute else op)
    assert np.array_equal(sg, np.ones(d) if not signs else os_)
    Pi = oracle.rpbh_matrix(perm.astype(np.int64), sg.astype(np.int64))
    _act_parity(X, d, bits, Pi=Pi, r=r)


@pytest.mark.parametrize("d", [1024, 3072])
def test_ablation_handle_rotate_only(d):
    X, _ = synth.student_t_act(40, d, seed=d)
    r = rbq.RPBH(d, 8, permute=False)
    perm, sg = r.export()
    Pi = oracle.rpbh_matrix(perm.astype(np.int64), sg.astype(np.int64))
    xr = rot_act(r, torch_bf16(X))
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    ora = oracle.rotate_only(X.astype(np.float64), Pi)
    check_bf16_rounding(bf16_to_numpy(xr), ora["xr"], "block-Hadamard rotate-only")


# --------------------------------------------------------------------------
# rotate-only (BF16 x') and offline weights
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d", [512, 1024, 8960])
def test_rotate_only_bf16(d):
    X, _ = synth.student_t_act(200, d, seed=9)
    r, Pi = _rpbh(d, 4)
    xr = rot_act(r, torch_bf16(X))
    torch.cuda.synchronize()
    ora = oracle.rotate_only(X.astype(np.float64), Pi)
    n = check_bf16_rounding(bf16_to_numpy(xr), ora["xr"], "rotate-only")
    print(f"rotate-only: {n} in-band BF16 rounding differences")


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_weights_lloydmax(bits):
    d = 3072
    W = synth.attn_proj()["W"][:200]
    W = W.copy()
    W[5] = 0.0
    r, Pi = _rpbh(d, 0)
    codes, rn = qweights(r, torch_bf16(W), bits)
    torch.cuda.synchronize()
    _, bounds = oracle.lloydmax_table(d, bits)
    ora = oracle.quantize_weights_lloydmax(W.astype(np.float64), Pi, bounds)
    check_codes(_unpack(codes, bits, d), ora["codes"], ora["v"], bounds, d)
    check_bf16_rounding(bf16_to_numpy(rn), ora["rnorm"], "row norms")


def test_weights_tiny_fp32():
    W = synth.tiny()["W"]
    r, Pi = _rpbh(256, 0)
    codes, rn = qweights(r, _dense(W, "f32"), 4)
    _, bounds = oracle.lloydmax_table(256, 4)
    ora = oracle.quantize_weights_lloydmax(W.astype(np.float64), Pi, bounds)
    check_codes(_unpack(codes, 4, 256), ora["codes"], ora["v"], bounds, 256)
    check_bf16_rounding(bf16_to_numpy(rn), ora["rnorm"], "row norms")


@pytest.mark.parametrize("shape", [(256, 256), (320, 4096), (64, 16384)])
def test_weights_int8(shape):
    n, d = shape
    W = synth.int8_dit_weight(0, "q")[:n, :d] if d == 4096 else \
        synth.gaussian_weights(synth.rng(11, d), n, d, outlier_frac=0.01).astype(np.float32)
    W = synth.to_bf16(W)
    W[1] = 0.0
    r, Pi = _rpbh(d, 2)
    q, sc = qweights(r, torch_bf16(W), 8, mode="int8")
    torch.cuda.synchronize()
    ora = oracle.quantize_weights_int8(W.astype(np.float64), Pi)
    n_mis = check_int8(q.cpu().numpy().astype(np.int64), sc.cpu().numpy().astype(np.float64), ora)
    print(f"int8 {shape}: {n_mis} in-band rounding differences")


# --------------------------------------------------------------------------
# qlinear / qlinear_int8
# --------------------------------------------------------------------------

def _qlinear_case(X, W, d, bits_a, bits_w, seed=0, rows=None, dtype="bf16"):
    r, Pi = _rpbh(d, seed)
    a_codes, s = rq_act(r, _dense(X, dtype), bits_a)
    w_codes, rn = qweights(r, _dense(W, dtype), bits_w)
    y = qlin(a_codes, s, bits_a, w_codes, rn, bits_w, d)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    la, _ = oracle.lloydmax_table(d, bits_a)
    lw, _ = oracle.lloydmax_table(d, bits_w)
    pa = _unpack(a_codes[torch.as_tensor(rows).cuda()], bits_a, d)
    pw = _unpack(w_codes, bits_w, d)
    ref = oracle.qlinear(pa, s.cpu().numpy()[rows], la, pw, bf16_to_numpy(rn), lw)
    got = bf16_to_numpy(y[torch.as_tensor(rows).cuda()])
    err = rel_frobenius(got, ref)
    return err, got, ref


def test_qlinear_tiny_w4a4():
    data = synth.tiny()
    err, got, ref = _qlinear_case(data["X"], data["W"], 256, 4, 4, dtype="f32")
    assert err < QLINEAR_RTOL, err
    # and the quantised layer approximates the dense one (OrbitQuant §2.2)
    dense = data["X"].astype(np.float64) @ data["W"].astype(np.float64).T
    assert rel_frobenius(got, dense) < 0.2


@pytest.mark.parametrize("M,N,K,ba,bw", [(1, 8, 64, 4, 4), (130, 136, 128, 4, 2), (257, 264, 320, 3, 3),
                                         (64, 512, 256, 6, 4), (200, 128, 192, 8, 8), (77, 72, 64, 2, 6),
                                         # TMA-fed kernel (K % 128 == 0): every code-stage kind
                                         (130, 256, 384, 8, 8), (64, 264, 256, 2, 6), (300, 520, 256, 5, 7),
                                         (129, 512, 1024, 4, 4), (513, 1032, 512, 3, 1), (1, 256, 128, 4, 4)])
def test_qlinear_ragged_shapes_and_bit_widths(M, N, K, ba, bw):
    g = np.random.default_rng(M * N)
    X = synth.to_bf16(g.standard_t(3, (M, K)).astype(np.float32))
    W = synth.to_bf16((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    err, _, _ = _qlinear_case(X, W, K, ba, bw, seed=M)
    assert err < QLINEAR_RTOL, err


def test_qlinear_attention_projection_full_size_sampled():
    data = synth.attn_proj()
    rows = np.random.default_rng(2).choice(4608, 48, replace=False)
    err, _, _ = _qlinear_case(data["X"], data["W"], 3072, 4, 4, rows=rows)
    print(f"qlinear attn_proj W4A4 rel. Frobenius error {err:.2e}")
    assert err < QLINEAR_RTOL


@pytest.mark.parametrize("ba,bw", [(4, 2), (3, 3)])
def test_qlinear_mlp_full_size_sampled(ba, bw):
    m = synth.mlp()
    rows = np.random.default_rng(3).choice(4608, 16, replace=False)
    err_up, _, _ = _qlinear_case(m["X_up"], m["W_up"], 3072, ba, bw, seed=4, rows=rows)
    err_dn, _, _ = _qlinear_case(m["X_dn"], m["W_dn"], 12288, ba, bw, seed=5, rows=rows)
    assert err_up < QLINEAR_RTOL and err_dn < QLINEAR_RTOL, (err_up, err_dn)


def _qlinear_i8_case(X, W, d, bits_a, bits_w, seed=0, rows=None):
    """qlinear_int8_levels on the library's own codes vs the oracle's integer
    layer on the same codes: BF16 outputs bit-exact outside the rounding band
    (the integer sum is exact on both sides, only the fp32 scaling differs)."""
    r, _ = _rpbh(d, seed)
    a_codes, s = rq_act(r, _dense(X, "bf16"), bits_a)
    w_codes, rn = qweights(r, _dense(W, "bf16"), bits_w)
    y = qlin_i8(a_codes, s, bits_a, w_codes, rn, bits_w, d)
    y_fp16 = qlin(a_codes, s, bits_a, w_codes, rn, bits_w, d)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    idx = torch.as_tensor(rows).cuda()
    la, _ = oracle.lloydmax_table(d, bits_a)
    lw, _ = oracle.lloydmax_table(d, bits_w)
    pa = _unpack(a_codes[idx], bits_a, d)
    pw = _unpack(w_codes, bits_w, d)
    exact = oracle.qlinear_int8_levels(pa, s.cpu().numpy()[rows], la, pw, bf16_to_numpy(rn), lw)
    got = bf16_to_numpy(y[idx])
    n_band = check_bf16_rounding(got, exact, "qlinear_int8_levels")
    # and against the exact-level layer: the levels' rounding only
    return n_band, rel_frobenius(got, bf16_to_numpy(y_fp16[idx]))


@pytest.mark.parametrize("M,N,K,ba,bw", [(1, 8, 128, 4, 4), (130, 136, 128, 4, 2), (257, 264, 384, 3, 3),
                                         (64, 512, 256, 6, 4), (200, 128, 256, 8, 8), (77, 72, 256, 2, 6),
                                         (300, 520, 256, 5, 7), (129, 512, 1024, 4, 4), (513, 1032, 512, 3, 1),
                                         (260, 256, 640, 1, 5), (128, 256, 128, 7, 3)])
def test_qlinear_int8_levels_ragged_shapes_and_bit_widths(M, N, K, ba, bw):
    g = np.random.default_rng(M * N + 1)
    X = synth.to_bf16(g.standard_t(3, (M, K)).astype(np.float32))
    W = synth.to_bf16((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    n_band, dev = _qlinear_i8_case(X, W, K, ba, bw, seed=M)
    print(f"int8-level qlinear {M}x{N}x{K} W{bw}A{ba}: {n_band} in-band roundings, {dev:.2e} from exact levels")


FP8_RTOL = 3e-3           # rel. Frobenius, fp32 sums of exact E4M3 products + BF16 output


# Each E4M3 level e_j / beta is within 2^-4 (half of a 3-bit mantissa step)
# of the exact level c_j, so every product e_w e_a / (beta_w beta_a) is within
# FP8_PRODUCT_REL = (1 + 2^-4)^2 - 1 of c_w c_a, and by the triangle
# inequality |y_fp8 - y_exact| <= FP8_PRODUCT_REL * s_m r'_n sum_k |c_w| |c_a|
# element by element.  That bound is on the sum of absolute products, not on
# |y_exact| itself: with cancellation in the sum the relative deviation can
# exceed FP8_PRODUCT_REL, so the test checks the absolute form.
FP8_PRODUCT_REL = (1 + 2.0 ** -4) ** 2 - 1


def _qlinear_fp8_case(X, W, d, bits_a, bits_w, seed=0, rows=None):
    """qlinear_fp8_levels on the library's own codes vs the oracle's FP8 layer
    (exact fp64 sums) on the same codes; returns (error vs oracle, deviation
    from the exact-level layer) and checks the deviation against the bound
    above (plus the kernel's own error against its oracle)."""
    r, _ = _rpbh(d, seed)
    a_codes, s = rq_act(r, _dense(X, "bf16"), bits_a)
    w_codes, rn = qweights(r, _dense(W, "bf16"), bits_w)
    y = qlin_fp8(a_codes, s, bits_a, w_codes, rn, bits_w, d)
    y_fp16 = qlin(a_codes, s, bits_a, w_codes, rn, bits_w, d)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    idx = torch.as_tensor(rows).cuda()
    la, _ = oracle.lloydmax_table(d, bits_a)
    lw, _ = oracle.lloydmax_table(d, bits_w)
    pa = _unpack(a_codes[idx], bits_a, d)
    pw = _unpack(w_codes, bits_w, d)
    s_np, rn_np = s.cpu().numpy()[rows], bf16_to_numpy(rn)
    ref = oracle.qlinear_fp8_levels(pa, s_np, la, pw, rn_np, lw)
    got = bf16_to_numpy(y[idx])
    exact = oracle.qlinear(pa, s_np, la, pw, rn_np, lw)
    abs_sum = oracle.qlinear(pa, s_np, np.abs(la), pw, rn_np, np.abs(lw))
    err = rel_frobenius(got, ref)
    bound = FP8_PRODUCT_REL * np.linalg.norm(abs_sum) + err * np.linalg.norm(ref)
    assert np.linalg.norm(got - exact) <= bound * (1 + 1e-9), (np.linalg.norm(got - exact), bound)
    return err, rel_frobenius(got, bf16_to_numpy(y_fp16[idx]))


@pytest.mark.parametrize("M,N,K,ba,bw", [(1, 8, 128, 4, 4), (130, 136, 128, 4, 2), (257, 264, 384, 3, 3),
                                         (64, 512, 256, 6, 4), (200, 128, 256, 8, 8), (300, 520, 256, 5, 7),
                                         (129, 512, 1024, 4, 4), (260, 256, 640, 1, 5)])
def test_qlinear_fp8_levels_ragged_shapes_and_bit_widths(M, N, K, ba, bw):
    g = np.random.default_rng(M * N + 2)
    X = synth.to_bf16(g.standard_t(3, (M, K)).astype(np.float32))
    W = synth.to_bf16((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    err, dev = _qlinear_fp8_case(X, W, K, ba, bw, seed=M)
    print(f"fp8-level qlinear {M}x{N}x{K} W{bw}A{ba}: {err:.2e} vs oracle, {dev:.2e} from exact levels")
    assert err < FP8_RTOL, err


def test_qlinear_fp8_levels_attention_projection_sampled():
    data = synth.attn_proj()
    rows = np.random.default_rng(7).choice(4608, 32, replace=False)
    err, dev = _qlinear_fp8_case(data["X"], data["W"], 3072, 4, 4, rows=rows)
    print(f"fp8-level qlinear attn_proj W4A4: {err:.2e} vs oracle, {dev:.2e} from exact levels")
    assert err < FP8_RTOL, err


def test_qlinear_int8_levels_attention_projection_sampled():
    data = synth.attn_proj()
    rows = np.random.default_rng(5).choice(4608, 32, replace=False)
    n_band, dev = _qlinear_i8_case(data["X"], data["W"], 3072, 4, 4, rows=rows)
    print(f"int8-level qlinear attn_proj W4A4: {n_band} in-band, {dev:.2e} from exact levels")
    assert dev < 2e-2


def test_qlinear_int8_levels_mlp_down_sampled():
    m = synth.mlp()
    rows = np.random.default_rng(6).choice(4608, 8, replace=False)
    n_band, dev = _qlinear_i8_case(m["X_dn"], m["W_dn"], 12288, 4, 2, seed=5, rows=rows)
    assert dev < 2e-2


@pytest.mark.parametrize("layer,M,N,K,ba,bw", [("fp16", 139264, 136, 1024, 4, 4), ("int8", 70000, 136, 1024, 4, 3)])
def test_large_activation_operand_tiles_walked_n_fastest(layer, M, N, K, ba, bw):
    """Activation operands larger than the weights, with weights that fit in
    half of L2, make the pair GEMMs walk their output tiles N-fastest; random
    codes, sampled rows (the first, the last and tiles in between) against the
    oracle."""
    gen = torch.Generator(device="cuda").manual_seed(M)
    a = torch.randint(0, 256, (M, K * ba // 8), dtype=torch.uint8, device="cuda", generator=gen)
    w = torch.randint(0, 256, (N, K * bw // 8), dtype=torch.uint8, device="cuda", generator=gen)
    s = torch.rand(M, device="cuda", generator=gen) + 0.5
    rn = (torch.rand(N, device="cuda", generator=gen) + 0.5).to(torch.bfloat16)
    fn = rbq.qlinear if layer == "fp16" else rbq.qlinear_int8_levels
    y = fn(a, s, ba, w, rn, bw, K, out=poison((M, N), torch.bfloat16))
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M).choice(M, 40, replace=False)]))
    idx = torch.as_tensor(rows).cuda()
    la, _ = oracle.lloydmax_table(K, ba)
    lw, _ = oracle.lloydmax_table(K, bw)
    pa = _unpack(a[idx], ba, K)
    pw = _unpack(w, bw, K)
    got = bf16_to_numpy(y[idx])
    if layer == "fp16":
        ref = oracle.qlinear(pa, s.cpu().numpy()[rows], la, pw, bf16_to_numpy(rn), lw)
        assert rel_frobenius(got, ref) < QLINEAR_RTOL
    else:
        ref = oracle.qlinear_int8_levels(pa, s.cpu().numpy()[rows], la, pw, bf16_to_numpy(rn), lw)
        check_bf16_rounding(got, ref, "qlinear_int8_levels")


@pytest.mark.parametrize("n_out,d_in", [(1536, 1536), (8960, 1536), (1536, 8960)])
def test_qlinear_video_w4a6_full_size_sampled(n_out, d_in):
    """The video-DiT workload (Wan 2.1 1.3B shape, OrbitQuant §3.2, W4A6):
    32760 tokens = 21 frames x 1560 patches, hidden 1536, MLP 8960.  Every
    layer expands its 6-bit activation codes in a pass of its own (fp16
    copies of 100 MB and, for the 8960-wide down-projection, 587 MB) before
    the pair GEMM.  Every token is quantised on the GPU; sampled rows (first,
    last, others) are compared."""
    T = 32760
    X = synth.video_act(d_in, layer=7)
    assert X.shape == (T, d_in)
    W = synth.video_weight(n_out, d_in, layer=7)
    rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(d_in + n_out).choice(T, 30, replace=False)]))
    err, _, _ = _qlinear_case(X, W, d_in, 6, 4, seed=1000 + 7, rows=rows)
    print(f"qlinear video {T}x{n_out}x{d_in} W4A6 rel. Frobenius error {err:.2e}")
    assert err < QLINEAR_RTOL, err


@pytest.mark.parametrize("bits_a,bits_w", [(1, 4), (2, 3), (3, 4), (5, 2), (6, 4), (7, 8), (8, 1)])
def test_qlinear_in_kernel_expansion_every_activation_width(bits_a, bits_w):
    """Activations whose fp16 copy would exceed 2 GiB take the in-kernel
    expansion route (the codes expanded inside the GEMM: byte permutes at 2,
    3 and 4 bits, a shared-memory level table otherwise): 1.1 M x 1024 x 2
    bytes = 2.25 GB here.  Random codes, sampled rows (the first, the last and
    tiles in between) against the oracle."""
    M, N, K = 1_100_000, 136, 1024
    assert M * K * 2 > 2 << 30
    gen = torch.Generator(device="cuda").manual_seed(bits_a * 16 + bits_w)
    a = torch.randint(0, 256, (M, K * bits_a // 8), dtype=torch.uint8, device="cuda", generator=gen)
    w = torch.randint(0, 256, (N, K * bits_w // 8), dtype=torch.uint8, device="cuda", generator=gen)
    s = torch.rand(M, device="cuda", generator=gen) + 0.5
    rn = (torch.rand(N, device="cuda", generator=gen) + 0.5).to(torch.bfloat16)
    y = qlin(a, s, bits_a, w, rn, bits_w, K)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], np.random.default_rng(M).choice(M, 40, replace=False)]))
    idx = torch.as_tensor(rows).cuda()
    la, _ = oracle.lloydmax_table(K, bits_a)
    lw, _ = oracle.lloydmax_table(K, bits_w)
    ref = oracle.qlinear(_unpack(a[idx], bits_a, K), s.cpu().numpy()[rows], la, _unpack(w, bits_w, K),
                         bf16_to_numpy(rn), lw)
    err = rel_frobenius(bf16_to_numpy(y[idx]), ref)
    print(f"qlinear in-kernel expansion W{bits_w}A{bits_a}: rel. Frobenius error {err:.2e}")
    assert err < QLINEAR_RTOL, err


def _int8_case(X, W, d, seed=0, rows=None):
    r, Pi = _rpbh(d, seed)
    xr = rot_act(r, torch_bf16(X))
    q, sc = qweights(r, torch_bf16(W), 8, mode="int8")
    y = qlin_int8(xr, q, sc)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows)
    idx = torch.as_tensor(rows).cuda()
    ref = oracle.qlinear_int8(bf16_to_numpy(xr[idx]), q.cpu().numpy(), sc.cpu().numpy())
    got = bf16_to_numpy(y[idx])
    return rel_frobenius(got, ref), got, Pi


@pytest.mark.parametrize("M,N,K", [(64, 256, 256), (130, 136, 192), (1, 8, 64)])
def test_qlinear_int8_small(M, N, K):
    g = np.random.default_rng(K)
    X = synth.to_bf16(g.standard_normal((M, K)).astype(np.float32))
    W = synth.to_bf16(synth.gaussian_weights(g, N, K, outlier_frac=0.01))
    err, _, _ = _int8_case(X, W, K, seed=K)
    assert err < QLINEAR8_RTOL, err


@pytest.mark.parametrize("name", ["q", "up", "down"])
def test_qlinear_int8_dit_block_sampled(name):
    W = synth.int8_dit_weight(0, name)
    d = W.shape[1]
    X = synth.int8_dit_act(d)
    rows = np.random.default_rng(4).choice(4096, 16, replace=False)
    err, got, Pi = _int8_case(X, W, d, seed=7, rows=rows)
    assert err < QLINEAR8_RTOL, err
    # rotated INT8 beats naive INT8 on these outlier weights (INT8-convrot §2)
    dense = X[rows].astype(np.float64) @ W.astype(np.float64).T
    naive = oracle.quantize_weights_int8(W.astype(np.float64))
    y_naive = oracle.qlinear_int8(X[rows].astype(np.float64), naive["q"], naive["scale"])
    assert rel_frobenius(got, dense) < rel_frobenius(y_naive, dense)
