"""Host-side checks of the C ABI (no GPU needed).

* librbq.so loads and exports every function include/rbq.h declares;
* rpbh_make reproduces the oracle's permutation and signs exactly;
* lloydmax_table (Newton's method, C++) agrees with the oracle's fixed-point
  iteration (two independent algorithms for the same optimum);
* invalid arguments are rejected before any device work, with the
  documented codes (so these calls are safe on a machine without a GPU).
"""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import rotation_bit_ptq_b200 as rbq
from rotation_bit_ptq_b200 import build as rbq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(rbq.LIB_PATH):
        rbq_build.build()
    return rbq.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "rbq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"rpbh_make", "lloydmax_table", "quantize_weights", "rotate_quantize_act", "qlinear"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert n in rbq.SIGNATURES, n


@pytest.mark.parametrize("d,seed", [(64, 0), (256, 0), (3072, 0), (3072, 12345), (12288, 7),
                                    (8960, 2 ** 64 - 1)])
def test_rpbh_make_matches_oracle(lib, d, seed):
    r = rbq.RPBH(d, seed)
    perm, signs = r.export()
    op, os_ = oracle.rpbh_draw(d, seed)
    assert np.array_equal(perm.astype(np.int64), op)
    assert np.array_equal(signs.astype(np.int64), os_)
    assert lib.rpbh_dim(r.handle) == d
    r.close()


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_lloydmax_table_matches_oracle(lib, bits):
    d = 3072
    lv, bd = rbq.lloydmax_table(d, bits)
    olv, obd = oracle.lloydmax_table(d, bits)
    # The oracle's plain iteration contracts slowly at 8 bits (rate ~0.9999),
    # which amplifies fp64 rounding to ~3e-11 sigma; Newton lands on the optimum.
    tol = 1e-12 if bits <= 7 else 1e-10
    sigma = 1 / np.sqrt(d)
    assert np.max(np.abs(lv - olv)) / sigma < tol
    assert np.max(np.abs(bd - obd)) / sigma < tol
    assert np.array_equal(lv, -lv[::-1])
    assert bd[len(bd) // 2] == 0.0
    assert np.array_equal(bd, 0.5 * (lv[:-1] + lv[1:]))


def test_rpbh_make_rejects_bad_arguments(lib):
    out = ctypes.c_void_p()
    for d, h in ((0, 64), (-64, 64), (100, 64), (256, 32), (65536 + 64, 64), (32768 + 64, 64)):
        assert lib.rpbh_make(d, h, 0, ctypes.byref(out)) == rbq.RBQ_EINVAL
    assert lib.rpbh_make(64, 64, 0, None) == rbq.RBQ_EINVAL
    assert lib.rpbh_export(None, None, None) == rbq.RBQ_EINVAL
    assert lib.rpbh_dim(None) == rbq.RBQ_EINVAL
    lib.rpbh_free(None)


@pytest.mark.parametrize("flags", [0, 1, 2, 3])
def test_rpbh_make_ablation_flags(lib, flags):
    d, seed = 1024, 99
    out = ctypes.c_void_p()
    assert lib.rpbh_make_ablation(d, 64, seed, flags, ctypes.byref(out)) == rbq.RBQ_OK
    perm = np.empty(d, dtype=np.int32)
    signs = np.empty(d, dtype=np.int8)
    assert lib.rpbh_export(out, perm.ctypes.data_as(ctypes.c_void_p), signs.ctypes.data_as(ctypes.c_void_p)) == 0
    lib.rpbh_free(out)
    op, os_ = oracle.rpbh_draw(d, seed)
    # the draw is consumed as by rpbh_make, then the switched-off parts reset
    expect_perm = np.arange(d) if flags & rbq.RBQ_RPBH_NO_PERMUTATION else op
    expect_signs = np.ones(d) if flags & rbq.RBQ_RPBH_NO_SIGNS else os_
    assert np.array_equal(perm, expect_perm)
    assert np.array_equal(signs, expect_signs)


def test_rpbh_make_ablation_rejects_unknown_flags(lib):
    out = ctypes.c_void_p(1234)
    assert lib.rpbh_make_ablation(256, 64, 0, 4, ctypes.byref(out)) == rbq.RBQ_EINVAL
    assert out.value is None
    assert lib.rpbh_make_ablation(100, 64, 0, 1, ctypes.byref(out)) == rbq.RBQ_EINVAL


def test_lloydmax_rejects_bad_arguments(lib):
    for d, b in ((0, 4), (64, 0), (64, 9), (-1, 2)):
        assert lib.lloydmax_table(d, b, None, None) == rbq.RBQ_EINVAL


def test_kernel_entry_points_validate_before_launch(lib):
    r = rbq.RPBH(256, 0)
    h = r.handle
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: rejected first
    odd = ctypes.c_void_p(0x10001)
    # empty inputs are a successful no-op
    assert lib.rotate_quantize_act(h, None, rbq.RBQ_BF16, 0, 4, None, None, None) == rbq.RBQ_OK
    assert lib.quantize_weights(h, None, rbq.RBQ_BF16, 0, rbq.RBQ_LLOYDMAX, 4, None, None, None) == rbq.RBQ_OK
    assert lib.qlinear(None, None, 4, None, None, 4, 0, 8, 64, None, None) == rbq.RBQ_OK
    assert lib.qlinear_int8(None, None, None, 8, 0, 64, None, None) == rbq.RBQ_OK
    # bad arguments
    assert lib.rotate_quantize_act(None, fake, rbq.RBQ_BF16, 4, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.rotate_quantize_act(h, fake, 7, 4, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.rotate_quantize_act(h, fake, rbq.RBQ_BF16, 4, 9, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.rotate_quantize_act(h, fake, rbq.RBQ_BF16, -1, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.rotate_quantize_act(h, fake, rbq.RBQ_BF16, 4, 4, fake, None, None) == rbq.RBQ_EINVAL
    assert lib.rotate_quantize_act(h, odd, rbq.RBQ_BF16, 4, 4, fake, fake, None) == rbq.RBQ_EALIGN
    assert lib.rotate_quantize_act(h, fake, rbq.RBQ_BF16, 4, 4, odd, fake, None) == rbq.RBQ_EALIGN
    assert lib.quantize_weights(h, fake, rbq.RBQ_BF16, 4, 5, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_weights(h, fake, rbq.RBQ_BF16, 4, rbq.RBQ_INT8_SYM, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_weights(h, odd, rbq.RBQ_BF16, 4, rbq.RBQ_LLOYDMAX, 4, fake, fake, None) == rbq.RBQ_EALIGN
    assert lib.qlinear(fake, fake, 4, fake, fake, 4, 8, 8, 100, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear(fake, fake, 0, fake, fake, 4, 8, 8, 64, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear(fake, fake, 4, fake, fake, 4, 8, 12, 64, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear(odd, fake, 4, fake, fake, 4, 8, 8, 64, fake, None) == rbq.RBQ_EALIGN
    assert lib.qlinear_int8(fake, fake, fake, 8, 8, 96, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8(fake, odd, fake, 8, 8, 64, fake, None) == rbq.RBQ_EALIGN
    # per-tensor INT8 takes bits 8 only; the zero-point variants
    assert lib.quantize_weights(h, fake, rbq.RBQ_BF16, 4, rbq.RBQ_INT8_TENSOR, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_weights(h, odd, rbq.RBQ_BF16, 4, rbq.RBQ_INT8_TENSOR, 8, fake, fake, None) == rbq.RBQ_EALIGN
    assert lib.quantize_weights_int8_asym(h, None, rbq.RBQ_BF16, 0, None, None, None, None) == rbq.RBQ_OK
    assert lib.quantize_weights_int8_asym(h, fake, rbq.RBQ_BF16, 4, fake, fake, None, None) == rbq.RBQ_EINVAL
    assert lib.quantize_weights_int8_asym(h, fake, 3, 4, fake, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_weights_int8_asym(h, fake, rbq.RBQ_BF16, 4, odd, fake, fake, None) == rbq.RBQ_EALIGN
    assert lib.qlinear_int8_asym(fake, fake, fake, fake, 8, 12, 64, fake, None) == rbq.RBQ_EINVAL   # N % 8
    assert lib.qlinear_int8_asym(fake, fake, fake, fake, 8, 8, 96, fake, None) == rbq.RBQ_EINVAL    # K % 64
    assert lib.qlinear_int8_asym(fake, fake, fake, None, 8, 8, 64, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_asym(odd, fake, fake, fake, 8, 8, 64, fake, None) == rbq.RBQ_EALIGN
    # integer-level layer: K % 128, N % 8, 16-byte code rows, bit widths, pointers
    assert lib.qlinear_int8_levels(None, None, 4, None, None, 4, 0, 8, 128, None, None) == rbq.RBQ_OK
    assert lib.qlinear_int8_levels(fake, fake, 4, fake, fake, 4, 8, 8, 64, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_levels(fake, fake, 4, fake, fake, 4, 8, 12, 128, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_levels(fake, fake, 9, fake, fake, 4, 8, 8, 128, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_levels(fake, fake, 4, fake, fake, 0, 8, 8, 128, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_levels(fake, fake, 4, fake, fake, 4, 8, 8, 32896, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_levels(fake, None, 4, fake, fake, 4, 8, 8, 128, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_int8_levels(odd, fake, 4, fake, fake, 4, 8, 8, 128, fake, None) == rbq.RBQ_EALIGN
    assert lib.qlinear_fp8_levels(None, None, 4, None, None, 4, 0, 8, 128, None, None) == rbq.RBQ_OK
    assert lib.qlinear_fp8_levels(fake, fake, 4, fake, fake, 4, 8, 8, 192, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_fp8_levels(fake, fake, 4, fake, fake, 4, 8, 4, 128, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_fp8_levels(fake, fake, 4, odd, fake, 4, 8, 8, 128, fake, None) == rbq.RBQ_EALIGN
    # the rotation fused into the code layer, and the quantiser on rotated rows
    nx = rbq.RPBH(512, 1)
    n = nx.handle
    assert lib.qlinear_rotate_next(None, None, 4, None, None, 4, 0, 128, n, rbq.RBQ_ACT_GELU, None, None) == rbq.RBQ_OK
    assert lib.qlinear_rotate_next(fake, fake, 4, fake, fake, 4, 8, 128, None, 0, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_rotate_next(fake, fake, 4, fake, fake, 4, 8, 96, n, 0, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_rotate_next(fake, fake, 9, fake, fake, 4, 8, 128, n, 0, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_rotate_next(fake, fake, 4, fake, fake, 4, 8, 128, n, 2, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_rotate_next(fake, fake, 4, fake, None, 4, 8, 128, n, 0, fake, None) == rbq.RBQ_EINVAL
    assert lib.qlinear_rotate_next(fake, fake, 4, odd, fake, 4, 8, 128, n, 0, fake, None) == rbq.RBQ_EALIGN
    assert lib.quantize_rotated(None, rbq.RBQ_BF16, 0, 256, 4, None, None, None) == rbq.RBQ_OK
    assert lib.quantize_rotated(fake, rbq.RBQ_F32, 4, 256, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_rotated(fake, rbq.RBQ_BF16, 4, 200, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_rotated(fake, rbq.RBQ_BF16, 4, 256, 0, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_rotated(fake, rbq.RBQ_BF16, -1, 256, 4, fake, fake, None) == rbq.RBQ_EINVAL
    assert lib.quantize_rotated(fake, rbq.RBQ_BF16, 4, 256, 4, fake, None, None) == rbq.RBQ_EINVAL
    assert lib.quantize_rotated(odd, rbq.RBQ_BF16, 4, 256, 4, fake, fake, None) == rbq.RBQ_EALIGN
    nx.close()
    r.close()


@pytest.mark.parametrize("bits", range(1, 9))
def test_fp8_levels_match_oracle(lib, bits):
    torch = pytest.importorskip("torch")
    for d in (64, 256, 1536, 3072, 4096, 8960, 12288, 16384):   # every width of the workloads
        lv, beta = rbq.fp8_levels(d, bits)
        vals = torch.from_numpy(lv).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        ov, obeta = oracle.fp8_levels(oracle.lloydmax_table(d, bits)[0])
        assert beta == obeta
        assert np.array_equal(vals, ov)
    assert lib.rbq_fp8_levels(64, 9, None, None) == rbq.RBQ_EINVAL


@pytest.mark.parametrize("bits", range(1, 9))
def test_int8_levels_match_oracle(lib, bits):
    for d in (64, 256, 1536, 3072, 4096, 8960, 12288, 16384):   # every width of the workloads
        lv, alpha = rbq.int8_levels(d, bits)
        olv, oalpha = oracle.int8_levels(oracle.lloydmax_table(d, bits)[0])
        assert np.array_equal(lv.astype(np.int64), olv)
        # the two solvers' 8-bit tables agree to ~3e-11 (see the test above)
        assert abs(alpha / oalpha - 1) < (1e-12 if bits <= 7 else 1e-10)
    assert lib.rbq_int8_levels(64, 0, None, None) == rbq.RBQ_EINVAL
    assert lib.rbq_int8_levels(0, 4, None, None) == rbq.RBQ_EINVAL


def test_error_strings(lib):
    for code in (0, -1, -2, -4, -5, -6, -99):
        assert isinstance(lib.rbq_error_string(code), bytes)


@pytest.mark.parametrize("d", [256, 1024, 3072, 8960, 12288])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_code_grid_lookup_matches_oracle(lib, d, bits):
    """The kernels' one-compare code search, evaluated here in fp32 with the
    library's table, equals the oracle's boundary count outside the band."""
    for variant in (0, 1):
        _check_grid_variant(d, bits, variant)


def _check_grid_variant(d, bits, variant):
    try:
        thr, base, cells, scale = rbq.code_grid(d, bits, variant)
    except rbq.RBQError as e:          # the [-1, 1] grid is only built while it stays small
        assert variant == 1 and e.code == rbq.RBQ_ECONVERGE and bits >= 7
        return
    assert cells % 2 == 0 and len(thr) == cells + 1
    _, bounds = oracle.lloydmax_table(d, bits)
    sigma = 1 / np.sqrt(d)
    g = np.random.default_rng(d * 16 + bits)
    v = np.concatenate([(g.standard_normal(300000) * sigma).astype(np.float32),
                        (g.uniform(-1, 1, 20000)).astype(np.float32),
                        np.float32([0.0, -0.0, 1.0, -1.0]), bounds.astype(np.float32),
                        np.nextafter(bounds.astype(np.float32), np.float32(np.inf)),
                        np.nextafter(bounds.astype(np.float32), np.float32(-np.inf))])
    u = np.clip(v * scale + np.float32(0.5), np.float32(0), np.float32(1)).astype(np.float32)
    q = (u * np.float32(cells) + np.float32(2.0 ** 23)).astype(np.float32)
    n = q.view(np.int32) - 0x4B000000
    assert n.min() >= 0 and n.max() <= cells
    code = base[n] + (v >= thr[n])
    ref = oracle.assign_codes(v.astype(np.float64), bounds)
    near = np.zeros(v.shape, dtype=bool)
    for t in bounds:
        near |= np.abs(v.astype(np.float64) - t) <= 1e-6 * max(abs(t), sigma)
    bad = (code != ref) & ~near
    assert not np.any(bad), (int(bad.sum()), v[bad][:5])
    # the zero coordinate takes the upper side of the middle boundary
    z = np.float32([0.0, -0.0])
    nz = (np.clip(z * scale + np.float32(0.5), 0, 1) * np.float32(cells) + np.float32(2.0 ** 23)).astype(np.float32)
    nn = nz.view(np.int32) - 0x4B000000
    assert np.all(base[nn] + (z >= thr[nn]) == 2 ** (bits - 1))


def test_binding_rejects_mismatched_layer_shapes():
    """The binding checks every operand's length before a call reaches the
    library: a short s or rnorm would be read past its end by the GEMM's
    epilogue, and a wrong out shape written past its end."""
    M, N, K, ba, bw = 100, 64, 256, 4, 3
    good = dict(a_shape=(M, K * ba // 8), s_shape=(M,), w_shape=(N, K * bw // 8), rn_shape=(N,), out_shape=(M, N))
    rbq.check_layer_shapes(M, N, K, ba, bw, **good)
    for key, bad in (("s_shape", (M - 1,)), ("rn_shape", (N + 8,)), ("out_shape", (M, N - 8)),
                     ("a_shape", (M, K * ba // 8 - 16)), ("w_shape", (N, K * 4 // 8)), ("s_shape", (M, 1))):
        with pytest.raises(ValueError):
            rbq.check_layer_shapes(M, N, K, ba, bw, **{**good, key: bad})
    with pytest.raises(ValueError):
        rbq.check_layer_shapes(M, N, 100, 3, bw, **good)            # 100 * 3 bits is not whole bytes


def test_binding_rejects_operands_on_different_devices():
    torch = pytest.importorskip("torch")
    a = torch.zeros(4)
    b = torch.zeros(4, device="meta")
    with pytest.raises(ValueError):
        rbq.check_same_device(a, b)
    assert rbq.check_same_device(a, None, torch.ones(2)) == torch.device("cpu")
