"""The rotation fused into the producing matmul (OrbitQuant §6.2), against the
oracle's composition on the weights in their original row order.

qlinear_int8_rotate_next runs the W8A16 layer on weight rows reordered by the
next layer's permutation and finishes the next layer's rotation in its
epilogue; the oracle computes Pi_next act(qlinear_int8(x', q, scale)) in fp64
with q and scale as quantize_weights returned them.  The kernel sums in fp32
on the tensor cores and rounds once to BF16, so the bar is the relative
Frobenius error of the other W8A16 parity tests (3e-3, well under the stated
2e-2)."""

import numpy as np
import pytest

import oracle
import synth
from parity import bf16_to_numpy, poison, rel_frobenius, torch_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import rotation_bit_ptq_b200 as rbq  # noqa: E402

FUSED_RTOL = 3e-3


def _pi(d, seed):
    perm, signs = oracle.rpbh_draw(d, seed)
    return oracle.rpbh_matrix(perm, signs) if d <= 4096 else (perm, signs)


def test_rows_in_next_order_is_the_permutation():
    nxt = rbq.RPBH(1024, 77)
    perm, _ = nxt.export()
    q = torch.randint(-127, 128, (1024, 320), dtype=torch.int8, device="cuda")
    sc = torch.rand(1024, device="cuda")
    q2, sc2 = rbq.rows_in_next_order(nxt, q), rbq.rows_in_next_order(nxt, sc)
    idx = torch.as_tensor(perm.astype(np.int64)).cuda()
    assert torch.equal(q2, q[idx]) and torch.equal(sc2, sc[idx])
    with pytest.raises(ValueError):
        rbq.rows_in_next_order(nxt, q[:512].contiguous())


def _fused_case(M, K, N, act, rows=None, seed=0):
    """Producing layer K -> N (rotation seed `seed`), next layer of width N."""
    g = np.random.default_rng(M * 7 + K + N + seed)
    X = synth.to_bf16(g.standard_t(3, (M, K)).astype(np.float32))
    W = synth.to_bf16(synth.gaussian_weights(g, N, K, outlier_frac=0.01))
    r, nxt = rbq.RPBH(K, seed), rbq.RPBH(N, seed + 1000)
    xr = rbq.rotate_act(r, torch_bf16(X))
    q, sc = rbq.quantize_weights(r, torch_bf16(W), 8, mode="int8")
    qn, scn = rbq.rows_in_next_order(nxt, q), rbq.rows_in_next_order(nxt, sc)
    out = poison((M, N), torch.bfloat16)
    y = rbq.qlinear_int8_rotate_next(xr, qn, scn, nxt, activation=act, out=out)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    rows = np.arange(M) if rows is None else np.asarray(rows)
    idx = torch.as_tensor(rows).cuda()
    ref = oracle.qlinear_int8_rotate_next(bf16_to_numpy(xr[idx]), q.cpu().numpy().astype(np.float64),
                                          sc.cpu().numpy().astype(np.float64), _pi(N, seed + 1000), activation=act)
    got = bf16_to_numpy(y[idx])
    assert np.all(np.isfinite(got))
    return rel_frobenius(got, ref), (xr, q, sc, nxt, y, idx)


@pytest.mark.parametrize("M,K,N,act", [(1, 64, 64, "gelu"), (130, 256, 512, "gelu"), (77, 192, 1024, "none"),
                                       (300, 512, 1536, "gelu"), (129, 1024, 320, "none")])
def test_fused_layer_ragged_shapes(M, K, N, act):
    err, _ = _fused_case(M, K, N, act)
    print(f"fused W8A16 -> rotation {M}x{K}->{N} act={act}: rel. Frobenius error {err:.2e}")
    assert err < FUSED_RTOL, err


def test_fused_layer_matches_the_unfused_pipeline():
    """The same layer run unfused on the GPU -- qlinear_int8, GELU in fp32,
    rotate_act -- agrees with the fused one up to the BF16 roundings the fused
    path skips (y and GELU(y) are not rounded to BF16 there)."""
    err, (xr, q, sc, nxt, y, idx) = _fused_case(200, 512, 1024, "gelu", seed=5)
    assert err < FUSED_RTOL
    y_un = rbq.qlinear_int8(xr, q, sc)
    g = torch.nn.functional.gelu(y_un.float()).to(torch.bfloat16)
    x_un = rbq.rotate_act(nxt, g)
    torch.cuda.synchronize()
    assert rel_frobenius(bf16_to_numpy(y), bf16_to_numpy(x_un)) < 1e-2


def test_fused_layer_dit_mlp_up_into_down_sampled():
    """The single-stream DiT block's MLP: up 4096 -> 16384 (4096 tokens) whose
    GELU output is the down-projection's input, rotated at d = 16384."""
    rows = np.random.default_rng(8).choice(4096, 12, replace=False)
    M, K, N = 4096, 4096, 16384
    W = synth.int8_dit_weight(0, "up")
    X = synth.int8_dit_act(K)
    r, nxt = rbq.RPBH(K, 100 + K), rbq.RPBH(N, 200 + N)
    xr = rbq.rotate_act(r, torch_bf16(X))
    q, sc = rbq.quantize_weights(r, torch_bf16(W), 8, mode="int8")
    qn, scn = rbq.rows_in_next_order(nxt, q), rbq.rows_in_next_order(nxt, sc)
    y = rbq.qlinear_int8_rotate_next(xr, qn, scn, nxt, activation="gelu", out=poison((M, N), torch.bfloat16))
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    idx = torch.as_tensor(rows).cuda()
    ref = oracle.qlinear_int8_rotate_next(bf16_to_numpy(xr[idx]), q.cpu().numpy().astype(np.float64),
                                          sc.cpu().numpy().astype(np.float64), _pi(N, 200 + N), activation="gelu")
    err = rel_frobenius(bf16_to_numpy(y[idx]), ref)
    print(f"fused DiT MLP up -> down rotation: rel. Frobenius error {err:.2e}")
    assert err < FUSED_RTOL, err


# --------------------------------------------------------------------------
# The code layer (OrbitQuant §2.2) fused with the next rotation, and the
# next layer's quantiser on the rotated rows (quantize_rotated)
# --------------------------------------------------------------------------

from parity import check_codes, check_rel  # noqa: E402

QLINEAR_RTOL = 4e-3        # rel. Frobenius, fp16 operands + BF16 output (bar: 2e-2)
NORM_RTOL = 1e-5


def _unpack(codes, bits, d):
    return oracle.unpack_codes(codes.cpu().numpy(), bits, d)


def _fused_codes_case(M, K, N, ba, bw, act, seed=0):
    g = np.random.default_rng(M * 5 + K + N + ba + bw + seed)
    X = synth.to_bf16(g.standard_t(3, (M, K)).astype(np.float32))
    W = synth.to_bf16(synth.gaussian_weights(g, N, K, outlier_frac=0.01))
    r, nxt = rbq.RPBH(K, seed + 3), rbq.RPBH(N, seed + 2000)
    a, s = rbq.rotate_quantize_act(r, torch_bf16(X), ba)
    w, rn = rbq.quantize_weights(r, torch_bf16(W), bw)
    wn, rnn = rbq.rows_in_next_order(nxt, w), rbq.rows_in_next_order(nxt, rn)
    y = rbq.qlinear_rotate_next(a, s, ba, wn, rnn, bw, K, nxt, activation=act, out=poison((M, N), torch.bfloat16))
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    la, _ = oracle.lloydmax_table(K, ba)
    lw, _ = oracle.lloydmax_table(K, bw)
    ref = oracle.qlinear_rotate_next(_unpack(a, ba, K), s.cpu().numpy().astype(np.float64), la, _unpack(w, bw, K),
                                     rn.float().cpu().numpy().astype(np.float64), lw, _pi(N, seed + 2000),
                                     activation=act)
    got = bf16_to_numpy(y)
    assert np.all(np.isfinite(got))
    return rel_frobenius(got, ref), (a, s, w, rn, r, nxt, y)


@pytest.mark.parametrize("M,K,N,ba,bw,act", [(1, 128, 64, 4, 4, "gelu"), (130, 256, 512, 4, 2, "gelu"),
                                             (77, 384, 1024, 3, 3, "none"), (300, 512, 1536, 6, 4, "gelu"),
                                             (257, 1024, 320, 2, 4, "none")])
def test_fused_code_layer_ragged_shapes(M, K, N, ba, bw, act):
    err, _ = _fused_codes_case(M, K, N, ba, bw, act)
    print(f"fused W{bw}A{ba} -> rotation {M}x{K}->{N} act={act}: rel. Frobenius error {err:.2e}")
    assert err < QLINEAR_RTOL, err


@pytest.mark.parametrize("d,T,bits", [(64, 3, 1), (512, 40, 8), (1024, 37, 4), (3072, 130, 2), (3072, 65, 3),
                                      (1536, 33, 6), (12288, 9, 5), (16384, 4, 7)])
def test_quantize_rotated_matches_the_oracle(d, T, bits):
    X, _ = synth.student_t_act(T, d, seed=d + bits)
    X = X.copy()
    X[0] = 0.0                                  # zero row: s = 0, every code 2^(b-1)
    if T > 2:
        X[2, 5] = np.nan                        # non-finite row: encoded as the zero vector
    r = rbq.RPBH(d, 31)
    xr = rbq.rotate_act(r, torch_bf16(X))
    codes, norms = rbq.quantize_rotated(xr, bits, codes=poison((T, d * bits // 8), torch.uint8),
                                        norms=poison((T,), torch.float32))
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    g = _unpack(codes, bits, d)
    assert np.all(g[0] == 2 ** (bits - 1)) and norms[0].item() == 0.0
    good = np.arange(T) if T <= 2 else np.setdiff1d(np.arange(T), [2])
    if T > 2:
        assert np.all(g[2] == 2 ** (bits - 1))
    _, bounds = oracle.lloydmax_table(d, bits)
    ora = oracle.quantize_rotated(bf16_to_numpy(xr)[good], bounds)
    check_codes(g[good], ora["codes"], ora["v"], bounds, d)
    check_rel(norms.cpu().numpy()[good], ora["norms"], NORM_RTOL, "quantize_rotated norms")


def test_fused_code_pipeline_against_the_unfused_one():
    """The next layer's codes through the fused path (qlinear_rotate_next, then
    quantize_rotated) and through the unfused one (qlinear, GELU, then
    rotate_quantize_act) differ only where the two paths' BF16 roundings (of
    x' in the first, of y and GELU(y) in the second) move a value across a
    decision boundary: few codes, each by one level."""
    M, K, N, ba, bw = 256, 1024, 3072, 4, 4
    err, (a, s, w, rn, r, nxt, y) = _fused_codes_case(M, K, N, ba, bw, "gelu", seed=9)
    assert err < QLINEAR_RTOL
    c_f, s_f = rbq.quantize_rotated(y, 4)
    y_un = rbq.qlinear(a, s, ba, w, rn, bw, K)
    x_un = torch.nn.functional.gelu(y_un.float()).to(torch.bfloat16)
    c_u, s_u = rbq.rotate_quantize_act(nxt, x_un, 4)
    torch.cuda.synchronize()
    g_f, g_u = _unpack(c_f, 4, N), _unpack(c_u, 4, N)
    diff = g_f != g_u
    assert diff.mean() < 0.02, diff.mean()
    assert np.all(np.abs(g_f[diff] - g_u[diff]) == 1)
    check_rel(s_f.cpu().numpy(), s_u.cpu().numpy(), 1e-2, "norms, fused vs unfused")
