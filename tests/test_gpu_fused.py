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
