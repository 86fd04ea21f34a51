"""qlinear_noalloc: the quantised linear for callers that cannot allocate.

Some hosts cannot let a library allocate device memory: they own all of it
through their own allocator, forbid allocation on the inference thread, or
load the library into a process whose allocator is not CUDA's.  For them the
library exports qlinear_noalloc, which keeps the fp16 weight workspace in a
fixed array inside the library instead of taking it from a memory pool.

The GPU test calls it through the C ABI on two different problems in a row
and then on the first one again, and compares each result with the ordinary
qlinear on the same inputs.  The second call overwrites the workspace the
first one used, so the test also shows that nothing stale from one call leaks
into the next; the third call finds its level tables already in the array's
slots and copies nothing before its kernels.  This file is named to be
collected last.
"""

import ctypes

import numpy as np
import pytest

import rotation_bit_ptq_b200 as rbq
import synth

QLINEAR_RTOL = 4e-3      # the tolerance the qlinear parity tests use


def test_noalloc_rejects_problems_beyond_its_scratch():
    # Validation runs before any CUDA call, so fake non-null pointers are safe
    # here and no GPU is needed: N*K = 8192*4096 > 2**24 -> RBQ_ESCRATCH.
    lib = rbq.lib()
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.qlinear_noalloc(fake, fake, 4, fake, fake, 4, 128, 8192, 4096, fake, None, None)
    assert rc == rbq.RBQ_ESCRATCH
    assert b"scratch" in lib.rbq_error_string(rc)
    # K not a multiple of 128 is outside the kernel it wraps
    assert lib.qlinear_noalloc(fake, fake, 4, fake, fake, 4, 128, 256, 192, fake, None, None) == rbq.RBQ_EINVAL


def _problem(M, N, K, ba, bw, seed):
    import torch
    from parity import torch_bf16
    g = np.random.default_rng(seed)
    X = synth.to_bf16(g.standard_t(3, (M, K)).astype(np.float32))
    W = synth.to_bf16((g.standard_normal((N, K)) * 0.02).astype(np.float32))
    r = rbq.RPBH(K, seed)
    a_codes, s = rbq.rotate_quantize_act(r, torch_bf16(X), ba)
    w_codes, rn = rbq.quantize_weights(r, torch_bf16(W), bw)
    torch.cuda.synchronize()
    r.close()
    return a_codes, s, w_codes, rn


@pytest.mark.gpu
def test_noalloc_matches_qlinear_on_two_calls_in_a_row():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from parity import bf16_to_numpy, rel_frobenius

    cases = [(4608, 3072, 3072, 4, 4, 11),      # the attention-projection layer
             (300, 1032, 1024, 3, 2, 12)]       # ragged M, smaller N, other widths
    probs = [_problem(*c) for c in cases]
    cases, probs = cases + cases[:1], probs + probs[:1]       # the first widths again: tables already in place
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for (M, N, K, ba, bw, _), (a, s, w, rn) in zip(cases, probs):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rbq.qlinear_noalloc(a, s, ba, w, rn, bw, K, y, err=err)
        outs.append(y)
    torch.cuda.synchronize()
    assert err.item() == 0
    for (M, N, K, ba, bw, _), (a, s, w, rn), y in zip(cases, probs, outs):
        ref = rbq.qlinear(a, s, ba, w, rn, bw, K)
        torch.cuda.synchronize()
        assert rbq.device_error() == 0
        got_np, ref_np = bf16_to_numpy(y), bf16_to_numpy(ref)
        assert np.all(np.isfinite(got_np))
        e = rel_frobenius(got_np, ref_np)
        print(f"qlinear_noalloc {M}x{N}x{K} W{bw}A{ba}: rel. Frobenius vs qlinear {e:.2e}, "
              f"{int(np.sum(got_np != ref_np))} differing elements")
        assert e < QLINEAR_RTOL, e


@pytest.mark.gpu
@pytest.mark.parametrize("ba,bw", [(1, 4), (2, 3), (3, 4), (4, 4), (5, 2), (6, 4), (7, 8), (8, 1)])
def test_noalloc_against_the_oracle_every_activation_width(ba, bw):
    """qlinear_noalloc always expands the activation codes inside the GEMM (it
    has no workspace for them), so it is also where that route meets the
    oracle at sizes below qlinear's 2 GiB switch: random codes, ragged M and
    N, every activation width."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from parity import bf16_to_numpy, rel_frobenius
    M, N, K = 300, 264, 1024
    gen = torch.Generator(device="cuda").manual_seed(ba * 16 + bw)
    a = torch.randint(0, 256, (M, K * ba // 8), dtype=torch.uint8, device="cuda", generator=gen)
    w = torch.randint(0, 256, (N, K * bw // 8), dtype=torch.uint8, device="cuda", generator=gen)
    s = torch.rand(M, device="cuda", generator=gen) + 0.5
    rn = (torch.rand(N, device="cuda", generator=gen) + 0.5).to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    rbq.qlinear_noalloc(a, s, ba, w, rn, bw, K, y, err=err)
    torch.cuda.synchronize()
    assert err.item() == 0 and rbq.device_error() == 0
    la, _ = oracle.lloydmax_table(K, ba)
    lw, _ = oracle.lloydmax_table(K, bw)
    ref = oracle.qlinear(oracle.unpack_codes(a.cpu().numpy(), ba, K), s.cpu().numpy(), la,
                         oracle.unpack_codes(w.cpu().numpy(), bw, K), bf16_to_numpy(rn), lw)
    e = rel_frobenius(bf16_to_numpy(y), ref)
    assert e < QLINEAR_RTOL, e
