"""Failure handling of the kernels' waits, checked without faulting the GPU.

Every wait the kernels make on a shared-memory barrier has an iteration and
clock limit; when it runs out the kernel records a bit in the library's
device error word and returns, so a lost arrival shows up as RBQ_EDEVICE on
the host instead of a hung GPU.  rbq_selftest_wait_limit launches a CTA whose
barriers nothing ever arrives at: each wait form must give up on its own
within about a second, the error must reach the host, and the context must
stay usable (a quantisation run after it gives the same bytes as one before).
"""

import ctypes
import time

import numpy as np
import pytest

import rotation_bit_ptq_b200 as rbq
import synth


def test_selftest_validates_its_pointer():
    lib = rbq.lib()
    assert lib.rbq_selftest_wait_limit(None, None) == rbq.RBQ_EINVAL
    assert lib.rbq_selftest_wait_limit(ctypes.c_void_p((1 << 20) + 2), None) == rbq.RBQ_EALIGN


@pytest.mark.gpu
def test_every_wait_form_gives_up_and_the_context_survives():
    import torch
    from parity import torch_bf16

    d, T, bits = 1024, 40, 4
    X, _ = synth.student_t_act(T, d, seed=21)
    r = rbq.RPBH(d, 9)
    xt = torch_bf16(X)
    before = [t.clone() for t in rbq.rotate_quantize_act(r, xt, bits)]
    torch.cuda.synchronize()
    assert rbq.device_error() == 0

    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    rbq.selftest_wait_limit(out)
    assert rbq.device_error() == rbq.RBQ_EDEVICE      # the give-up reached the host ...
    elapsed = time.perf_counter() - t0
    assert rbq.device_error() == 0                      # ... and reading it cleared it
    assert int(out.item()) == 15                        # all three forms + the shared flag
    assert elapsed < 30.0                               # ended by its own limit

    after = rbq.rotate_quantize_act(r, xt, bits)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    for a, b in zip(before, after):
        assert torch.equal(a, b)
