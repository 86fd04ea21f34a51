"""The debug build of the library (librbq_debug.so, compiled with RBQ_DEBUG).

Its kernels check the indices they compute on the device -- gather offsets
read from the permutation tables, code-grid entries derived from floats --
against their bounds before each access; an index out of range is recorded in
the device error word (rbq_device_error then reports RBQ_EDEVICE) and replaced
by one inside the buffer, so nothing traps.  The checks change no arithmetic:
on valid inputs the debug build must give the release build's bytes exactly,
with a clean error word.
"""

import ctypes

import numpy as np
import pytest

import rotation_bit_ptq_b200 as rbq
import synth


def test_debug_library_exports_every_symbol():
    dbg = rbq.debug_lib()
    rel = rbq.lib()
    for name in rbq.SIGNATURES:
        assert hasattr(dbg, name) and hasattr(rel, name), name
    # host-side paths agree (no device needed): the Lloyd-Max table
    a, b = np.empty(16), np.empty(15)
    c, e = np.empty(16), np.empty(15)
    assert dbg.lloydmax_table(3072, 4, a.ctypes.data_as(ctypes.c_void_p), b.ctypes.data_as(ctypes.c_void_p)) == 0
    assert rel.lloydmax_table(3072, 4, c.ctypes.data_as(ctypes.c_void_p), e.ctypes.data_as(ctypes.c_void_p)) == 0
    assert np.array_equal(a, c) and np.array_equal(b, e)


@pytest.mark.gpu
@pytest.mark.parametrize("d,T,bits,dtype", [(3072, 37, 4, "bf16"),    # token-pair kernel
                                            (1280, 40, 6, "bf16"),    # token-pair kernel, wide codebook
                                            (4096, 9, 3, "bf16"),     # register-staged kernel
                                            (12288, 5, 8, "bf16"),    # register-staged, clamped grid
                                            (512, 33, 2, "f32")])     # general kernel
def test_debug_build_matches_release_with_a_clean_error_word(d, T, bits, dtype):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from parity import poison, torch_bf16
    dbg = rbq.debug_lib()
    X, _ = synth.student_t_act(T, d, seed=d + bits)
    W = synth.to_bf16((np.random.default_rng(d).standard_normal((64, d)) * 0.02).astype(np.float32))
    if dtype == "bf16":
        xt, wt, code = torch_bf16(X), torch_bf16(W), rbq.RBQ_BF16
    else:
        xt = torch.from_numpy(X).cuda()
        wt = torch.from_numpy(W).cuda()
        code = rbq.RBQ_F32
    seed = 17
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # release build, through the binding
    r = rbq.RPBH(d, seed)
    a_rel, s_rel = rbq.rotate_quantize_act(r, xt, bits)
    w_rel, rn_rel = rbq.quantize_weights(r, wt, 4)
    y_rel = rbq.qlinear(a_rel, s_rel, bits, w_rel, rn_rel, 4, d) if d % 128 == 0 else None
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    # debug build, through its own C ABI
    h = ctypes.c_void_p()
    assert dbg.rpbh_make(d, 64, ctypes.c_uint64(seed), ctypes.byref(h)) == 0
    a_dbg, s_dbg = poison(tuple(a_rel.shape), torch.uint8), poison((T,), torch.float32)
    w_dbg, rn_dbg = poison(tuple(w_rel.shape), torch.uint8), poison((64,), torch.bfloat16)
    assert dbg.rotate_quantize_act(h, ctypes.c_void_p(xt.data_ptr()), code, T, bits,
                                   ctypes.c_void_p(a_dbg.data_ptr()), ctypes.c_void_p(s_dbg.data_ptr()), stream) == 0
    assert dbg.quantize_weights(h, ctypes.c_void_p(wt.data_ptr()), code, 64, rbq.RBQ_LLOYDMAX, 4,
                                ctypes.c_void_p(w_dbg.data_ptr()), ctypes.c_void_p(rn_dbg.data_ptr()), stream) == 0
    if y_rel is not None:
        y_dbg = poison(tuple(y_rel.shape), torch.bfloat16)
        assert dbg.qlinear(ctypes.c_void_p(a_dbg.data_ptr()), ctypes.c_void_p(s_dbg.data_ptr()), bits,
                           ctypes.c_void_p(w_dbg.data_ptr()), ctypes.c_void_p(rn_dbg.data_ptr()), 4, T, 64, d,
                           ctypes.c_void_p(y_dbg.data_ptr()), stream) == 0
    assert dbg.rbq_device_error(stream) == 0
    dbg.rpbh_free(h)
    assert torch.equal(a_rel, a_dbg) and torch.equal(s_rel, s_dbg)
    assert torch.equal(w_rel, w_dbg) and torch.equal(rn_rel.view(torch.int16), rn_dbg.view(torch.int16))
    if y_rel is not None:
        assert torch.equal(y_rel.view(torch.int16), y_dbg.view(torch.int16))
    r.close()
