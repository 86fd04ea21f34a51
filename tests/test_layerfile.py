"""Quantised layer files (the "quantized model file" of the INT8-convrot page,
section 1: quantised weights, their quantisation parameters and the transform
info that reproduces the rotation).  Host-side: runs without a GPU, except the
last test, which checks that a layer read back gives the same output."""

import ctypes

import numpy as np
import pytest

import oracle
import rotation_bit_ptq_b200 as rbq


def _arrays(kind, rows, d, bits=4, seed=0):
    g = np.random.default_rng(seed)
    if kind == "lloydmax":
        return g.integers(0, 256, (rows, d * bits // 8), dtype=np.uint8), \
            g.integers(0, 2 ** 16, rows, dtype=np.uint16), None
    codes = g.integers(-127, 128, (rows, d), dtype=np.int8)
    if kind == "int8_asym":
        codes = codes.view(np.uint8)
    zp = g.integers(0, 256, rows, dtype=np.uint8) if kind == "int8_asym" else None
    return codes, g.random(rows).astype(np.float32), zp


@pytest.mark.parametrize("kind,bits,permute,signs", [("lloydmax", 4, True, True), ("lloydmax", 3, False, True),
                                                      ("int8", 8, True, True), ("int8_tensor", 8, True, False),
                                                      ("int8_asym", 8, False, False)])
def test_round_trip_and_transform_info(tmp_path, kind, bits, permute, signs):
    d, rows, seed = 1024, 24, 2 ** 63 + 5
    r = rbq.RPBH(d, seed, permute=permute, signs=signs)
    codes, aux, zp = _arrays(kind, rows, d, bits)
    path = tmp_path / "layer.rbq"
    rbq.save_layer(path, r, kind, codes, aux, zero_point=zp, bits=bits)
    L = rbq.load_layer(path)
    assert L["kind"] == kind and L["rows"] == rows and L["d"] == d and L["bits"] == (bits if kind == "lloydmax" else 8)
    assert np.array_equal(L["codes"].view(np.uint8), codes.view(np.uint8))
    assert np.array_equal(L["aux"].view(np.uint8), aux.view(np.uint8))
    if zp is not None:
        assert np.array_equal(L["zero_point"], zp)
    # the transform info rebuilds the same pi and D (and the oracle agrees)
    p0, s0 = r.export()
    p1, s1 = L["rpbh"].export()
    assert np.array_equal(p0, p1) and np.array_equal(s0, s1)
    op, os_ = oracle.rpbh_draw(d, seed)
    assert np.array_equal(p1, op if permute else np.arange(d))
    assert np.array_equal(s1, os_ if signs else np.ones(d))


def test_corrupt_short_and_foreign_files(tmp_path):
    r = rbq.RPBH(512, 1)
    codes, aux, _ = _arrays("int8", 8, 512)
    path = tmp_path / "a.rbq"
    rbq.save_layer(path, r, "int8", codes, aux)
    raw = path.read_bytes()
    lib = rbq.lib()
    info = rbq.LayerInfo()
    buf_c = np.empty(codes.nbytes, np.uint8)
    buf_a = np.empty(aux.nbytes, np.uint8)

    def read(p):
        return lib.rbq_layer_read(str(p).encode(), ctypes.byref(info), buf_c.ctypes.data_as(ctypes.c_void_p),
                                  buf_c.nbytes, buf_a.ctypes.data_as(ctypes.c_void_p), buf_a.nbytes, None, 0)

    assert read(path) == rbq.RBQ_OK
    bad = bytearray(raw)
    bad[64 + 100] ^= 1                              # one payload bit: checksum
    (tmp_path / "b.rbq").write_bytes(bytes(bad))
    assert read(tmp_path / "b.rbq") == rbq.RBQ_EIO
    (tmp_path / "c.rbq").write_bytes(raw[:-3])      # truncated
    assert read(tmp_path / "c.rbq") == rbq.RBQ_EIO
    (tmp_path / "d.rbq").write_bytes(raw + b"x")    # trailing bytes
    assert read(tmp_path / "d.rbq") == rbq.RBQ_EIO
    (tmp_path / "e.rbq").write_bytes(b"NOTALAYER" + raw[9:])
    assert read(tmp_path / "e.rbq") == rbq.RBQ_EIO
    assert read(tmp_path / "missing.rbq") == rbq.RBQ_EIO
    assert b"layer file" in lib.rbq_error_string(rbq.RBQ_EIO)


def test_read_rejects_a_file_larger_than_the_buffers(tmp_path):
    """A caller sizes its buffers from an info-only read; if the file is then
    replaced by one whose header asks for more bytes, the data read must refuse
    (RBQ_EINVAL) and leave the buffers untouched instead of overrunning them."""
    lib = rbq.lib()
    path = tmp_path / "layer.rbq"
    small, big = _arrays("int8", 8, 512), _arrays("int8", 16, 512, seed=1)
    rbq.save_layer(path, rbq.RPBH(512, 3), "int8", small[0], small[1])
    info = rbq.LayerInfo()
    assert lib.rbq_layer_read(str(path).encode(), ctypes.byref(info), None, 0, None, 0, None, 0) == rbq.RBQ_OK
    nc, na = ctypes.c_uint64(), ctypes.c_uint64()
    assert lib.rbq_layer_sizes(ctypes.byref(info), ctypes.byref(nc), ctypes.byref(na), None) == rbq.RBQ_OK
    buf_c = np.full(nc.value + 64, 0x5A, np.uint8)       # guard bytes past the sized part
    buf_a = np.full(na.value + 64, 0x5A, np.uint8)
    rbq.save_layer(path, rbq.RPBH(512, 3), "int8", big[0], big[1])          # swapped in between
    rc = lib.rbq_layer_read(str(path).encode(), ctypes.byref(info), buf_c.ctypes.data_as(ctypes.c_void_p), nc.value,
                            buf_a.ctypes.data_as(ctypes.c_void_p), na.value, None, 0)
    assert rc == rbq.RBQ_EINVAL
    assert np.all(buf_c == 0x5A) and np.all(buf_a == 0x5A)
    # sized for the new file, the same call reads it
    info2 = rbq.LayerInfo()
    lib.rbq_layer_read(str(path).encode(), ctypes.byref(info2), None, 0, None, 0, None, 0)
    lib.rbq_layer_sizes(ctypes.byref(info2), ctypes.byref(nc), ctypes.byref(na), None)
    bc, ba = np.empty(nc.value, np.uint8), np.empty(na.value, np.uint8)
    assert lib.rbq_layer_read(str(path).encode(), ctypes.byref(info2), bc.ctypes.data_as(ctypes.c_void_p), bc.nbytes,
                              ba.ctypes.data_as(ctypes.c_void_p), ba.nbytes, None, 0) == rbq.RBQ_OK
    assert np.array_equal(bc, big[0].view(np.uint8).reshape(-1))


def test_layer_sizes_and_invalid_descriptions():
    lib = rbq.lib()
    nc, na, nz = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    info = rbq.LayerInfo(3072, 64, 0, 0, rbq.RBQ_LAYER_LLOYDMAX, 4, 100)
    assert lib.rbq_layer_sizes(ctypes.byref(info), ctypes.byref(nc), ctypes.byref(na), ctypes.byref(nz)) == 0
    assert (nc.value, na.value, nz.value) == (100 * 3072 // 2, 200, 0)
    info = rbq.LayerInfo(3072, 64, 0, 0, rbq.RBQ_LAYER_INT8_ASYM, 8, 100)
    assert lib.rbq_layer_sizes(ctypes.byref(info), ctypes.byref(nc), ctypes.byref(na), ctypes.byref(nz)) == 0
    assert (nc.value, na.value, nz.value) == (100 * 3072, 400, 100)
    for bad in (rbq.LayerInfo(100, 64, 0, 0, 0, 4, 1), rbq.LayerInfo(128, 32, 0, 0, 0, 4, 1),
                rbq.LayerInfo(128, 64, 0, 4, 0, 4, 1), rbq.LayerInfo(128, 64, 0, 0, 9, 4, 1),
                rbq.LayerInfo(128, 64, 0, 0, rbq.RBQ_LAYER_INT8_SYM, 4, 1), rbq.LayerInfo(128, 64, 0, 0, 0, 9, 1),
                rbq.LayerInfo(128, 64, 0, 0, 0, 4, 0)):
        assert lib.rbq_layer_sizes(ctypes.byref(bad), None, None, None) == rbq.RBQ_EINVAL
    assert lib.rbq_layer_write(b"/nonexistent-dir/x.rbq", ctypes.byref(rbq.LayerInfo(128, 64, 0, 0, 1, 8, 1)),
                               ctypes.c_void_p(1), ctypes.c_void_p(1), None) == rbq.RBQ_EIO


@pytest.mark.gpu
def test_layer_read_back_gives_the_same_output(tmp_path):
    import torch
    from parity import torch_bf16
    import synth
    d, n = 1024, 64
    W = synth.to_bf16((np.random.default_rng(3).standard_normal((n, d)) * 0.02).astype(np.float32))
    X = synth.to_bf16(np.random.default_rng(4).standard_t(3, (40, d)).astype(np.float32))
    r = rbq.RPBH(d, 31)
    wc, rn = rbq.quantize_weights(r, torch_bf16(W), 4)
    a, s = rbq.rotate_quantize_act(r, torch_bf16(X), 4)
    y0 = rbq.qlinear(a, s, 4, wc, rn, 4, d)
    rbq.save_layer(tmp_path / "w.rbq", r, "lloydmax", wc, rn, bits=4)
    L = rbq.load_layer(tmp_path / "w.rbq", device="cuda")
    a1, s1 = rbq.rotate_quantize_act(L["rpbh"], torch_bf16(X), 4)      # the rebuilt transform
    y1 = rbq.qlinear(a1, s1, 4, L["codes"], L["aux"], L["bits"], d)
    torch.cuda.synchronize()
    assert rbq.device_error() == 0
    assert torch.equal(a, a1) and torch.equal(y0, y1)
