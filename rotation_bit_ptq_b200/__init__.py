"""Python binding of librbq.so, the B200 rotate-then-quantize library.

Argument marshalling only: every step of the path runs inside the library's
CUDA kernels (see include/rbq.h for the C ABI).  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the library is
missing every call raises.

Sources: the OrbitQuant write-up (hotelren.com/news/3376620) §2.1-§2.3 and
§4.2, and INT8-convrot (cloud.baidu.com/article/9430339) §4.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librbq.so")
LIB_DEBUG_PATH = os.path.join(_HERE, "librbq_debug.so")

RBQ_F32, RBQ_BF16 = 0, 1
RBQ_LLOYDMAX, RBQ_INT8_SYM, RBQ_INT8_TENSOR = 0, 1, 2
RBQ_ROTATE_ONLY = 16
RBQ_OK, RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA, RBQ_ENOMEM, RBQ_ECONVERGE, RBQ_EDEVICE = 0, -1, -2, -3, -4, -5, -6
RBQ_ESCRATCH = -7
RBQ_RPBH_NO_PERMUTATION, RBQ_RPBH_NO_SIGNS = 1, 2
RBQ_EIO = -8
RBQ_ACT_NONE, RBQ_ACT_GELU = 0, 1
_ACTS = {None: RBQ_ACT_NONE, "none": RBQ_ACT_NONE, "gelu": RBQ_ACT_GELU}
RBQ_LAYER_LLOYDMAX, RBQ_LAYER_INT8_SYM, RBQ_LAYER_INT8_TENSOR, RBQ_LAYER_INT8_ASYM = 0, 1, 2, 3
_LAYER_KINDS = {"lloydmax": RBQ_LAYER_LLOYDMAX, "int8": RBQ_LAYER_INT8_SYM, "int8_tensor": RBQ_LAYER_INT8_TENSOR,
                "int8_asym": RBQ_LAYER_INT8_ASYM}


class LayerInfo(ctypes.Structure):
    """rbq_layer_info of include/rbq.h."""
    _fields_ = [("d", ctypes.c_int32), ("h", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("rpbh_flags", ctypes.c_int32), ("mode", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("rows", ctypes.c_int32)]

# name -> (restype, argtypes); mirrors include/rbq.h
_P, _I, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
SIGNATURES = {
    "rpbh_make": (_I, [_I, _I, _U64, ctypes.POINTER(_P)]),
    "rpbh_make_ablation": (_I, [_I, _I, _U64, _I, ctypes.POINTER(_P)]),
    "rpbh_free": (None, [_P]),
    "rpbh_export": (_I, [_P, _P, _P]),
    "rpbh_dim": (_I, [_P]),
    "rpbh_describe": (_I, [_P, _P, _P, _P, _P]),
    "rbq_layer_sizes": (_I, [_P, _P, _P, _P]),
    "rbq_layer_write": (_I, [ctypes.c_char_p, _P, _P, _P, _P]),
    "rbq_layer_read": (_I, [ctypes.c_char_p, _P, _P, _U64, _P, _U64, _P, _U64]),
    "lloydmax_table": (_I, [_I, _I, _P, _P]),
    "rotate_quantize_act": (_I, [_P, _P, _I, _I, _I, _P, _P, _P]),
    "quantize_weights": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "qlinear": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P]),
    "qlinear_int8": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "quantize_weights_int8_asym": (_I, [_P, _P, _I, _I, _P, _P, _P, _P]),
    "qlinear_int8_asym": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "qlinear_noalloc": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "qlinear_int8_levels": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P]),
    "rbq_int8_levels": (_I, [_I, _I, _P, _P]),
    "qlinear_fp8_levels": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P]),
    "rbq_fp8_levels": (_I, [_I, _I, _P, _P]),
    "rbq_error_string": (ctypes.c_char_p, [_I]),
    "rbq_device_error": (_I, [_P]),
    "rbq_selftest_wait_limit": (_I, [_P, _P]),
    "rbq_code_grid": (_I, [_I, _I, _I, _P, _P, _P, _P]),
    "rpbh_gather_rows": (_I, [_P, _P, ctypes.c_longlong, _P, _P]),
    "qlinear_int8_rotate_next": (_I, [_P, _P, _P, _I, _I, _P, _I, _P, _P]),
    "qlinear_rotate_next": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P, _P]),
    "quantize_rotated": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
}

_lib = None


class RBQError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        msg = lib().rbq_error_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{where}: {msg} ({code})")


def lib():
    """Load librbq.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m rotation_bit_ptq_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


_debug_lib = None


def debug_lib():
    """librbq_debug.so: the same kernels built with RBQ_DEBUG, whose
    device-side bounds checks on computed indices record into the device error
    word instead of trapping.  Loaded beside librbq.so with the same
    signatures, for tests and debugging only; its handles, codebook cache and
    error word are its own.  Raises if it has not been built."""
    global _debug_lib
    if _debug_lib is None:
        if not os.path.exists(LIB_DEBUG_PATH):
            raise RuntimeError(f"{LIB_DEBUG_PATH} is missing: build it with "
                               "`python -m rotation_bit_ptq_b200.build --debug`")
        handle = ctypes.CDLL(LIB_DEBUG_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _debug_lib = handle
    return _debug_lib


def _check(rc, where):
    if rc != RBQ_OK:
        raise RBQError(rc, where)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need_cuda(t, name, dtype=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _need_shape(t, shape, name):
    """Caller-supplied buffers must have exactly the shape the kernel writes or
    reads; a short one would be overrun on the device."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def check_layer_shapes(M, N, K, bits_a, bits_w, a_shape, s_shape, w_shape, rn_shape, out_shape=None):
    """Shapes of a quantised linear layer's operands (pure Python, no device):
    a_codes [M, K*bits_a/8], s [M], w_codes [N, K*bits_w/8], rnorm [N],
    out [M, N].  Raises ValueError on any mismatch."""
    if K <= 0 or (K * bits_a) % 8 or (K * bits_w) % 8:
        raise ValueError("K times each bit width must be a whole number of bytes")
    if tuple(a_shape) != (M, K * bits_a // 8) or tuple(w_shape) != (N, K * bits_w // 8):
        raise ValueError("code row widths do not match K and the bit widths")
    if tuple(s_shape) != (M,):
        raise ValueError(f"s must have shape ({M},), got {tuple(s_shape)}")
    if tuple(rn_shape) != (N,):
        raise ValueError(f"rnorm must have shape ({N},), got {tuple(rn_shape)}")
    if out_shape is not None and tuple(out_shape) != (M, N):
        raise ValueError(f"out must have shape ({M}, {N}), got {tuple(out_shape)}")


def check_same_device(*tensors):
    """Every operand of one call on one device (the library launches on the
    device that is current, which the binding sets to that one)."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) > 1:
        raise ValueError(f"operands are on different devices: {sorted(str(d) for d in devs)}")
    return next(iter(devs)) if devs else None


def _device_ctx(*tensors):
    import torch
    return torch.cuda.device(check_same_device(*tensors))


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return RBQ_BF16
    if t.dtype == torch.float32:
        return RBQ_F32
    raise TypeError("dense inputs must be bfloat16 or float32")


# ---------------------------------------------------------------------------
# RPBH handle and codebook (host)
# ---------------------------------------------------------------------------

class RPBH:
    """Pi_d = blkdiag(H_64 D_1, ..., H_64 D_{d/64}) · P_pi drawn from `seed`.

    permute=False gives pi = identity and signs=False gives D = +1 (the
    ablations of OrbitQuant §3.3, through rpbh_make_ablation)."""

    def __init__(self, d, seed, h=64, permute=True, signs=True):
        out = ctypes.c_void_p()
        flags = (0 if permute else RBQ_RPBH_NO_PERMUTATION) | (0 if signs else RBQ_RPBH_NO_SIGNS)
        if flags:
            _check(lib().rpbh_make_ablation(int(d), int(h), ctypes.c_uint64(seed & (2 ** 64 - 1)), flags,
                                            ctypes.byref(out)), "rpbh_make_ablation")
        else:
            _check(lib().rpbh_make(int(d), int(h), ctypes.c_uint64(seed & (2 ** 64 - 1)), ctypes.byref(out)),
                   "rpbh_make")
        self._h = out
        self.d = int(d)
        self.seed = int(seed)

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("RPBH handle already freed")
        return self._h

    @classmethod
    def from_description(cls, d, seed, flags, h=64):
        return cls(d, seed, h=h, permute=not (flags & RBQ_RPBH_NO_PERMUTATION),
                   signs=not (flags & RBQ_RPBH_NO_SIGNS))

    def describe(self):
        """(d, h, seed, flags): the transform info that rebuilds this handle."""
        d, h, flags = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        seed = ctypes.c_uint64()
        _check(lib().rpbh_describe(self.handle, ctypes.byref(d), ctypes.byref(h), ctypes.byref(seed),
                                   ctypes.byref(flags)), "rpbh_describe")
        return d.value, h.value, seed.value, flags.value

    def export(self):
        perm = np.empty(self.d, dtype=np.int32)
        signs = np.empty(self.d, dtype=np.int8)
        _check(lib().rpbh_export(self.handle, perm.ctypes.data_as(_P), signs.ctypes.data_as(_P)),
               "rpbh_export")
        return perm, signs

    def close(self):
        if getattr(self, "_h", None) is not None and _lib is not None:
            _lib.rpbh_free(self._h)
        self._h = None

    def __del__(self):
        self.close()


def lloydmax_table(d, bits):
    """(levels[2^bits], bounds[2^bits - 1]) of the N(0, 1/d) Lloyd-Max quantiser."""
    L = 2 ** int(bits)
    levels = np.empty(L, dtype=np.float64)
    bounds = np.empty(L - 1, dtype=np.float64)
    _check(lib().lloydmax_table(int(d), int(bits), levels.ctypes.data_as(_P), bounds.ctypes.data_as(_P)),
           "lloydmax_table")
    return levels, bounds


# ---------------------------------------------------------------------------
# kernels
# ---------------------------------------------------------------------------

def rotate_quantize_act(rpbh, X, bits, codes=None, norms=None, stream=None):
    """Packed codes uint8[T, d*bits/8] and norms float32[T] of the rows of X."""
    import torch
    _need_cuda(X, "X")
    T, d = X.shape
    if d != rpbh.d:
        raise ValueError("X width does not match the RPBH handle")
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=X.device)
    if norms is None:
        norms = torch.empty((T,), dtype=torch.float32, device=X.device)
    _need_cuda(codes, "codes", torch.uint8)
    _need_cuda(norms, "norms", torch.float32)
    _need_shape(codes, (T, d * bits // 8), "codes")
    _need_shape(norms, (T,), "norms")
    with _device_ctx(X, codes, norms):
        _check(lib().rotate_quantize_act(rpbh.handle, _ptr(X), _dtype_code(X), T, int(bits), _ptr(codes),
                                         _ptr(norms), _stream(stream)), "rotate_quantize_act")
    return codes, norms


def rotate_act(rpbh, X, out=None, norms=None, stream=None):
    """x' = Pi x in BF16 (the activation operand of qlinear_int8)."""
    import torch
    _need_cuda(X, "X")
    T, d = X.shape
    if d != rpbh.d:
        raise ValueError("X width does not match the RPBH handle")
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=X.device)
    _need_cuda(out, "out", torch.bfloat16)
    _need_shape(out, (T, d), "out")
    if norms is not None:
        _need_cuda(norms, "norms", torch.float32)
        _need_shape(norms, (T,), "norms")
    with _device_ctx(X, out, norms):
        _check(lib().rotate_quantize_act(rpbh.handle, _ptr(X), _dtype_code(X), T, RBQ_ROTATE_ONLY, _ptr(out),
                                         _ptr(norms), _stream(stream)), "rotate_quantize_act")
    return out


def quantize_weights(rpbh, W, bits, mode="lloydmax", out=None, aux=None, stream=None):
    """Offline weights.  mode='lloydmax': (codes uint8, r' bfloat16[N]);
    mode='int8': (q int8[N, d], scale float32[N]) with one scale per row;
    mode='int8_tensor': the same with one scale for the tensor (repeated)."""
    import torch
    _need_cuda(W, "W")
    N, d = W.shape
    if d != rpbh.d:
        raise ValueError("W width does not match the RPBH handle")
    if mode == "lloydmax":
        code = RBQ_LLOYDMAX
        if out is None:
            out = torch.empty((N, d * bits // 8), dtype=torch.uint8, device=W.device)
        if aux is None:
            aux = torch.empty((N,), dtype=torch.bfloat16, device=W.device)
        _need_cuda(out, "codes", torch.uint8)
        _need_cuda(aux, "rnorm", torch.bfloat16)
        _need_shape(out, (N, d * bits // 8), "codes")
    elif mode in ("int8", "int8_tensor"):
        code, bits = (RBQ_INT8_SYM if mode == "int8" else RBQ_INT8_TENSOR), 8
        if out is None:
            out = torch.empty((N, d), dtype=torch.int8, device=W.device)
        if aux is None:
            aux = torch.empty((N,), dtype=torch.float32, device=W.device)
        _need_cuda(out, "q", torch.int8)
        _need_cuda(aux, "scale", torch.float32)
        _need_shape(out, (N, d), "q")
    else:
        raise ValueError("mode must be 'lloydmax', 'int8' or 'int8_tensor'")
    _need_shape(aux, (N,), "rnorm" if mode == "lloydmax" else "scale")
    with _device_ctx(W, out, aux):
        _check(lib().quantize_weights(rpbh.handle, _ptr(W), _dtype_code(W), N, code, int(bits), _ptr(out),
                                      _ptr(aux), _stream(stream)), "quantize_weights")
    return out, aux


def qlinear(a_codes, s, bits_a, w_codes, rnorm, bits_w, K, out=None, stream=None):
    """y[m, n] = s_m r'_n sum_k C_w[q_nk] C_a[p_mk] as bfloat16 [M, N]."""
    import torch
    for t, n, dt in ((a_codes, "a_codes", torch.uint8), (s, "s", torch.float32),
                     (w_codes, "w_codes", torch.uint8), (rnorm, "rnorm", torch.bfloat16)):
        _need_cuda(t, n, dt)
    M, N = a_codes.shape[0], w_codes.shape[0]
    check_layer_shapes(M, N, int(K), int(bits_a), int(bits_w), a_codes.shape, s.shape, w_codes.shape,
                       rnorm.shape, None if out is None else out.shape)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    _need_cuda(out, "out", torch.bfloat16)
    with _device_ctx(a_codes, s, w_codes, rnorm, out):
        _check(lib().qlinear(_ptr(a_codes), _ptr(s), int(bits_a), _ptr(w_codes), _ptr(rnorm), int(bits_w), M, N,
                             int(K), _ptr(out), _stream(stream)), "qlinear")
    return out


def qlinear_int8_levels(a_codes, s, bits_a, w_codes, rnorm, bits_w, K, out=None, stream=None):
    """qlinear with each codebook's levels rounded onto a signed 8-bit grid and
    the sum taken exactly on the INT8 tensor cores:
    y[m, n] = s_m r'_n sum_k l_w[q_nk] l_a[p_mk] / (alpha_w alpha_a), bfloat16 [M, N]
    (see int8_levels).  K a multiple of 128, N of 8."""
    import torch
    for t, n, dt in ((a_codes, "a_codes", torch.uint8), (s, "s", torch.float32),
                     (w_codes, "w_codes", torch.uint8), (rnorm, "rnorm", torch.bfloat16)):
        _need_cuda(t, n, dt)
    M, N = a_codes.shape[0], w_codes.shape[0]
    check_layer_shapes(M, N, int(K), int(bits_a), int(bits_w), a_codes.shape, s.shape, w_codes.shape,
                       rnorm.shape, None if out is None else out.shape)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    _need_cuda(out, "out", torch.bfloat16)
    with _device_ctx(a_codes, s, w_codes, rnorm, out):
        _check(lib().qlinear_int8_levels(_ptr(a_codes), _ptr(s), int(bits_a), _ptr(w_codes), _ptr(rnorm),
                                         int(bits_w), M, N, int(K), _ptr(out), _stream(stream)), "qlinear_int8_levels")
    return out


def qlinear_fp8_levels(a_codes, s, bits_a, w_codes, rnorm, bits_w, K, out=None, stream=None):
    """qlinear with each codebook's levels rounded to FP8 E4M3 (times a power
    of two) and summed in fp32 on the FP8 tensor cores:
    y[m, n] = s_m r'_n sum_k e_w[q_nk] e_a[p_mk] / (beta_w beta_a), bfloat16 [M, N]
    (see fp8_levels).  K a multiple of 128, N of 8."""
    import torch
    for t, n, dt in ((a_codes, "a_codes", torch.uint8), (s, "s", torch.float32),
                     (w_codes, "w_codes", torch.uint8), (rnorm, "rnorm", torch.bfloat16)):
        _need_cuda(t, n, dt)
    M, N = a_codes.shape[0], w_codes.shape[0]
    check_layer_shapes(M, N, int(K), int(bits_a), int(bits_w), a_codes.shape, s.shape, w_codes.shape,
                       rnorm.shape, None if out is None else out.shape)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    _need_cuda(out, "out", torch.bfloat16)
    with _device_ctx(a_codes, s, w_codes, rnorm, out):
        _check(lib().qlinear_fp8_levels(_ptr(a_codes), _ptr(s), int(bits_a), _ptr(w_codes), _ptr(rnorm),
                                        int(bits_w), M, N, int(K), _ptr(out), _stream(stream)), "qlinear_fp8_levels")
    return out


def fp8_levels(d, bits):
    """(E4M3 bytes uint8[2^bits], beta) that qlinear_fp8_levels uses for
    (d, bits): bytes = E4M3(beta * c), beta = 2^(7 - floor(log2 max |c|))."""
    lv = np.empty(2 ** int(bits), dtype=np.uint8)
    beta = ctypes.c_double(0.0)
    _check(lib().rbq_fp8_levels(int(d), int(bits), lv.ctypes.data_as(_P), ctypes.byref(beta)), "rbq_fp8_levels")
    return lv, beta.value


def int8_levels(d, bits):
    """(levels int8[2^bits], alpha) that qlinear_int8_levels uses for (d, bits):
    levels = RNE(alpha * c), alpha = 127 / max |c|, c the Lloyd-Max levels."""
    lv = np.empty(2 ** int(bits), dtype=np.int8)
    alpha = ctypes.c_double(0.0)
    _check(lib().rbq_int8_levels(int(d), int(bits), lv.ctypes.data_as(_P), ctypes.byref(alpha)), "rbq_int8_levels")
    return lv, alpha.value


def qlinear_noalloc(a_codes, s, bits_a, w_codes, rnorm, bits_w, K, out, err=None, stream=None):
    """qlinear without any device allocation inside the library (its workspace
    is a fixed array in the library, N*K <= 2**24).  `out` (bfloat16 [M, N])
    and the optional error word `err` (int32 [1], OR-ed non-zero on a pipeline
    time-out) are the caller's.  Calls that overlap on the GPU race."""
    import torch
    for t, n, dt in ((a_codes, "a_codes", torch.uint8), (s, "s", torch.float32),
                     (w_codes, "w_codes", torch.uint8), (rnorm, "rnorm", torch.bfloat16),
                     (out, "out", torch.bfloat16)):
        _need_cuda(t, n, dt)
    if err is not None:
        _need_cuda(err, "err", torch.int32)
    M, N = a_codes.shape[0], w_codes.shape[0]
    check_layer_shapes(M, N, int(K), int(bits_a), int(bits_w), a_codes.shape, s.shape, w_codes.shape,
                       rnorm.shape, out.shape)
    if err is not None and err.numel() < 1:
        raise ValueError("err must hold one int32")
    with _device_ctx(a_codes, s, w_codes, rnorm, out, err):
        _check(lib().qlinear_noalloc(_ptr(a_codes), _ptr(s), int(bits_a), _ptr(w_codes), _ptr(rnorm), int(bits_w),
                                     M, N, int(K), _ptr(out), _ptr(err), _stream(stream)), "qlinear_noalloc")
    return out


def qlinear_int8(xrot, q, scale, out=None, stream=None):
    """y[m, n] = scale_n sum_k q_nk x'_mk as bfloat16 [M, N]."""
    import torch
    _need_cuda(xrot, "xrot", torch.bfloat16)
    _need_cuda(q, "q", torch.int8)
    _need_cuda(scale, "scale", torch.float32)
    M, K = xrot.shape
    N = q.shape[0]
    if q.shape[1] != K:
        raise ValueError("q and xrot disagree on K")
    _need_shape(scale, (N,), "scale")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xrot.device)
    _need_cuda(out, "out", torch.bfloat16)
    _need_shape(out, (M, N), "out")
    with _device_ctx(xrot, q, scale, out):
        _check(lib().qlinear_int8(_ptr(xrot), _ptr(q), _ptr(scale), M, N, K, _ptr(out), _stream(stream)),
               "qlinear_int8")
    return out


def quantize_weights_int8_asym(rpbh, W, q=None, scale=None, zero_point=None, stream=None):
    """Asymmetric per-channel INT8 of the rotated rows: (q uint8[N, d],
    scale float32[N], zero_point uint8[N]); w' ~ scale (q - z)."""
    import torch
    _need_cuda(W, "W")
    N, d = W.shape
    if d != rpbh.d:
        raise ValueError("W width does not match the RPBH handle")
    q = torch.empty((N, d), dtype=torch.uint8, device=W.device) if q is None else q
    scale = torch.empty((N,), dtype=torch.float32, device=W.device) if scale is None else scale
    zero_point = torch.empty((N,), dtype=torch.uint8, device=W.device) if zero_point is None else zero_point
    _need_cuda(q, "q", torch.uint8)
    _need_cuda(scale, "scale", torch.float32)
    _need_cuda(zero_point, "zero_point", torch.uint8)
    _need_shape(q, (N, d), "q")
    _need_shape(scale, (N,), "scale")
    _need_shape(zero_point, (N,), "zero_point")
    with _device_ctx(W, q, scale, zero_point):
        _check(lib().quantize_weights_int8_asym(rpbh.handle, _ptr(W), _dtype_code(W), N, _ptr(q), _ptr(scale),
                                                _ptr(zero_point), _stream(stream)), "quantize_weights_int8_asym")
    return q, scale, zero_point


def qlinear_int8_asym(xrot, q, scale, zero_point, out=None, stream=None):
    """Y = bf16(scale[n] * sum_k (q[n,k] - z[n]) * x'[m,k]) on asymmetric INT8 weights."""
    import torch
    _need_cuda(xrot, "xrot", torch.bfloat16)
    _need_cuda(q, "q", torch.uint8)
    _need_cuda(scale, "scale", torch.float32)
    _need_cuda(zero_point, "zero_point", torch.uint8)
    M, K = xrot.shape
    N = q.shape[0]
    if q.shape[1] != K:
        raise ValueError("q and xrot disagree on K")
    _need_shape(scale, (N,), "scale")
    _need_shape(zero_point, (N,), "zero_point")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xrot.device)
    _need_cuda(out, "out", torch.bfloat16)
    _need_shape(out, (M, N), "out")
    with _device_ctx(xrot, q, scale, zero_point, out):
        _check(lib().qlinear_int8_asym(_ptr(xrot), _ptr(q), _ptr(scale), _ptr(zero_point), M, N, K, _ptr(out),
                                       _stream(stream)), "qlinear_int8_asym")
    return out


def rows_in_next_order(next_rpbh, t, out=None, stream=None):
    """The offline reordering for qlinear_int8_rotate_next: out[k] = t[pi(k)]
    for the rows of a device tensor t [d, ...] (d = next_rpbh.d), pi the
    permutation of the next layer's rotation (rpbh_gather_rows)."""
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise ValueError("t must be a contiguous CUDA tensor")
    if t.shape[0] != next_rpbh.d:
        raise ValueError(f"t must have {next_rpbh.d} rows (the next layer's width)")
    out = torch.empty_like(t) if out is None else out
    if out.shape != t.shape or out.dtype != t.dtype or not out.is_contiguous() or out.data_ptr() == t.data_ptr():
        raise ValueError("out must be a different contiguous tensor of t's shape and dtype")
    row_bytes = t[0].numel() * t.element_size() if t.dim() > 1 else t.element_size()
    with _device_ctx(t, out):
        _check(lib().rpbh_gather_rows(next_rpbh.handle, _ptr(t), int(row_bytes), _ptr(out), _stream(stream)),
               "rpbh_gather_rows")
    return out


def qlinear_int8_rotate_next(xrot, q_next_order, scale_next_order, next_rpbh, activation="gelu", out=None,
                             stream=None):
    """The W8A16 layer fused with the next layer's input rotation:
    out = bf16(Pi_next act(scale_n sum_k q_nk x'_mk)) as bfloat16 [M, next.d];
    q and scale in the next layer's permutation order (rows_in_next_order)."""
    import torch
    _need_cuda(xrot, "xrot", torch.bfloat16)
    _need_cuda(q_next_order, "q_next_order", torch.int8)
    _need_cuda(scale_next_order, "scale_next_order", torch.float32)
    M, K = xrot.shape
    N = next_rpbh.d
    _need_shape(q_next_order, (N, K), "q_next_order")
    _need_shape(scale_next_order, (N,), "scale_next_order")
    if activation not in _ACTS:
        raise ValueError("activation must be None, 'none' or 'gelu'")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xrot.device)
    _need_cuda(out, "out", torch.bfloat16)
    _need_shape(out, (M, N), "out")
    with _device_ctx(xrot, q_next_order, scale_next_order, out):
        _check(lib().qlinear_int8_rotate_next(_ptr(xrot), _ptr(q_next_order), _ptr(scale_next_order), M, K,
                                              next_rpbh.handle, _ACTS[activation], _ptr(out), _stream(stream)),
               "qlinear_int8_rotate_next")
    return out


def qlinear_rotate_next(a_codes, s, bits_a, w_codes_next_order, rnorm_next_order, bits_w, K, next_rpbh,
                        activation="gelu", out=None, stream=None):
    """The code layer of qlinear fused with the next layer's input rotation:
    out = bf16(Pi_next act(s_m r'_n sum_k C_w[q_nk] C_a[p_mk])) as bfloat16
    [M, next.d]; the weight codes and r' in the next layer's permutation order
    (rows_in_next_order).  quantize_rotated then gives that layer's codes."""
    import torch
    for t, n, dt in ((a_codes, "a_codes", torch.uint8), (s, "s", torch.float32),
                     (w_codes_next_order, "w_codes_next_order", torch.uint8),
                     (rnorm_next_order, "rnorm_next_order", torch.bfloat16)):
        _need_cuda(t, n, dt)
    M = a_codes.shape[0]
    N = next_rpbh.d
    _need_shape(a_codes, (M, K * bits_a // 8), "a_codes")
    _need_shape(s, (M,), "s")
    _need_shape(w_codes_next_order, (N, K * bits_w // 8), "w_codes_next_order")
    _need_shape(rnorm_next_order, (N,), "rnorm_next_order")
    if activation not in _ACTS:
        raise ValueError("activation must be None, 'none' or 'gelu'")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    _need_cuda(out, "out", torch.bfloat16)
    _need_shape(out, (M, N), "out")
    with _device_ctx(a_codes, s, w_codes_next_order, rnorm_next_order, out):
        _check(lib().qlinear_rotate_next(_ptr(a_codes), _ptr(s), int(bits_a), _ptr(w_codes_next_order),
                                         _ptr(rnorm_next_order), int(bits_w), M, int(K), next_rpbh.handle,
                                         _ACTS[activation], _ptr(out), _stream(stream)),
               "qlinear_rotate_next")
    return out


def quantize_rotated(xrot, bits, codes=None, norms=None, stream=None):
    """OrbitQuant §2.2 steps 2-4 on already rotated BF16 rows [T, d]: packed
    codes uint8[T, d*bits/8] and norms float32[T]."""
    import torch
    _need_cuda(xrot, "xrot", torch.bfloat16)
    T, d = xrot.shape
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=xrot.device)
    if norms is None:
        norms = torch.empty((T,), dtype=torch.float32, device=xrot.device)
    _need_cuda(codes, "codes", torch.uint8)
    _need_cuda(norms, "norms", torch.float32)
    _need_shape(codes, (T, d * bits // 8), "codes")
    _need_shape(norms, (T,), "norms")
    with _device_ctx(xrot, codes, norms):
        _check(lib().quantize_rotated(_ptr(xrot), _dtype_code(xrot), T, d, int(bits), _ptr(codes), _ptr(norms),
                                      _stream(stream)), "quantize_rotated")
    return codes, norms


def _host_bytes(t):
    """A contiguous host numpy copy of a torch tensor or array (bytes only)."""
    if hasattr(t, "detach"):
        t = t.detach().contiguous().cpu()
        import torch
        return np.ascontiguousarray(t.view(torch.uint8).numpy()) if t.dtype != torch.uint8 else \
            np.ascontiguousarray(t.numpy())
    return np.ascontiguousarray(t)


def save_layer(path, rpbh, kind, codes, aux, zero_point=None, bits=None):
    """Write one quantised linear layer (weights, quantisation parameters and
    the transform info) to `path`: kind 'lloydmax' (codes + BF16 r', give
    bits), 'int8', 'int8_tensor' or 'int8_asym' (+ zero_point)."""
    d, h, seed, flags = rpbh.describe()
    mode = _LAYER_KINDS[kind]
    rows = codes.shape[0]
    info = LayerInfo(d, h, seed, flags, mode, int(bits) if mode == RBQ_LAYER_LLOYDMAX else 8, rows)
    c, a = _host_bytes(codes), _host_bytes(aux)
    z = _host_bytes(zero_point) if zero_point is not None else None
    nc, na, nz = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(lib().rbq_layer_sizes(ctypes.byref(info), ctypes.byref(nc), ctypes.byref(na), ctypes.byref(nz)),
           "rbq_layer_sizes")
    if c.nbytes != nc.value or a.nbytes != na.value or (nz.value and (z is None or z.nbytes != nz.value)):
        raise ValueError("array sizes do not match the layer description")
    _check(lib().rbq_layer_write(os.fsencode(path), ctypes.byref(info), c.ctypes.data_as(_P), a.ctypes.data_as(_P),
                                 z.ctypes.data_as(_P) if z is not None else None), "rbq_layer_write")


def load_layer(path, device=None):
    """Read a layer file: dict(kind, bits, rpbh (rebuilt from the transform
    info), codes, aux, zero_point) -- numpy arrays, or torch tensors on
    `device` when given."""
    info = LayerInfo()
    _check(lib().rbq_layer_read(os.fsencode(path), ctypes.byref(info), None, 0, None, 0, None, 0), "rbq_layer_read")
    nc, na, nz = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(lib().rbq_layer_sizes(ctypes.byref(info), ctypes.byref(nc), ctypes.byref(na), ctypes.byref(nz)),
           "rbq_layer_sizes")
    c = np.empty(nc.value, dtype=np.uint8)
    a = np.empty(na.value, dtype=np.uint8)
    z = np.empty(nz.value, dtype=np.uint8) if nz.value else None
    _check(lib().rbq_layer_read(os.fsencode(path), ctypes.byref(info), c.ctypes.data_as(_P), c.nbytes,
                                a.ctypes.data_as(_P), a.nbytes, z.ctypes.data_as(_P) if z is not None else None,
                                z.nbytes if z is not None else 0), "rbq_layer_read")
    kind = {v: k for k, v in _LAYER_KINDS.items()}[info.mode]
    rows, d = info.rows, info.d
    if kind == "lloydmax":
        codes, aux = c.reshape(rows, d * info.bits // 8), a.view(np.uint16)
    else:
        codes = c.reshape(rows, d).view(np.int8 if kind != "int8_asym" else np.uint8)
        aux = a.view(np.float32)
    out = {"kind": kind, "bits": info.bits, "d": d, "rows": rows,
           "rpbh": RPBH.from_description(d, info.seed, info.rpbh_flags, h=info.h),
           "codes": codes, "aux": aux, "zero_point": z}
    if device is not None:
        import torch
        out["codes"] = torch.from_numpy(np.ascontiguousarray(codes)).to(device)
        aux_t = torch.from_numpy(np.ascontiguousarray(aux))
        out["aux"] = (aux_t.view(torch.bfloat16) if kind == "lloydmax" else aux_t).to(device)
        out["zero_point"] = torch.from_numpy(z).to(device) if z is not None else None
    return out


def code_grid(d, bits, variant=0):
    """A code-search table of the kernels: (thr float32[n], base int32[n], cells, scale).
    variant 0: clamped grid just wider than the boundaries; 1: grid over [-1, 1]."""
    cells, scale = ctypes.c_int(), ctypes.c_float()
    _check(lib().rbq_code_grid(int(d), int(bits), int(variant), None, None, ctypes.byref(cells),
                               ctypes.byref(scale)), "rbq_code_grid")
    thr = np.empty(cells.value + 1, dtype=np.float32)
    base = np.empty(cells.value + 1, dtype=np.int32)
    _check(lib().rbq_code_grid(int(d), int(bits), int(variant), thr.ctypes.data_as(_P), base.ctypes.data_as(_P),
                               None, None), "rbq_code_grid")
    return thr, base, cells.value, np.float32(scale.value)


def device_error(stream=None):
    """Synchronise and read/clear the library's device error word (0 = clean)."""
    return lib().rbq_device_error(_stream(stream))


def selftest_wait_limit(out, stream=None):
    """Launch the kernel whose barriers nothing arrives at, so that every
    bounded-wait form gives up (about a second); ``out`` is a CUDA int32[1]
    that receives the bit mask of the waits that gave up (15 when all did)."""
    import torch
    if not (out.is_cuda and out.dtype == torch.int32 and out.numel() >= 1):
        raise ValueError("out must be a CUDA int32 tensor with at least one element")
    _check(lib().rbq_selftest_wait_limit(_P(out.data_ptr()), _stream(stream)), "rbq_selftest_wait_limit")
