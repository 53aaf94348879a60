"""Python binding of libhyena_b200.so -- the Hyena implicit long-convolution
hot path on B200 (sm_100a).

This module only marshals arguments: every step of the path runs in the CUDA
kernels behind the C ABI declared in ``include/hyena.h``.  PyTorch supplies
device memory and the current stream.  If the shared library is missing the
import of this package still works, but every call raises
``HyenaLibraryMissing`` -- there is no CPU fallback.

Functions mirror the C entry points (same names, same semantics):
``hyena_filter_gen``, ``hyena_filter_spectrum``, ``hyena_fftconv``,
``hyena_operator``, ``hyena_nd_conv``, ``spectral_gate``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

__all__ = [
    "HyenaError", "HyenaLibraryMissing", "LIB_PATH", "lib", "spectrum_bins",
    "hyena_filter_gen", "hyena_filter_spectrum", "filter_spectrum_workspace",
    "hyena_fftconv", "hyena_operator", "operator_workspace", "hyena_operator_noalloc", "hyena_nd_conv",
    "nd_conv_workspace", "spectral_gate", "operator_host_workspace", "hyena_operator_host",
    "spectral_gate_host_workspace", "spectral_gate_host", "nd_conv_host_workspace", "hyena_nd_conv_host",
    "projection_workspace", "hyena_projection", "operator_backward_workspace", "hyena_operator_backward",
    "spectral_gate_decode", "device_faults", "selftest_bounded_wait", "hyena_register_film",
    "STATUS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhyena_b200.so")

STATUS = {0: "HY_OK", 1: "HY_ERR_INVALID_ARG", 2: "HY_ERR_UNSUPPORTED", 3: "HY_ERR_WORKSPACE",
          4: "HY_ERR_CUDA", 5: "HY_ERR_TIMEOUT"}
HY_F32, HY_BF16 = 0, 1
HY_ACT_SILU, HY_ACT_IDENTITY, HY_ACT_SINE = 0, 1, 2
HY_WIN_EXP, HY_WIN_GAUSS = 0, 1
HY_FAULT_STREAM_INPUT, HY_FAULT_STREAM_GATE, HY_FAULT_PROJECTION, HY_FAULT_TC_CONV = 0x1, 0x2, 0x4, 0x8
HY_FAULT_FILTER_MMA = 0x10
HY_FAULT_MULTIPASS = 0x20
HY_FAULT_SELFTEST = 0x80000000


class HyenaLibraryMissing(RuntimeError):
    pass


class HyenaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        self.status_name = STATUS.get(status, str(status))
        super().__init__("%s: %s" % (self.status_name, message))


class FilterDesc(ctypes.Structure):
    _fields_ = [
        ("ndim", ctypes.c_int), ("L", ctypes.c_int), ("grid", ctypes.c_int),
        ("circular", ctypes.c_int), ("n_freq", ctypes.c_int), ("include_t", ctypes.c_int),
        ("n_layers", ctypes.c_int), ("widths", ctypes.POINTER(ctypes.c_int)),
        ("W", ctypes.POINTER(ctypes.c_void_p)), ("b", ctypes.POINTER(ctypes.c_void_p)),
        ("act", ctypes.c_int), ("film_gamma", ctypes.c_void_p), ("film_beta", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("n_sets", ctypes.c_int),
        ("omega", ctypes.c_void_p), ("window", ctypes.c_int),
    ]


_lib = None
_VP = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


def lib():
    """The loaded shared library (raises HyenaLibraryMissing if not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise HyenaLibraryMissing(
            "libhyena_b200.so is not built (run implicit_long_convolution_b200/build.py); "
            "there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "hyena_abi_version": (_I, []),
        "hyena_status_string": (ctypes.c_char_p, [_I]),
        "hyena_last_error": (ctypes.c_char_p, []),
        "hyena_init": (_I, []),
        "hyena_spectrum_bins": (_I64, [_I64]),
        "hyena_filter_gen": (_I, [ctypes.POINTER(FilterDesc), _VP, _VP]),
        "hyena_filter_spectrum_workspace": (_SZ, [_I64, _I, ctypes.POINTER(_I), _I]),
        "hyena_filter_spectrum": (_I, [_I64, _I, ctypes.POINTER(_I), _I, _VP, _VP, _VP, _SZ, _VP]),
        "hyena_fftconv": (_I, [_I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
        "hyena_operator_workspace": (_SZ, [_I, _I, _I, _I, _I]),
        "hyena_operator": (_I, [_I, _I, _I, _I, _I, _VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP),
                                ctypes.POINTER(_VP), _VP, _VP, _SZ, _VP]),
        "hyena_operator_noalloc": (_I, [_I, _I, _I, _I, _I, _VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP),
                                        ctypes.POINTER(_VP), _VP, _VP]),
        "hyena_nd_conv_workspace": (_SZ, [_I, ctypes.POINTER(_I), _I, _I, _I]),
        "hyena_nd_conv": (_I, [_I, ctypes.POINTER(_I), _I, _I, _I, _VP, _VP, _I64, _VP, _VP, _VP,
                               _VP, _SZ, _VP]),
        "spectral_gate": (_I, [_I, _I, _I, _I, _I, _VP, _VP, _I64, _VP, _VP, _VP]),
        "hyena_operator_host_workspace": (_SZ, [_I, _I, _I, _I, _I]),
        "hyena_operator_host": (_I, [_I, _I, _I, _I, _I, _VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP),
                                     ctypes.POINTER(_VP), _VP, _VP, _SZ, _VP]),
        "hyena_operator_backward_workspace": (_SZ, [_I, _I, _I, _I, _I]),
        "hyena_operator_backward": (_I, [_I, _I, _I, _I, _I, _VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP),
                                         ctypes.POINTER(_VP), _VP, _VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP),
                                         ctypes.POINTER(_VP), _VP, _SZ, _VP]),
        "spectral_gate_decode": (_I, [_I, _I, _I, _I, _I, _I64, _VP, _VP, _I64, _VP, _VP, _VP, _VP]),
        "hyena_projection_workspace": (_SZ, []),
        "hyena_projection": (_I, [_I, _I, _I, _I, _I, _I, _VP, _VP, _VP, ctypes.POINTER(_VP), _VP, _SZ, _VP]),
        "hyena_nd_conv_host_workspace": (_SZ, [_I, ctypes.POINTER(_I), _I, _I, _I]),
        "hyena_nd_conv_host": (_I, [_I, ctypes.POINTER(_I), _I, _I, _I, _VP, _VP, _I64, _VP, _VP, _VP,
                                    _VP, _SZ, _VP]),
        "spectral_gate_host_workspace": (_SZ, [_I, _I, _I, _I, _I]),
        "spectral_gate_host": (_I, [_I, _I, _I, _I, _I, _VP, _VP, _I64, _VP, _VP, _VP, _SZ, _VP]),
        "hyena_device_faults": (_I, [ctypes.POINTER(ctypes.c_uint32), _I, _VP]),
        "hyena_register_film": (_I, [_I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
        "hyena_selftest_bounded_wait": (_I, [ctypes.c_uint32, _VP]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        msg = lib().hyena_last_error()
        raise HyenaError(status, msg.decode() if msg else "")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _dt(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return HY_F32
    if t.dtype == torch.bfloat16:
        return HY_BF16
    raise HyenaError(1, "dtype %s not supported (float32 or bfloat16)" % t.dtype)


def _ints(seq):
    return (_I * len(seq))(*seq)


def _ptrs(seq):
    return (_VP * len(seq))(*[_ptr(t) for t in seq])


def spectrum_bins(L: int) -> int:
    """Bins of one causal filter spectrum row: M + 1, M = max(16, next pow2 >= L)."""
    return int(lib().hyena_spectrum_bins(L))


def hyena_filter_gen(h_out, *, ndim: int, Ws: Sequence, bs: Sequence, alpha, n_freq: int,
                     L: int = 0, include_t: bool = True, grid: int = 0, circular: bool = False,
                     film_gamma=None, film_beta=None, n_sets: int = 1, act: int = HY_ACT_SILU,
                     omega=None, window: int = HY_WIN_EXP, stream=None):
    """Fill h_out (fp32, device) with implicit filters; see hyena.h."""
    widths = [int(Ws[0].shape[1])] + [int(w.shape[0]) for w in Ws]
    keep = (_ints(widths), _ptrs(Ws), _ptrs(bs))
    d = FilterDesc(ndim, L, grid, int(circular), n_freq, int(include_t), len(Ws),
                   keep[0], keep[1], keep[2], act, _ptr(film_gamma), _ptr(film_beta),
                   _ptr(alpha), n_sets, _ptr(omega), window)
    _check(lib().hyena_filter_gen(ctypes.byref(d), _ptr(h_out), _stream(stream)))
    return h_out


def filter_spectrum_workspace(rows: int, ndim: int, dims: Sequence[int], circular: bool = False) -> int:
    return int(lib().hyena_filter_spectrum_workspace(rows, ndim, _ints(dims), int(circular)))


def hyena_filter_spectrum(h, H_out, *, rows: int, ndim: int, dims: Sequence[int],
                          circular: bool = False, ws=None, stream=None):
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_filter_spectrum(rows, ndim, _ints(dims), int(circular), _ptr(h), _ptr(H_out),
                                       _ptr(ws), wsb, _stream(stream)))
    return H_out


def hyena_fftconv(u, H, y, *, Dskip=None, gate=None, ws=None, stream=None):
    B, D, L = u.shape
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_fftconv(B, D, L, _dt(u), _ptr(u), _ptr(H), _ptr(Dskip), _ptr(gate), _ptr(y),
                               _ptr(ws), wsb, _stream(stream)))
    return y


def operator_workspace(order: int, B: int, D: int, L: int, dtype_code: int = HY_F32) -> int:
    return int(lib().hyena_operator_workspace(order, B, D, L, dtype_code))


def hyena_operator(v, xs: Sequence, Hs: Sequence, y, *, Dskips: Optional[Sequence] = None,
                   ws=None, stream=None):
    B, D, L = v.shape
    order = len(xs) + 1
    dsk = _ptrs(Dskips) if Dskips is not None else None
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_operator(order, B, D, L, _dt(v), _ptr(v), _ptrs(xs), _ptrs(Hs), dsk, _ptr(y),
                                _ptr(ws), wsb, _stream(stream)))
    return y


def hyena_operator_noalloc(v, xs: Sequence, Hs: Sequence, y, *, Dskips: Optional[Sequence] = None,
                           stream=None):
    """hyena_operator for callers that cannot allocate device memory: long
    sequences use the library's static device scratch (see hyena.h)."""
    B, D, L = v.shape
    order = len(xs) + 1
    dsk = _ptrs(Dskips) if Dskips is not None else None
    _check(lib().hyena_operator_noalloc(order, B, D, L, _dt(v), _ptr(v), _ptrs(xs), _ptrs(Hs), dsk,
                                        _ptr(y), _stream(stream)))
    return y


def nd_conv_workspace(dims: Sequence[int], B: int, D: int, circular: bool = False) -> int:
    return int(lib().hyena_nd_conv_workspace(3, _ints(dims), B, D, int(circular)))


def hyena_nd_conv(u, H, y, *, H_batch_stride: int = 0, circular: bool = False, Dskip=None,
                  gate=None, ws=None, stream=None):
    B, D = u.shape[:2]
    dims = list(u.shape[2:])
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_nd_conv(len(dims), _ints(dims), B, D, int(circular), _ptr(u), _ptr(H),
                               H_batch_stride, _ptr(Dskip), _ptr(gate), _ptr(y), _ptr(ws), wsb,
                               _stream(stream)))
    return y


def spectral_gate(x, g, y, *, x2=None, g_batch_stride: int = 0, stream=None):
    B, Hh, Dh, L = x.shape
    _check(lib().spectral_gate(B, Hh, Dh, L, _dt(x), _ptr(x), _ptr(g), g_batch_stride, _ptr(x2),
                               _ptr(y), _stream(stream)))
    return y


def operator_host_workspace(order: int, B: int, D: int, L: int, dtype_code: int) -> int:
    return int(lib().hyena_operator_host_workspace(order, B, D, L, dtype_code))


def hyena_operator_host(v, xs: Sequence, Hs: Sequence, y, *, Dskips: Optional[Sequence] = None,
                        ws=None, stream=None):
    """hyena_operator with v, xs and y in (page-locked) host memory; Hs,
    Dskips and ws on the device.  Copies and compute overlap chunk by chunk;
    y is valid once the stream is synchronised (see hyena.h)."""
    B, D, L = v.shape
    order = len(xs) + 1
    dsk = _ptrs(Dskips) if Dskips is not None else None
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_operator_host(order, B, D, L, _dt(v), _ptr(v), _ptrs(xs), _ptrs(Hs), dsk, _ptr(y),
                                     _ptr(ws), wsb, _stream(stream)))
    return y


def spectral_gate_host_workspace(B: int, H: int, Dh: int, L: int, dtype_code: int) -> int:
    return int(lib().spectral_gate_host_workspace(B, H, Dh, L, dtype_code))


def spectral_gate_host(x, g, y, *, x2=None, g_batch_stride: int = 0, ws=None, stream=None):
    """spectral_gate with x, x2 and y in (page-locked) host memory; g and ws
    on the device (see hyena.h)."""
    B, Hh, Dh, L = x.shape
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().spectral_gate_host(B, Hh, Dh, L, _dt(x), _ptr(x), _ptr(g), g_batch_stride, _ptr(x2),
                                    _ptr(y), _ptr(ws), wsb, _stream(stream)))
    return y


def nd_conv_host_workspace(dims: Sequence[int], B: int, D: int, circular: bool = False) -> int:
    return int(lib().hyena_nd_conv_host_workspace(3, _ints(dims), B, D, int(circular)))


def hyena_nd_conv_host(u, H, y, *, H_batch_stride: int = 0, circular: bool = False, Dskip=None,
                       gate=None, ws=None, stream=None):
    """hyena_nd_conv with u, gate and y in (page-locked) host memory; H,
    Dskip and ws on the device (see hyena.h)."""
    B, D = u.shape[:2]
    dims = list(u.shape[2:])
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_nd_conv_host(len(dims), _ints(dims), B, D, int(circular), _ptr(u), _ptr(H),
                                    H_batch_stride, _ptr(Dskip), _ptr(gate), _ptr(y), _ptr(ws), wsb,
                                    _stream(stream)))
    return y


def hyena_register_film(reg, W_film, gamma, beta, *, query=None, scores=None, b_film=None, stream=None):
    """z(x) = softmax-weighted mean of the register activations reg (B, R, C)
    and the FiLM parameters (gamma, beta) = W_film z + b_film, each (B, H)
    (device tensors; see hyena.h)."""
    B, R, C = reg.shape
    H = gamma.shape[1]
    _check(lib().hyena_register_film(B, R, C, H, _ptr(reg), _ptr(query), _ptr(scores), _ptr(W_film),
                                     _ptr(b_film), _ptr(gamma), _ptr(beta), _stream(stream)))
    return gamma, beta


def projection_workspace() -> int:
    return int(lib().hyena_projection_workspace())


def hyena_projection(x, W, outs: Sequence, *, bias=None, ws=None, stream=None):
    """out_k[b, d, l] = bias[kD + d] + sum_c W[kD + d, c] x[b, l, c] for the
    n_out = len(outs) projections (device tensors; see hyena.h)."""
    B, L, C = x.shape
    n_out = len(outs)
    D = outs[0].shape[1]
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_projection(B, L, C, D, n_out, _dt(x), _ptr(x), _ptr(W), _ptr(bias), _ptrs(outs),
                                  _ptr(ws), wsb, _stream(stream)))
    return outs


def operator_backward_workspace(order: int, B: int, D: int, L: int, dtype_code: int) -> int:
    return int(lib().hyena_operator_backward_workspace(order, B, D, L, dtype_code))


def hyena_operator_backward(v, xs: Sequence, Hs: Sequence, dy, dv, dxs: Sequence, *,
                            Dskips: Optional[Sequence] = None, dhs: Optional[Sequence] = None,
                            dDs: Optional[Sequence] = None, ws=None, stream=None):
    """Gradients of the operator (see hyena.h): dv, dxs[k] (like v), dhs[k]
    (fp32 (D, L)) and dDs[k] (fp32 (D,)); dhs / dDs may be None."""
    B, D, L = v.shape
    order = len(xs) + 1
    wsb = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().hyena_operator_backward(
        order, B, D, L, _dt(v), _ptr(v), _ptrs(xs), _ptrs(Hs), _ptrs(Dskips) if Dskips is not None else None,
        _ptr(dy), _ptr(dv), _ptrs(dxs), _ptrs(dhs) if dhs is not None else None,
        _ptrs(dDs) if dDs is not None else None, _ptr(ws), wsb, _stream(stream)))
    return dv


def spectral_gate_decode(x, g, cache, y, *, pos: int, x2=None, g_batch_stride: int = 0, stream=None):
    """One streaming step at position pos: x, x2, y are (B, H, Dh) device
    tensors (the new token's values), cache the (B, H, Dh, n/2+1) complex64
    prefix spectrum, updated in place (see hyena.h)."""
    B, Hh, Dh = x.shape
    n = 2 * (cache.shape[-1] - 1)
    _check(lib().spectral_gate_decode(B, Hh, Dh, n, _dt(x), pos, _ptr(x), _ptr(g), g_batch_stride, _ptr(x2),
                                      _ptr(cache), _ptr(y), _stream(stream)))
    return y


def device_faults(*, clear: bool = True, stream=None) -> int:
    """The current device's fault word (HY_FAULT_* bits) once the work queued
    on `stream` has finished; 0 when no bounded device wait gave up.  Unlike
    the other calls this does not raise on HY_ERR_TIMEOUT: it returns the
    bits (and resets them when `clear`)."""
    v = ctypes.c_uint32(0)
    st = lib().hyena_device_faults(ctypes.byref(v), int(clear), _stream(stream))
    if st not in (0, 5):
        _check(st)
    return int(v.value)


def selftest_bounded_wait(limit_us: int = 2000, *, stream=None):
    """Launch the bounded-wait self-test: a wait that can never be satisfied
    runs out after limit_us and records HY_FAULT_SELFTEST."""
    _check(lib().hyena_selftest_bounded_wait(limit_us, _stream(stream)))
