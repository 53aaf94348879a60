"""The C-ABI library loads, exports every function include/hyena.h declares,
and rejects bad arguments on the host with the documented status -- all
without a GPU (validation happens before any CUDA call)."""
import ctypes
import os
import re

import pytest

import implicit_long_convolution_b200 as hy

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hyena.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(hy.LIB_PATH):
        pytest.fail("libhyena_b200.so is not built; run __graft_entry__.build()")
    return hy.lib()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "hyena_operator" in names and "spectral_gate" in names and "hyena_filter_gen" in names
    for n in names:
        assert hasattr(lib, n), "missing export %s" % n


def test_version_and_strings(lib):
    assert lib.hyena_abi_version() == 3
    assert lib.hyena_status_string(3) == b"HY_ERR_WORKSPACE"
    assert lib.hyena_spectrum_bins(8192) == 8193
    assert lib.hyena_spectrum_bins(1000) == 1025
    assert lib.hyena_spectrum_bins(1) == 17
    assert lib.hyena_spectrum_bins(0) == 0


def test_header_constants_match_binding():
    """Every enum value and fault bit the header defines that the binding
    mirrors has the same value there (no GPU, no library call)."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    consts = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(HY_[A-Z0-9_]+)\s*=\s*(\d+)", src)}
    consts.update({m.group(1): int(m.group(2), 16)
                   for m in re.finditer(r"#define\s+(HY_FAULT_[A-Z_]+)\s+0x([0-9a-fA-F]+)u", src)})
    mirrored = [k for k in consts if hasattr(hy, k)]
    assert len(mirrored) >= 10, mirrored
    for k in mirrored:
        assert getattr(hy, k) == consts[k], k
    for code, name in hy.STATUS.items():
        assert consts[name] == code, name


def test_fault_api_validation(lib):
    # host-side checks only: a null output and an out-of-range limit are
    # rejected before the device is touched
    assert _err(lib, lib.hyena_device_faults(None, 1, None), "null output") == 1
    assert _err(lib, lib.hyena_selftest_bounded_wait(0, None), "limit") == 1
    assert _err(lib, lib.hyena_selftest_bounded_wait(2000000, None), "limit") == 1
    assert lib.hyena_status_string(5) == b"HY_ERR_TIMEOUT"


def _err(lib, status, substring):
    msg = lib.hyena_last_error().decode()
    assert status != 0 and substring in msg, (status, msg)
    return status


FAKE = 0x10000  # a non-null, aligned pointer value; never dereferenced: calls fail validation first


def test_operator_validation(lib):
    X = (ctypes.c_void_p * 1)(FAKE)
    H = (ctypes.c_void_p * 1)(FAKE)
    # order out of range
    assert _err(lib, lib.hyena_operator(1, 1, 1, 64, 0, FAKE, X, H, None, FAKE * 2, None, 0, None), "order") == 2
    # null x array
    assert _err(lib, lib.hyena_operator(2, 1, 1, 64, 0, FAKE, None, H, None, FAKE * 2, None, 0, None), "null") == 1
    # bad sizes
    assert lib.hyena_operator(2, 0, 1, 64, 0, FAKE, X, H, None, FAKE * 2, None, 0, None) == 1
    assert lib.hyena_operator(2, 1, 1, 0, 0, FAKE, X, H, None, FAKE * 2, None, 0, None) == 1
    # unknown dtype
    assert lib.hyena_operator(2, 1, 1, 64, 7, FAKE, X, H, None, FAKE * 2, None, 0, None) == 1
    # output aliases input
    assert _err(lib, lib.hyena_operator(2, 1, 4, 64, 0, FAKE, X, H, None, FAKE + 64, None, 0, None), "alias") == 1
    # misaligned signal
    assert lib.hyena_operator(2, 1, 1, 64, 0, FAKE + 4, X, H, None, FAKE * 4, None, 0, None) == 1
    # long sequence without workspace
    big = 1 << 20
    need = lib.hyena_operator_workspace(3, 1, 2, big, 0)
    assert need > 0
    X2 = (ctypes.c_void_p * 2)(FAKE * 64, FAKE * 128)
    H2 = (ctypes.c_void_p * 2)(FAKE, FAKE)
    st = lib.hyena_operator(3, 1, 2, big, 0, FAKE * 16, X2, H2, None, FAKE * 256, None, 0, None)
    assert _err(lib, st, "workspace") == 3
    assert lib.hyena_operator_workspace(2, 1, 1, 8192, 1) == 0


def test_fftconv_and_gate_validation(lib):
    assert lib.hyena_fftconv(1, 1, 64, 0, None, FAKE, None, None, FAKE, None, 0, None) == 1
    assert lib.hyena_fftconv(1, 1, 64, 0, FAKE, None, None, None, FAKE * 2, None, 0, None) == 1
    # spectral gate: L must be a power of two in [32, 32768]
    assert lib.spectral_gate(1, 1, 1, 100, 1, FAKE, FAKE, 0, None, FAKE * 2, None) == 2
    assert lib.spectral_gate(1, 1, 1, 65536, 1, FAKE, FAKE, 0, None, FAKE * 2, None) == 2
    assert lib.spectral_gate(1, 1, 1, 64, 1, FAKE, None, 0, None, FAKE * 2, None) == 1
    assert lib.spectral_gate(1, 1, 1, 64, 1, FAKE, FAKE, -1, None, FAKE * 2, None) == 1
    assert _err(lib, lib.spectral_gate(1, 2, 2, 64, 1, FAKE, FAKE, 0, None, FAKE + 64, None), "alias") == 1


def test_filter_and_nd_validation(lib):
    dims = (ctypes.c_int * 3)(64, 64, 64)
    assert lib.hyena_nd_conv(2, dims, 1, 1, 0, FAKE, FAKE, 0, None, None, FAKE * 2, None, 0, None) == 2
    bad = (ctypes.c_int * 3)(64, 48, 64)
    assert lib.hyena_nd_conv(3, bad, 1, 1, 0, FAKE, FAKE, 0, None, None, FAKE * 2, None, 0, None) == 2
    assert lib.hyena_nd_conv(3, dims, 1, 1, 0, FAKE, FAKE, -5, None, None, FAKE * 2, None, 0, None) == 1
    one = (ctypes.c_int * 1)(64)
    assert lib.hyena_filter_spectrum(0, 1, one, 0, FAKE, FAKE * 2, None, 0, None) == 1
    assert lib.hyena_filter_spectrum(4, 2, one, 0, FAKE, FAKE * 2, None, 0, None) == 1
    assert lib.hyena_filter_spectrum(4, 1, (ctypes.c_int * 1)(100), 1, FAKE, FAKE * 2, None, 0, None) == 2
    assert lib.hyena_filter_gen(None, FAKE, None) == 1
    # widths[0] inconsistent with the encoding
    widths = (ctypes.c_int * 3)(16, 32, 16)
    W = (ctypes.c_void_p * 2)(FAKE, FAKE)
    d = hy.FilterDesc(1, 1024, 0, 0, 8, 1, 2, widths, W, W, 0, None, None, FAKE, 1)
    assert _err(lib, lib.hyena_filter_gen(ctypes.byref(d), FAKE * 2, None), "include_t + 2F") == 1
    d = hy.FilterDesc(3, 0, 48, 0, 4, 0, 2, (ctypes.c_int * 3)(24, 64, 8), W, W, 0, None, None, FAKE, 1)
    assert lib.hyena_filter_gen(ctypes.byref(d), FAKE * 2, None) == 2
    # unknown activation or window
    d = hy.FilterDesc(1, 1024, 0, 0, 8, 1, 2, (ctypes.c_int * 3)(17, 32, 16), W, W, 7, None, None, FAKE, 1)
    assert _err(lib, lib.hyena_filter_gen(ctypes.byref(d), FAKE * 2, None), "activation") == 1
    d = hy.FilterDesc(1, 1024, 0, 0, 8, 1, 2, (ctypes.c_int * 3)(17, 32, 16), W, W, 2, None, None, FAKE, 1, None, 5)
    assert _err(lib, lib.hyena_filter_gen(ctypes.byref(d), FAKE * 2, None), "window") == 1


def test_host_entry_validation_and_workspace(lib):
    X = (ctypes.c_void_p * 2)(FAKE, FAKE)
    H = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert _err(lib, lib.hyena_operator_host(1, 1, 1, 64, 0, FAKE, X, H, None, FAKE * 2, None, 0, None), "order") == 2
    assert _err(lib, lib.hyena_operator_host(2, 0, 1, 64, 0, FAKE, X, H, None, FAKE * 2, None, 0, None), "B, D, L") == 1
    assert _err(lib, lib.hyena_operator_host(2, 1, 1, 64, 0, None, X, H, None, FAKE * 2, None, 0, None), "v is null") == 1
    assert _err(lib, lib.hyena_operator_host(2, 1, 1, 64, 0, FAKE, None, H, None, FAKE * 2, None, 0, None), "null x") == 1
    assert _err(lib, lib.hyena_operator_host(2, 1, 1, 64, 0, FAKE, X, H, None, FAKE * 2, None, 0, None), "workspace") == 3
    assert _err(lib, lib.spectral_gate_host(0, 1, 1, 64, 0, FAKE, FAKE, 0, None, FAKE * 2, None, 0, None), "B, H") == 1
    assert _err(lib, lib.spectral_gate_host(1, 1, 1, 64, 0, FAKE, FAKE, -1, None, FAKE * 2, None, 0, None), "stride") == 1
    assert _err(lib, lib.spectral_gate_host(1, 1, 1, 64, 0, FAKE, FAKE, 0, None, FAKE * 2, None, 0, None), "workspace") == 3
    # ring of 3 slots x (inputs + output), chunks of about 16 MB per signal:
    # the order-2 bf16 operator B8 D768 L8192 moves one batch (12.6 MB) per chunk
    assert lib.hyena_operator_host_workspace(2, 8, 768, 8192, 1) == 3 * 3 * 768 * 8192 * 2
    # the spectral gate B4 H32 Dh64 L32768 bf16 moves 4 heads (16 MB) per chunk
    assert lib.spectral_gate_host_workspace(4, 32, 64, 32768, 1) == 3 * 3 * 4 * 64 * 32768 * 2
    # multi-pass: chunks of 8 rows of 2^20 plus the multi-pass workspace of 8 rows
    assert lib.hyena_operator_host_workspace(3, 1, 256, 1 << 20, 0) == \
        3 * 4 * 8 * (1 << 20) * 4 + lib.hyena_operator_workspace(3, 1, 8, 1 << 20, 0)
    assert lib.hyena_operator_host_workspace(1, 8, 768, 8192, 1) == 0
    dims = (ctypes.c_int * 3)(64, 64, 64)
    # 3-D: 16 slabs of 64^3 fp32 per chunk, plus the N-D workspace of 16 slabs
    assert lib.hyena_nd_conv_host_workspace(3, dims, 2, 128, 0) == \
        3 * 3 * 16 * 64 ** 3 * 4 + lib.hyena_nd_conv_workspace(3, dims, 1, 16, 0)
    assert _err(lib, lib.hyena_nd_conv_host(2, dims, 1, 1, 0, FAKE, FAKE, 0, None, None, FAKE * 2, None, 0, None),
                "ndim") == 2
    assert _err(lib, lib.hyena_nd_conv_host(3, dims, 1, 1, 0, FAKE, FAKE, -1, None, None, FAKE * 2, None, 0, None),
                "stride") == 1
    assert _err(lib, lib.hyena_nd_conv_host(3, dims, 1, 1, 0, FAKE, FAKE, 0, None, None, FAKE * 2, None, 0, None),
                "workspace") == 3


def test_chunk_pipeline_workspaces(lib):
    """The workspace queries of the chunked paths return one chunk buffer per
    chunk pipeline that can be busy: two when the rows (slabs) take more than
    one chunk, else one chunk of exactly the rows; the calls accept one chunk
    buffer as the minimum (checked on the host: a byte less is refused)."""
    MB = 1 << 20
    row = 8 << 20                                    # L = 2^20: M = 2^20 complex points of 8 bytes
    cr = (104 * MB) // row                           # 13 rows per chunk
    assert cr == 13
    assert lib.hyena_operator_workspace(3, 1, 256, 1 << 20, 0) == 2 * cr * row
    assert lib.hyena_operator_workspace(3, 1, 14, 1 << 20, 0) == 2 * cr * row
    assert lib.hyena_operator_workspace(3, 1, 13, 1 << 20, 0) == cr * row
    assert lib.hyena_operator_workspace(2, 1, 5, 1 << 20, 1) == 5 * row
    one = (ctypes.c_int * 1)(1 << 20)
    assert lib.hyena_filter_spectrum_workspace(512, 1, one, 0) == 2 * cr * row
    assert lib.hyena_filter_spectrum_workspace(13, 1, one, 0) == cr * row
    dims = (ctypes.c_int * 3)(64, 64, 64)
    per_c = 64 * 128 * 65 * 8                        # one slab's planes of the 3-D convolution
    cs = (80 * MB) // per_c                          # 19 slabs per chunk
    assert lib.hyena_nd_conv_workspace(3, dims, 1, 40, 0) == 2 * cs * per_c
    assert lib.hyena_nd_conv_workspace(3, dims, 2, 19, 0) == 2 * cs * per_c
    assert lib.hyena_nd_conv_workspace(3, dims, 1, 19, 0) == cs * per_c
    assert lib.hyena_nd_conv_workspace(3, dims, 1, 5, 0) == 5 * per_c
    per_s = 128 * 128 * 65 * 8                       # one 128^3 kernel's planes of the 3-D spectrum
    assert lib.hyena_filter_spectrum_workspace(40, 3, dims, 0) == 2 * ((80 * MB) // per_s) * per_s
    assert lib.hyena_filter_spectrum_workspace(9, 3, dims, 0) == 9 * per_s
    # the minimum accepted: one chunk buffer (a byte less is a workspace error)
    far = 1 << 40                                    # fake device addresses far apart (no overlap)
    X2 = (ctypes.c_void_p * 2)(2 * far, 3 * far)
    H2 = (ctypes.c_void_p * 2)(5 * far, 6 * far)
    st = lib.hyena_operator(3, 1, 14, 1 << 20, 0, ctypes.c_void_p(far), X2, H2, None, ctypes.c_void_p(4 * far),
                            ctypes.c_void_p(7 * far), ctypes.c_size_t(cr * row - 1), None)
    assert _err(lib, st, "workspace") == 3


def test_binding_raises_named_errors(lib):
    with pytest.raises(hy.HyenaError) as ei:
        hy._check(lib.spectral_gate(1, 1, 1, 100, 1, FAKE, FAKE, 0, None, FAKE * 2, None))
    assert ei.value.status_name == "HY_ERR_UNSUPPORTED"


def test_spectrum_alias_check_uses_the_exact_extent(lib):
    """The aliasing check covers exactly the spectrum's bins: a circular
    spectrum (L/2+1 bins) right after the filters is accepted up to the
    launch (which fails without a GPU only after validation), one that
    overlaps is rejected; a ragged causal spectrum is M+1 bins long."""
    one = (ctypes.c_int * 1)(512)
    h = 0x100000
    # rows = 2, L = 512: h spans 4096 bytes; a spectrum starting there does not alias
    st = lib.hyena_filter_spectrum(2, 1, one, 1, h, h + 2 * 512 * 4, None, 0, None)
    assert st != 1 or b"aliases" not in lib.hyena_last_error()
    assert _err(lib, lib.hyena_filter_spectrum(2, 1, one, 1, h, h + 2 * 512 * 4 - 8, None, 0, None), "aliases") == 1
    # ragged causal L = 1000 -> 1025 bins per row: a spectrum ending inside h aliases
    ragged = (ctypes.c_int * 1)(1000)
    assert _err(lib, lib.hyena_filter_spectrum(1, 1, ragged, 0, h, h - 1025 * 8 + 8, None, 0, None), "aliases") == 1
