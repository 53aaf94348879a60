"""hyena_operator_noalloc: the operator for callers that cannot allocate device
memory (allocator callbacks, plugins whose host owns all device memory,
real-time loops that must stay out of the driver's allocator).  Long sequences
keep their intermediates in the library's static device scratch instead of a
caller workspace; the results must match hyena_operator with a caller
workspace, call after call, although every call reuses the same scratch.

This file is collected last on purpose: a failure here leaves every other test
already run.  It passes alone in a fresh process and after the other tests."""
import numpy as np
import pytest

import hyena_workloads as hw
from _helpers import check, f32_dev, to_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _case(B, D, L, order, dtype, seed):
    w = hw.make("c3", seed=seed, B=B, D=D, L=L, order=order, dtype=dtype)
    K = order - 1
    rng = np.random.default_rng(seed)
    h32 = (rng.standard_normal((K * D, L)) * np.exp(-rng.uniform(0.1, 2.0, (K * D, 1)) * np.arange(L) / L)
           ).astype(np.float32)
    nb = hy.spectrum_bins(L)
    H = torch.empty((K * D, nb), dtype=torch.complex64, device="cuda")
    wsb = hy.filter_spectrum_workspace(K * D, 1, [L])
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(h32), H, rows=K * D, ndim=1, dims=[L], ws=ws)
    v = to_dev(w.v, dtype)
    xs = [to_dev(x, dtype) for x in w.xs]
    Hs = [H[k * D:(k + 1) * D] for k in range(K)]
    dsk = [f32_dev(w.Dskip[k]) for k in range(K)]
    return v, xs, Hs, dsk


def _with_workspace(v, xs, Hs, dsk):
    B, D, L = v.shape
    code = hy.HY_BF16 if v.dtype == torch.bfloat16 else hy.HY_F32
    wsb = hy.operator_workspace(len(xs) + 1, B, D, L, code)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(v)
    hy.hyena_operator(v, xs, Hs, y, Dskips=dsk, ws=ws)
    return y


def test_noalloc_matches_workspace_path_on_consecutive_calls():
    cases = [(1, 3, 1 << 17, 3, "f32", 11), (2, 5, 50000, 2, "bf16", 12)]
    prepared = [_case(*c) for c in cases]
    refs = [_with_workspace(*p) for p in prepared]
    torch.cuda.synchronize()
    # two calls in a row on the shared scratch, then the first shape again
    for i in (0, 1, 0):
        v, xs, Hs, dsk = prepared[i]
        y = torch.empty_like(v)
        hy.hyena_operator_noalloc(v, xs, Hs, y, Dskips=dsk)
        torch.cuda.synchronize()
        B, D, L = v.shape
        check(to_np(y).reshape(B * D, L), to_np(refs[i]).reshape(B * D, L), cases[i][4],
              "no-alloc vs workspace path, case %d" % i)


def test_noalloc_at_the_maximum_length_with_a_ragged_last_chunk():
    """L = 2^20, the longest sequence the static scratch takes: one row needs
    8 MiB of it, so the 32 MiB array holds four rows per chunk and the fifth
    row is a chunk of its own.  Two consecutive calls, both equal to the
    workspace path."""
    v, xs, Hs, dsk = _case(1, 5, 1 << 20, 2, "f32", 14)
    ref = _with_workspace(v, xs, Hs, dsk)
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.empty_like(v)
        hy.hyena_operator_noalloc(v, xs, Hs, y, Dskips=dsk)
        torch.cuda.synchronize()
        check(to_np(y).reshape(5, -1), to_np(ref).reshape(5, -1), "f32", "no-alloc at L = 2^20, call %d" % call)


def test_noalloc_short_sequences_and_limits():
    # on-chip lengths need no scratch at all
    v, xs, Hs, dsk = _case(2, 3, 4096, 2, "bf16", 13)
    y = torch.empty_like(v)
    hy.hyena_operator_noalloc(v, xs, Hs, y, Dskips=dsk)
    ref = _with_workspace(v, xs, Hs, dsk)
    torch.cuda.synchronize()
    check(to_np(y).reshape(6, -1), to_np(ref).reshape(6, -1), "bf16", "no-alloc on chip")
    # longer than one row of the static scratch (8 bytes per complex point of
    # the 2L transform, 64 MiB here): rejected before any launch
    L = 1 << 23
    x = torch.empty((1, 1, L), device="cuda")
    H = torch.empty((1, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    with pytest.raises(hy.HyenaError) as ei:
        hy.hyena_operator_noalloc(x, [x], [H], torch.empty_like(x))
    assert ei.value.status_name in ("HY_ERR_WORKSPACE", "HY_ERR_UNSUPPORTED")
    assert "scratch" in str(ei.value)
