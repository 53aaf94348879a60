"""Input projection (v, x_1, ... = split(W_proj x), written channel-major)
against the float64 oracle: ragged and odd sizes in bf16 (the tcgen05 GEMM:
partial M, L and K tiles, several tiles per CTA) and fp32, with and without
bias; bf16 outputs are the fp32 result plus bias rounded once (within one
bf16 ulp of the float64 value); the projection feeding the operator end to
end; and the order-2 projection at the width of the operator workload (B8
L8192, 768 -> 2 x 768) on sampled rows."""
import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import bf16_ulp_diff, check, f32_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _bf16_dev(a):
    return torch.from_numpy(hw.bf16_round(a).view(np.int16)).view(torch.bfloat16).cuda()


def _ws():
    return torch.empty(hy.projection_workspace(), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("B,L,C,D,n_out,dtype,with_bias", [
    (2, 1000, 64, 48, 3, "bf16", True),
    (3, 257, 24, 40, 2, "bf16", False),
    (4, 8000, 200, 100, 3, "bf16", True),
    (1, 513, 32, 16, 2, "f32", True),
    (2, 64, 8, 5, 4, "f32", False),
])
def test_projection_vs_oracle(B, L, C, D, n_out, dtype, with_bias):
    rng = np.random.default_rng(B * 1000 + L)
    x = rng.standard_normal((B, L, C)).astype(np.float32)
    W = (rng.standard_normal((n_out * D, C)) / np.sqrt(C)).astype(np.float32)
    bias = rng.standard_normal(n_out * D).astype(np.float32) if with_bias else None
    if dtype == "bf16":
        xd, Wd = _bf16_dev(x), _bf16_dev(W)
        x, W = hw.bf16_to_f32(hw.bf16_round(x)), hw.bf16_to_f32(hw.bf16_round(W))   # the values the GPU sees
        tdt = torch.bfloat16
    else:
        xd, Wd = f32_dev(x), f32_dev(W)
        tdt = torch.float32
    outs = [torch.empty((B, D, L), dtype=tdt, device="cuda") for _ in range(n_out)]
    hy.hyena_projection(xd, Wd, outs, bias=f32_dev(bias) if with_bias else None, ws=_ws())
    torch.cuda.synchronize()
    ref = oracle.projection(x, W, bias, n_out)
    for k in range(n_out):
        check(to_np(outs[k]), ref[k], dtype, "projection %s out %d" % (dtype, k))
        if dtype == "bf16":
            # one rounding of the fp32 accumulator plus bias
            assert bf16_ulp_diff(outs[k], ref[k]) <= 1, "projection out %d: more than 1 bf16 ulp" % k


def test_projection_then_operator():
    """x -> (v, x1) by the projection -> the order-2 operator, against the
    oracle's own projection (rounded to bf16 like the GPU's) -> direct chain."""
    B, L, C, D = 2, 2048, 64, 32
    rng = np.random.default_rng(21)
    x = hw.bf16_to_f32(hw.bf16_round(rng.standard_normal((B, L, C)).astype(np.float32)))
    W = hw.bf16_to_f32(hw.bf16_round((rng.standard_normal((2 * D, C)) / 8).astype(np.float32)))
    t = np.arange(L)
    h = (rng.standard_normal((D, L)) * np.exp(-rng.uniform(0.5, 3, (D, 1)) * t / L)).astype(np.float32)
    Dk = rng.standard_normal(D).astype(np.float32)
    v_d = torch.empty((B, D, L), dtype=torch.bfloat16, device="cuda")
    x1_d = torch.empty_like(v_d)
    hy.hyena_projection(_bf16_dev(x), _bf16_dev(W), [v_d, x1_d], ws=_ws())
    H = torch.empty((D, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(h), H, rows=D, ndim=1, dims=[L])
    y = torch.empty_like(v_d)
    hy.hyena_operator(v_d, [x1_d], [H], y, Dskips=[f32_dev(Dk)])
    torch.cuda.synchronize()
    pv, px1 = oracle.projection(x, W, None, 2)
    pv = hw.bf16_to_f32(hw.bf16_round(pv.astype(np.float32)))
    px1 = hw.bf16_to_f32(hw.bf16_round(px1.astype(np.float32)))
    ref = oracle.hyena_rows(pv, [px1], h[None].astype(np.float64), Dk[None])
    check(to_np(y).reshape(B * D, L), ref, "bf16", "projection -> operator")


def test_projection_operator_width_sampled():
    B, L, C, D = 8, 8192, 768, 768
    rng = np.random.default_rng(22)
    x = rng.standard_normal((B, L, C)).astype(np.float32)
    W = (rng.standard_normal((2 * D, C)) / np.sqrt(C)).astype(np.float32)
    bias = (0.1 * rng.standard_normal(2 * D)).astype(np.float32)
    outs = [torch.empty((B, D, L), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    hy.hyena_projection(_bf16_dev(x), _bf16_dev(W), outs, bias=f32_dev(bias), ws=_ws())
    torch.cuda.synchronize()
    xs = hw.bf16_to_f32(hw.bf16_round(x))
    Ws = hw.bf16_to_f32(hw.bf16_round(W))
    for b, ls in [(0, slice(0, 256)), (5, slice(4000, 4128)), (7, slice(8192 - 200, 8192))]:
        ref = oracle.projection(xs[b:b + 1, ls], Ws, bias, 2)
        for k in range(2):
            check(to_np(outs[k][b:b + 1, :, ls]), ref[k], "bf16", "projection B8 L8192 b%d out %d" % (b, k))
            assert bf16_ulp_diff(outs[k][b:b + 1, :, ls].contiguous(), ref[k]) <= 1
