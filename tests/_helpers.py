"""Shared test helpers: moving seeded inputs to the device and comparing
device results with the float64 oracle."""
import numpy as np

# measured errors of this session (written out by conftest when PARITY_LOG is set)
RECORD = []

# tolerances of the hot path (fp32 math): fp32 I/O and bf16 I/O
F32_REL_L2 = 1e-5
F32_MAXABS_OF_RMS = 1e-4
BF16_REL_L2 = 1e-2


def to_dev(sig, dtype, device="cuda"):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(sig.bf16).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(sig.f32)).to(device)


def f32_dev(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float32))).to(device)


def c64_dev(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.complex64))).to(device)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a, ref):
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(a - ref) / (den if den > 0 else 1.0))


def check(a, ref, dtype, what=""):
    """Assert the hot-path tolerance: fp32 rel-L2 <= 1e-5 and max-abs <=
    1e-4 * RMS(ref); bf16 I/O rel-L2 <= 1e-2."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    assert a.shape == ref.shape, (a.shape, ref.shape)
    assert np.all(np.isfinite(a)), what + ": non-finite output"
    r = rel_l2(a, ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    mx = float(np.max(np.abs(a - ref))) if ref.size else 0.0
    RECORD.append({"what": what, "dtype": dtype, "rel_l2": r, "maxabs_over_rms": mx / rms if rms else 0.0})
    if dtype == "bf16":
        assert r <= BF16_REL_L2, "%s: rel-L2 %.3e > %.0e" % (what, r, BF16_REL_L2)
    else:
        assert r <= F32_REL_L2, "%s: rel-L2 %.3e > %.0e" % (what, r, F32_REL_L2)
        assert mx <= F32_MAXABS_OF_RMS * rms + 1e-30, "%s: max-abs %.3e > 1e-4*RMS %.3e" % (what, mx, rms)
    return r


def check_part(a, ref, rms_full, dtype, what=""):
    """The same tolerance for a slice of an output (a prefix, sampled
    positions), with errors measured against the RMS of the whole output the
    slice belongs to: RMS(err) <= 1e-5 * RMS_full and max-abs <= 1e-4 * RMS_full
    for fp32; RMS(err) <= 1e-2 * RMS_full for bf16 I/O."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    assert a.shape == ref.shape
    assert np.all(np.isfinite(a)), what + ": non-finite output"
    err = a - ref
    rms_err = float(np.sqrt(np.mean(err ** 2)))
    tol = BF16_REL_L2 if dtype == "bf16" else F32_REL_L2
    assert rms_err <= tol * rms_full, "%s: RMS err %.3e > %.0e * %.3e" % (what, rms_err, tol, rms_full)
    if dtype != "bf16":
        mx = float(np.max(np.abs(err)))
        assert mx <= F32_MAXABS_OF_RMS * rms_full, "%s: max-abs %.3e" % (what, mx)
    return rms_err / rms_full


def bf16_ulp_diff(dev_bf16_tensor, ref64, floor_of_rms=1e-2):
    """Largest distance in bf16 units-in-the-last-place between the device's
    bf16 output and the float64 reference rounded to bf16, over elements whose
    reference magnitude is at least floor_of_rms * RMS (near zero, fp32
    rounding of the convolution dominates the bf16 spacing)."""
    import hyena_workloads as hw
    got = dev_bf16_tensor.detach().cpu().view(__import__("torch").int16).numpy().view(np.uint16)
    want = hw.bf16_round(np.asarray(ref64, np.float32))

    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    ref = np.asarray(ref64, np.float64).ravel()
    mask = np.abs(ref) >= floor_of_rms * np.sqrt(np.mean(ref ** 2))
    d = np.abs(key(got.ravel()) - key(want.ravel()))[mask]
    return int(d.max()) if d.size else 0
