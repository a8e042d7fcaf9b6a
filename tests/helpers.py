"""Shared helpers for the GPU parity tests (plumbing only: no attention math)."""
import numpy as np

TOL_O = 1e-2     # max |O_gpu - O_oracle|
TOL_LSE = 1e-3   # max |LSE_gpu - LSE_oracle|


def to_dev_bf16(bits, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def to_dev_i32(a, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def to_f64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def bf16_half_ulp(x):
    """Half a bf16 ulp at |x| (the rounding error of a bf16 output)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def assert_o_close(o_gpu, o_ref, bf16_out: bool, what=""):
    """|dO| <= 1e-2 on fp32 output; on bf16 output |dO| <= max(1e-2, half a bf16
    ulp of the reference value), since for |O| >= 4 the correctly rounded bf16
    value alone can be 0.0156 away."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    tol = np.maximum(TOL_O, bf16_half_ulp(o_ref)) if bf16_out else TOL_O
    bad = err > tol
    assert not bad.any(), (f"{what}: max|dO|={err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}, "
                           f"{bad.sum()} elements over tolerance")
    return float(err.max())


def assert_lse_close(l_gpu, l_ref, what=""):
    l_gpu = np.asarray(l_gpu, dtype=np.float64)
    l_ref = np.asarray(l_ref, dtype=np.float64)
    assert l_gpu.shape == l_ref.shape
    inf_ref = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(l_gpu), inf_ref), f"{what}: -inf pattern differs"
    fin = ~inf_ref
    err = np.abs(l_gpu[fin] - l_ref[fin]) if fin.any() else np.zeros(1)
    assert np.isfinite(l_gpu[fin]).all(), f"{what}: non-finite LSE"
    assert err.max() <= TOL_LSE, f"{what}: max|dLSE|={err.max():.3g}"
    return float(err.max())
