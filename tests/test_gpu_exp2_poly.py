"""The polynomial 2^x of the tcgen05 prefill kernel, checked on its own over its
whole domain (through the msa_selftest_exp2_poly hook of the C ABI).

The kernel takes part of its softmax exponentials as 2^x = 2^n * p(f), with n the
nearest integer to x, f = x - n in [-1/2, 1/2] and p a Remez cubic whose relative
error on that interval is 7.48e-5 in exact arithmetic (computed here in fp64).
Evaluated in fp32 it gains a few units of 2^-24. The bound asserted is the
kernel's stated 7.5e-5, against an fp64 reference; CUDA's exp2f on the same grid
is checked too (much tighter), so a wrong grid or reference would show."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

POLY_REL = 7.5e-5


def _grid():
    rng = np.random.default_rng(5)
    dense = np.linspace(-125.0, 64.0, 1 << 21)
    ints = np.arange(-125, 65, dtype=np.float64)
    near = np.concatenate([ints + 0.5, ints - 0.5, ints + 0.5 - 1e-6, ints + 0.5 + 1e-6, ints])
    rand = rng.uniform(-125.0, 64.0, 1 << 20)
    x = np.concatenate([dense, near, rand]).astype(np.float32)
    return x[(x >= -125.0) & (x <= 64.0)]


def _run(x: np.ndarray):
    from sparse_attention_routed_b200 import msa_selftest_exp2_poly
    xd = torch.from_numpy(x).cuda()
    yp = torch.empty_like(xd)
    yl = torch.empty_like(xd)
    msa_selftest_exp2_poly(xd.data_ptr(), yp.data_ptr(), yl.data_ptr(), xd.numel(),
                           torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return yp.cpu().numpy().astype(np.float64), yl.cpu().numpy().astype(np.float64)


def test_exp2_poly_relative_error_over_its_domain():
    x = _grid()
    yp, yl = _run(x)
    ref = np.exp2(x.astype(np.float64))
    rel_poly = np.abs(yp / ref - 1.0)
    rel_lib = np.abs(yl / ref - 1.0)
    assert np.all(np.isfinite(yp)) and np.all(yp > 0)
    assert rel_poly.max() <= POLY_REL, f"polynomial 2^x relative error {rel_poly.max():.3e} at x={x[rel_poly.argmax()]}"
    assert rel_lib.max() <= 1e-6, f"exp2f relative error {rel_lib.max():.3e}"
    # the error is the cubic's: it must come close to its equioscillation level somewhere
    assert rel_poly.max() >= 5e-5
    print(f"max relative error: polynomial {rel_poly.max():.3e}, exp2f {rel_lib.max():.3e} over {x.size} points")


def test_exp2_poly_clamps_outside_its_domain():
    x = np.array([-1000.0, -126.0, -125.0, 64.0, 65.0, 1000.0], dtype=np.float32)
    yp, _ = _run(x)
    lo = np.exp2(-125.0)
    hi = np.exp2(64.0)
    # below -125 the result is 2^-125 (within the polynomial's error); above 64 it stays at 2^64
    assert np.all(np.abs(yp[:3] / lo - 1.0) <= POLY_REL)
    assert np.all(np.abs(yp[3:] / hi - 1.0) <= POLY_REL)
