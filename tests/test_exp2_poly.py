"""The exp2 cubic that the forward softmax uses for part of P = exp(S - m_new)
("Building Flash Attention from Scratch in Pure NumPy", Step 2, in base 2).

The device function exp2_poly_pair splits x = j + f (j = round(x) by the
1.5 * 2^23 rounding trick, f in [-0.5, 0.5]), evaluates a cubic p(f) by
Horner's rule with fused multiply-adds, and adds j to p's exponent field.
Pinned here against the mathematics, not against the kernel:
  * the constants in common.cuh are exactly the float32 output of the fit in
    fit_exp2_poly.py (an iteratively re-weighted least-squares approximation of
    the minimax cubic for relative error);
  * a float32 emulation of the whole device function (range reduction,
    Horner, exponent add) stays within the stated 7.5e-5 relative error of
    float64 exp2 for -125.5 <= x <= 0, and below 2^-125 under that;
  * on the GPU, the device function itself meets the same bounds, element by
    element, and its output is within one float32 step of the emulation's.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from tiled_exact_attention_forward_b200 import fit_exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 7.5e-5


def header_coefficients():
    """(c0, c1, c2, c3) as written in exp2_poly_pair (Horner order c3, c2, c1, c0)."""
    src = open(os.path.join(ROOT, "tiled_exact_attention_forward_b200", "csrc", "common.cuh")).read()
    body = src[src.index("uint64_t exp2_poly_pair"):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"f2_pack\(([0-9.eE+-]+)f, \1f\)", body)
    lits = [v for v in lits if v not in ("12582912.0",)]
    assert len(lits) == 4, lits
    c3, c2, c1, c0 = (np.float32(v) for v in lits)
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def emulate(x):
    """float32 emulation of exp2_poly_pair for an array of float32 x."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.5))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    c0, c1, c2, c3 = (np.float64(v) for v in header_coefficients())

    def fma(a, b, c):  # a * b is exact in float64; one rounding to float32
        return (a.astype(np.float64) * b.astype(np.float64) + c).astype(np.float32)

    p = fma(np.full_like(f, np.float32(c3)), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = (t.view(np.uint32).astype(np.uint64) << 23) + p.view(np.uint32).astype(np.uint64)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_header_constants_are_the_fit():
    fitted = fit_exp2_poly.fit()
    assert np.array_equal(header_coefficients().view(np.uint32), fitted.view(np.uint32)), (
        header_coefficients(), fitted)


def test_fitted_cubic_meets_its_bound_on_the_reduced_interval():
    err = fit_exp2_poly.max_rel_error_f32(header_coefficients())
    assert err <= BOUND, err
    # ... and is near the minimax level: a plain least-squares cubic would sit well above.
    assert err >= 5e-5


def test_emulated_device_function_within_bound():
    x = np.concatenate([np.linspace(-125.5, 0.0, 400001), -np.arange(0, 126) - 0.5,
                        -np.arange(0, 126).astype(np.float64)]).astype(np.float32)
    x = x[x >= -125.5]
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() <= BOUND, (rel.max(), x[np.argmax(rel)])


def test_emulated_device_function_floor_below_the_range():
    x = np.concatenate([np.linspace(-1000.0, -125.5, 10001), [-np.inf]]).astype(np.float32)
    got = emulate(x[:-1]).astype(np.float64)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -125)
    assert emulate(np.array([-np.inf], dtype=np.float32))[0] < 1e-38


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_device_exp2_poly_matches_emulation_and_bound():
    import tiled_exact_attention_forward_b200 as fa

    lib = fa.library()
    xs = np.concatenate([np.linspace(-125.5, 0.0, 1 << 20), np.linspace(-1000.0, -125.5, 4097),
                         [-np.inf, np.nan]]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    y = torch.full_like(x, float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fa_selftest_exp2_poly(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                     x.numel(), stream) == fa.FA_OK
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    got = y.cpu().numpy()
    inside = xs >= -125.5
    ref = np.exp2(xs[inside].astype(np.float64))
    rel = np.abs(got[inside].astype(np.float64) - ref) / ref
    assert rel.max() <= BOUND, rel.max()
    below = ~inside & ~np.isnan(xs)
    assert np.all(got[below] >= 0) and np.all(got[below] < 2.0 ** -125)
    # The clamp also swallows NaN (the softmax tracks NaN rows on its own).
    assert np.isfinite(got[-1]) and got[-1] < 2.0 ** -125
    # The emulation models the device function: equal to within one float32 step
    # (its fused multiply-add is emulated in float64 and rounded once more).
    finite = ~np.isnan(xs)
    steps = np.abs(got[finite].view(np.int32).astype(np.int64) - emulate(xs[finite]).view(np.int32).astype(np.int64))
    assert steps.max() <= 1, steps.max()
