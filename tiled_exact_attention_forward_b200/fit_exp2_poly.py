"""Derive the cubic used for part of the exp2 work in the forward softmax.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-0.5, 0.5]
(Cody-Waite range reduction); 2^j goes into the float's exponent field, and
2^f is approximated by a cubic p(f).  The cubic minimises the maximum
RELATIVE error on [-0.5, 0.5]: a least-squares fit on Chebyshev points,
re-weighted towards the points of largest error until the error curve levels
out (an iteratively re-weighted approximation of the minimax polynomial).
P is rounded to bf16 (relative step 2^-8) right after, so an error below
1e-4 is invisible in the result.

    python -m tiled_exact_attention_forward_b200.fit_exp2_poly
prints the float32 coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the error.
"""
import numpy as np


def fit(degree=3, lo=-0.5, hi=0.5, iters=60):
    x = np.cos(np.linspace(0.0, np.pi, 2000)) * (hi - lo) / 2 + (hi + lo) / 2
    y = np.exp2(x)
    w = np.ones_like(x)
    for _ in range(iters):
        A = np.vander(x, degree + 1, increasing=True) / y[:, None]
        c, *_ = np.linalg.lstsq(A * np.sqrt(w)[:, None], np.sqrt(w), rcond=None)
        err = np.abs(np.polyval(c[::-1], x) - y) / y
        w = w * (1 + 10 * err / err.max())
        w /= w.mean()
    return c.astype(np.float32)


def max_rel_error_f32(c, lo=-0.5, hi=0.5, n=200001):
    f = np.linspace(lo, hi, n).astype(np.float32)
    p = np.zeros_like(f)
    for ci in np.asarray(c, dtype=np.float32)[::-1]:
        p = (p * f + ci).astype(np.float32)
    ref = np.exp2(f.astype(np.float64))
    return float((np.abs(p.astype(np.float64) - ref) / ref).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0..c3):", [float(v) for v in c])
    print("max relative error (float32 Horner):", max_rel_error_f32(c))
