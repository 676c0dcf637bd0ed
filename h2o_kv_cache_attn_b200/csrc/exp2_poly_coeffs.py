"""Coefficients of the polynomial 2^f on [-1/2, 1/2] used by the tensor-core
attention kernel to compute part of its exponentials on the FMA pipe.

Method: near-minimax fit of the RELATIVE error by Lawson's algorithm
(iteratively reweighted least squares on Chebyshev points), degree 4.  The
kernel evaluates 2^x as 2^n * p(f) with n = rint(x), f = x - n, p in Horner
form in float32; ``max_rel_error`` below evaluates exactly that in float32
(fma emulated in float64) and is checked by tests/test_exp2_poly.py.

    python h2o_kv_cache_attn_b200/csrc/exp2_poly_coeffs.py
"""

import numpy as np

DEGREE = 4


def fit(degree=DEGREE, iters=60):
    x = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = np.exp2(x)
    V = np.vander(x, degree + 1, increasing=True)
    w = np.ones_like(x)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V / y[:, None] * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def exp2_poly(x, coeffs):
    """float32 model of the kernel's evaluation for x in [-126, 0]."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23: x + magic holds rint(x) in its low bits
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = fma32(n, np.float32(-1.0), x)
    p = np.full_like(f, coeffs[-1])
    for k in range(len(coeffs) - 2, -1, -1):
        p = fma32(p, f, np.float32(coeffs[k]))
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def max_rel_error(coeffs, n=2_000_001):
    x = np.linspace(-125.9, 0.0, n).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(exp2_poly(x, coeffs).astype(np.float64) / ref - 1.0)))


# Coefficients compiled into attn_tc.cu (c0 + c1 f + c2 f^2 + c3 f^3 + c4 f^4).
KERNEL_COEFFS = np.array([0.9999992847442627, 0.6931217908859253, 0.240247443318367,
                          0.05591786280274391, 0.009570101276040077], np.float32)

if __name__ == "__main__":
    c = fit()
    print("fitted:", [float(v) for v in c], "max rel err", max_rel_error(c))
    print("kernel:", [float(v) for v in KERNEL_COEFFS], "max rel err", max_rel_error(KERNEL_COEFFS))
