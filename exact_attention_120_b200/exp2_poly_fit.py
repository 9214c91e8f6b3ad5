"""Fit of the polynomial the kernel uses to evaluate 2^x on the FMA pipe.

The softmax needs one exp2 per score; the hardware exp2 unit (MUFU) delivers
16 results per clock per SM, which at head dim 128 is exactly the rate the
tensor cores consume scores.  The kernel therefore evaluates a fixed share of
its exp2 with ordinary FMA-pipe arithmetic:

* range reduction after Cody and Waite ("Software Manual for the Elementary
  Functions", 1980): x = n + f with n = round(x) (obtained by adding and
  subtracting 1.5 * 2^23, which rounds to an integer in fp32) and
  f in [-1/2, 1/2];
* 2^f from a degree-3 polynomial c0 + c1 f + c2 f^2 + c3 f^3 whose
  coefficients are fitted here to minimise the maximum *relative* error on
  [-1/2, 1/2] (iteratively reweighted least squares on a dense grid, which
  converges to the equioscillating minimax solution);
* 2^n applied by adding n to the fp32 exponent field.

The result is rounded to bf16 right after (relative half-ulp 2^-9), so a
relative error near 1e-4 is far below what the output keeps.

Run ``python -m exact_attention_120_b200.exp2_poly_fit`` to print the
coefficients as fp32 literals; tests/test_exp2_poly.py checks that the
constants in the kernel match this fit and its error bound.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3
INTERVAL = (-0.5, 0.5)
# Smallest argument evaluated: keeps n + the exponent of 2^f (>= 126) a
# normal exponent; anything below (masked scores are -inf) gives 2^-125 ~ 0.
CLAMP = -125.0


def fit(degree: int = DEGREE, iters: int = 60):
    f = np.linspace(*INTERVAL, 20001)
    target = np.exp2(f)
    w = np.ones_like(f)
    V = np.vander(f, degree + 1, increasing=True)
    coef = None
    for _ in range(iters):
        # weighted least squares on the relative error
        A = V * (w / target)[:, None]
        b = w
        coef, *_ = np.linalg.lstsq(A, b, rcond=None)
        err = np.abs(V @ coef / target - 1.0)
        w = w * (err / err.max()) ** 0.5 + 1e-12  # push weight toward the peaks
        w /= w.max()
    rel = np.abs(V @ coef / target - 1.0).max()
    return coef.astype(np.float32), float(rel)


def exp2_emulated(x):
    """The kernel's sequence of fp32 operations, in NumPy float32 (for tests)."""
    c, _ = fit()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(CLAMP))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    fr = (x - r).astype(np.float32)
    q = (fr * c[3] + c[2]).astype(np.float32)
    q = (q * fr + c[1]).astype(np.float32)
    q = (q * fr + c[0]).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    coef, rel = fit()
    for i, c in enumerate(coef):
        print(f"c{i} = {float(c):.9e}f  (hex {np.float32(c).view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
