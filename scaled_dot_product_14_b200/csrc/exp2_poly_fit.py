"""Fits the polynomial the prefill softmax uses to evaluate 2^x on the FMA
pipe for a share of its exponentials, so that the MUFU unit is not the only
source of them.

Method (range reduction as in Cody and Waite): n = round(x) through the
float "magic number" 1.5 * 2^23 (one FADD, no conversion instruction),
f = x - n in [-1/2, 1/2], and a cubic p(f) ~ 2^f fitted by least squares in
relative error on a dense grid; the result is p with n added to its exponent
field.  The printed coefficients are the ones in common.cuh; the bound is far
below the 2^-9 relative rounding of the bf16 P (2^-11 for fp16) the result is
rounded to.

    python scaled_dot_product_14_b200/csrc/exp2_poly_fit.py
"""
import numpy as np

MAGIC = np.float32(12582912.0)   # 1.5 * 2^23


def fit():
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    A = np.stack([np.ones_like(f), f, f ** 2, f ** 3], axis=1) / y[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return tuple(np.float32(v) for v in c)


def evaluate(x, c):
    """The kernel's arithmetic in float32 (inputs clamped at -126 as in the kernel)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + MAGIC).astype(np.float32)
    n = (t - MAGIC).astype(np.float32)
    f = (x - n).astype(np.float32)
    c0, c1, c2, c3 = c
    p = ((f * c3 + c2) * f + c1) * f + c0
    bits = p.astype(np.float32).view(np.uint32) + (t.view(np.uint32) << np.uint32(23)) \
        - (MAGIC.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c = fit()
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(evaluate(x, c).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    print("c0 = %.9ef, c1 = %.9ef, c2 = %.9ef, c3 = %.9ef" % c)
    print("max relative error on [-120, 8]: %.3e" % rel.max())
