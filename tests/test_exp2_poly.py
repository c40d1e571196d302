"""The softmax evaluates a share of its exponentials with a cubic on the FMA
pipe (common.cuh, f2_exp2_poly).  Its constants must be the fit that
exp2_poly_fit.py produces, and the kernel's float32 arithmetic (re-run here in
numpy) must stay within a relative error far below the rounding of the 16-bit
P it feeds (2^-9 for bf16, 2^-11 for fp16)."""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "scaled_dot_product_14_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def kernel_coefficients():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("f2_exp2_poly(uint64_t x)"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([0-9.]+e[+-][0-9]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals
    return tuple(np.float32(v) for v in (c0, c1, c2, c3))


def test_constants_are_the_fit():
    m = _fit_module()
    assert kernel_coefficients() == m.fit()


def test_relative_error_bound():
    m = _fit_module()
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-120.0, 8.0, 1_000_001, dtype=np.float32),
                        np.arange(-120, 9, dtype=np.float32),            # integers: f = 0
                        np.arange(-120, 8, dtype=np.float32) + 0.5])     # ties of the rounding
    rel = np.abs(m.evaluate(x, c).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2.0 ** -12          # 2.4e-4, vs bf16 2^-9 and fp16 2^-11
    # monotone enough that p never exceeds the row maximum's 2^0 by more than the error
    assert m.evaluate(np.float32(0.0), c) <= 1.0 + 2.0 ** -12
