"""The FMA-pipe exp2 used for part of the forward's exponentials.

Checks that the coefficients in the kernel source are the generator's fit,
and that the kernel's fp32 arithmetic (replayed in numpy) stays within its
stated relative error of exp2 over the whole range the softmax uses.  The GPU
parity tests then check the kernels that use it end to end.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_attention_106_b200", "csrc")
sys.path.insert(0, CSRC)
import gen_exp2_poly  # noqa: E402


def kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    line = next(ln for ln in src.splitlines() if "const float p = fmaf(" in ln)
    nums = [float(x) for x in re.findall(r"([0-9]+\.[0-9]+(?:e-?[0-9]+)?)f", line)]
    # nested Horner: c3, c2, c1, then c0
    c3, c2, c1, c0 = nums
    return [c0, c1, c2, c3]


def test_kernel_uses_the_fitted_coefficients():
    fitted, err = gen_exp2_poly.fit()
    assert err < 1.1e-4
    got = kernel_coefficients()
    want = [float(np.float32(v)) for v in fitted]
    assert got == want, (got, want)


def test_fp32_relative_error_bound():
    c = kernel_coefficients()
    x = np.linspace(-126.0, 8.0, 4_000_001).astype(np.float32)
    y = gen_exp2_poly.emulate_fp32(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.1e-4


def test_exact_at_integers_and_zero_below_range():
    c = kernel_coefficients()
    ints = np.arange(-126, 9, dtype=np.float32)
    np.testing.assert_array_equal(gen_exp2_poly.emulate_fp32(ints, c), np.exp2(ints.astype(np.float64)))
    low = np.array([-127.0, -200.0, -np.inf], dtype=np.float32)
    np.testing.assert_array_equal(gen_exp2_poly.emulate_fp32(low, c), np.zeros(3, np.float32))
