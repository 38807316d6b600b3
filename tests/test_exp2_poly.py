"""The FMA-pipe exp2 of the kernels (the maps' row sums): constants and error bound (CPU).

The kernels' coefficients (common.cuh, kExp2C0..4) must be exactly what
csrc/exp2_poly.py derives (Remez minimax of 2^f on [-1/2, 1/2]), and the kernel's fp32
step sequence (clamp, 1.5 * 2^23 rounding shift, Horner, exponent-field add) must stay
within 3e-6 relative error of exp2 over the whole input range the softmax produces."""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "structured_sparse_attention_b200", "csrc")
sys.path.insert(0, CSRC)

import exp2_poly  # noqa: E402


def kernel_constants():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    vals = dict(re.findall(r"constexpr float kExp2C(\d) = ([0-9eE+\-.]+)f;", src))
    return np.array([np.float32(vals[str(k)]) for k in range(len(vals))], np.float32)


def test_constants_match_generator():
    assert np.array_equal(kernel_constants(), exp2_poly.coefficients_f32())


def test_relative_error_bound():
    c = kernel_constants()
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly.emulate(x, c).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 3e-6, rel.max()


def test_special_values():
    c = kernel_constants()
    # integers are reproduced to the polynomial's accuracy, -inf (a masked logit) clamps
    # to 2^-126 and stays positive
    x = np.array([0.0, 1.0, -1.0, 8.0, -126.0, -np.inf], np.float32)
    got = exp2_poly.emulate(x, c).astype(np.float64)
    want = np.exp2(np.maximum(x.astype(np.float64), -126.0))
    assert np.all(np.abs(got / want - 1.0) <= 3e-6)
    assert got[-1] > 0.0
