"""Pin of the FMA-pipe exponential used by the attention softmax on full blocks.

The kernel evaluates 2^x as 2^floor(x) * p(x - floor(x)) with a cubic p
(p(0) = 1) whose coefficients sit in the kernel source. This test reads them
from the source and checks the relative error of the construction against
numpy's exp2 in float32 arithmetic, over the arguments the softmax produces
(x <= 8 after the reference max; x clamped at -127): it must stay below 1e-4,
i.e. below the bf16 rounding (2^-9) that P undergoes right after.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "sparse_rank_attention_block_b200", "csrc", "ex2_fma.cuh")


def _coeffs():
    text = open(SRC).read()
    m = re.search(r"kPoly1 = ([0-9.eE+-]+)f, kPoly2 = ([0-9.eE+-]+)f, kPoly3 = ([0-9.eE+-]+)f", text)
    assert m, "polynomial coefficients not found in the kernel source"
    return [np.float32(m.group(i)) for i in (1, 2, 3)]


def _ex2_emulated(x):
    """Float32 restatement of the kernel's steps (round-down split, Horner, exponent add)."""
    c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    j = np.floor(x).astype(np.float32)            # the kernel gets floor(x) from a round-down add
    f = (x - j).astype(np.float32)
    p = np.float32(c3) * f + c2
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    return np.ldexp(p.astype(np.float64), j.astype(np.int64))


def test_relative_error_below_bf16_rounding():
    x = np.linspace(-60.0, 8.0, 200001)
    got = _ex2_emulated(x)
    want = np.exp2(x.astype(np.float32).astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_integer_arguments_are_exact_powers_of_two():
    x = np.arange(-40, 9, dtype=np.float32)
    assert np.array_equal(_ex2_emulated(x), np.exp2(x.astype(np.float64)))


def test_continuity_at_the_integer_boundaries():
    # p(1-) must meet 2 * p(0) = 2 closely, else the curve jumps at every integer
    c1, c2, c3 = _coeffs()
    assert abs((1.0 + c1 + c2 + c3) - 2.0) < 2e-4
