"""The FMA-pipe exp2 of the softmax (ex2_poly in csrc/ptx.cuh): its
coefficients are the ones the Remez fit in exp2_poly.py produces, and the
whole bit-level algorithm, replayed in fp32 on the CPU, stays within a
relative error far below bf16's 2^-9 over every input the softmax can give
it (scaled logits minus the running max: at most +8 with lazy rescaling)."""
import os
import re

import numpy as np

from long_context_sequence_ulysses_b200 import exp2_poly

PTX = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_sequence_ulysses_b200", "csrc", "ptx.cuh")


def _device_coefficients():
    src = open(PTX).read()
    body = src[src.index("float ex2_poly(float x)"):]
    body = body[:body.index("return")]
    lits = [float(v) for v in re.findall(r"([0-9]\.[0-9]+)f", body)]
    # fmaf(c3, f, c2), fmaf(p, f, c1), fmaf(p, f, c0)
    c3, c2, c1, c0 = lits[-4:]
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def _packed_device_coefficients():
    src = open(PTX).read()
    body = src[src.index("void ex2_poly2("):]
    body = body[:body.index("y0 = ")]
    lits = [float(v) for v in re.findall(r"([0-9]\.[0-9]+)f", body)]
    c3, c2, c1, c0 = lits[-4:]                      # operand order: c3, c2, c1, c0
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_coefficients_match_the_fit():
    assert np.array_equal(_device_coefficients(), exp2_poly.fp32_coefficients())
    assert np.array_equal(_packed_device_coefficients(), exp2_poly.fp32_coefficients())


def test_packed_exponent_insertion_is_the_same():
    # the packed form adds bits(t) << 23 instead of (bits(t) - 0x4B400000) << 23
    x = np.linspace(-125, 8, 200001, dtype=np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    tb = t.view(np.int32).astype(np.int64)
    a = (tb << 23) & 0xFFFFFFFF
    b = ((tb - 0x4B400000) << 23) & 0xFFFFFFFF
    assert np.array_equal(a, b)


def test_relative_error_bound():
    c = exp2_poly.fp32_coefficients()
    xs = np.concatenate([np.linspace(-125, 8, 2000001, dtype=np.float32),
                         np.arange(-125, 9, dtype=np.float32) + np.float32(0.5),
                         np.arange(-125, 9, dtype=np.float32)])
    got = exp2_poly.emulate(xs, c).astype(np.float64)
    rel = np.abs(got / np.exp2(xs.astype(np.float64)) - 1)
    assert rel.max() < 1e-4
    assert np.all(got > 0) and np.all(np.isfinite(got))


def test_masked_inputs_give_negligible_positive_values():
    c = exp2_poly.fp32_coefficients()
    got = exp2_poly.emulate(np.array([-np.inf, -1e30, -200.0, -125.0], dtype=np.float32), c)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 2.0 ** -124)
