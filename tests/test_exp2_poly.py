"""The FMA-pipe exp2 used by the prefill softmax, emulated step by step in
float32 on the CPU: round-to-nearest split with the 1.5 * 2^23 shift, cubic
polynomial on [-1/2, 1/2], exponent-field add; checked against exp2 and the
bf16 rounding it feeds (relative step 2^-8)."""

import re
import os

import numpy as np

import exp2_poly_fit as fit_exp2_poly

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "attention_online_softmax_fwd_b200", "csrc", "common.cuh")


def kernel_coefficients():
    text = open(CSRC).read()
    m = re.search(r"c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f", text)
    return [np.float32(float(g)) for g in m.groups()]


def emulate(x):
    c0, c1, c2, c3 = kernel_coefficients()
    x = np.minimum(np.maximum(x.astype(np.float32), np.float32(-126)), np.float32(64))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(c3) * f + c2
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_coefficients_match_the_fit():
    c, rel = fit_exp2_poly.fit()
    assert rel < 1e-4
    for a, b in zip(kernel_coefficients(), c):
        assert abs(float(a) - b) < 1e-7


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-40.0, 8.0, 400001, dtype=np.float32)
    y = emulate(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 2e-4, rel.max()          # far below the bf16 step of 2^-8


def test_underflow_and_masked_inputs_are_harmless():
    y = emulate(np.array([-np.inf, -1e30, -200.0, -126.0, -125.5], dtype=np.float32))
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 1e-37)
