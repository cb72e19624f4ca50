"""The FMA-pipe exp2 used for a share of the softmax exponentials.

The kernel computes 2^x as 2^round(x) * q(r), r = x - round(x) in [-1/2, 1/2],
q(r) = 1 + r*(c1 + r*(c2 + r*c3)) with c1..c3 from csrc/gen_exp2_poly.py
(minimax relative error with q(0) = 1, so integer arguments are exact).  This test replays the exact float32 operation
sequence (the 1.5*2^23 rounding trick, Horner with fused multiply-add, the
integer add into the exponent field) and bounds its error against 2^x, and
checks that the constants in the kernel are the generator's output.
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "sm_attn_fwd_b200", "csrc", "attn_prefill.cu")
GEN = os.path.join(ROOT, "sm_attn_fwd_b200", "csrc", "gen_exp2_poly.py")


def kernel_coefficients():
    """(c3, c2, c1) as written in the kernel's exp2_fma."""
    text = open(SRC).read()
    body = text[text.index("float exp2_fma(float x)"):]
    body = body[:body.index("}")]
    vals = [np.float32(v) for v in re.findall(r"([0-9.]+e[-+][0-9]+)f", body)]
    return vals[0], vals[1], vals[2]


def fma32(a, b, c):
    return (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)


def exp2_fma(x, c3, c2, c1):
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0)).astype(np.float32)
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    r = (x - (t - k).astype(np.float32)).astype(np.float32)
    q = fma32(np.float32(c3), r, np.float32(c2))
    q = fma32(q, r, np.float32(c1))
    q = fma32(q, r, np.float32(1.0))
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_kernel_constants_come_from_the_generator():
    out = subprocess.run([sys.executable, GEN], capture_output=True, text=True, check=True).stdout
    gen = [np.float32(v) for v in re.findall(r"c\d = ([0-9.e+-]+)f", out)]
    c3, c2, c1 = kernel_coefficients()
    assert [c1, c2, c3] == gen


def test_relative_error_bound_over_the_softmax_range():
    c3, c2, c1 = kernel_coefficients()
    # arguments s*c - m: at most 8 (lazy rescale threshold), down to deep underflow
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32(np.random.default_rng(0).uniform(-30, 8, 500_000))])
    got = exp2_fma(x, c3, c2, c1).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    normal = x >= -125.0
    rel = np.abs(got[normal] / want[normal] - 1.0)
    assert rel.max() < 1.1e-4          # vs bf16 rounding of P: 2^-9 = 2e-3
    # at the clamp the exponent add reaches the subnormal range: tiny absolute error
    assert np.abs(got[~normal] - want[~normal]).max() < 2.0 ** -125


def test_integer_arguments_are_exact():
    c3, c2, c1 = kernel_coefficients()
    xi = np.arange(-125, 9, dtype=np.float32)
    assert np.array_equal(exp2_fma(xi, c3, c2, c1).astype(np.float64), np.exp2(xi.astype(np.float64)))


def test_clamped_below():
    c3, c2, c1 = kernel_coefficients()
    y = exp2_fma(np.array([-1000.0, -np.inf, -126.0], dtype=np.float32), c3, c2, c1)
    assert np.all(y > 0) and np.all(y < 2.0 ** -125)
