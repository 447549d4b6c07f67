"""Error bound of the FMA-pipe exp2 used by the attention softmax.

The kernel reduces x = n + f with n = round(x) (the 1.5 * 2^23 shifter), evaluates a degree-3
polynomial for 2^f on [-1/2, 1/2] with fused multiply-adds in fp32, and adds n to the exponent
field.  This test redoes those fp32 steps in numpy over the argument range the softmax produces
and bounds the relative error against 2^x in float64; it also checks that the coefficients in the
kernel source are the ones the Remez generator produces.
"""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "request_candidate_sharing_b200", "csrc")


def _kernel_coeffs():
    src = open(os.path.join(CSRC, "softmax_math.cuh")).read()
    m = re.search(r"c3 = dup2\(([0-9.e+-]+)f\), c2 = dup2\(([0-9.e+-]+)f\), c1 = dup2\(([0-9.e+-]+)f\), "
                  r"c0 = dup2\(([0-9.e+-]+)f\)", src)
    assert m, "polynomial coefficients not found in softmax_math.cuh"
    c3, c2, c1, c0 = (np.float32(float(v)) for v in m.groups())
    return c0, c1, c2, c3


def _fma32(a, b, c):
    # fp32 fused multiply-add: the fp32 x fp32 product is exact in float64
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x, coeffs):
    c0, c1, c2, c3 = coeffs
    x = np.maximum(x.astype(np.float32), np.float32(-126))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32), n


def test_coefficients_match_generator():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, err = gen.remez(3)
    assert err < 8e-5
    np.testing.assert_allclose(np.array(_kernel_coeffs(), dtype=np.float64), c.astype(np.float64), rtol=2e-7)


def test_relative_error_bound():
    rng = np.random.default_rng(0)
    # the softmax argument s*log2(e)/sqrt(d) - m lies in (-inf, 8]; cover the normal range densely,
    # plus every half-integer boundary of the range reduction
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), rng.uniform(-30, 8, 1_000_000),
                        np.arange(-125.5, 8.0, 0.5), np.arange(-125.5, 8.0, 0.5) + 1e-6]).astype(np.float32)
    y, n = _exp2_poly(x, _kernel_coeffs())
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - ref) / ref
    # 7.5e-5 from the minimax fit plus a few fp32 roundings (2^-24 each) in the reduction and Horner
    assert rel.max() < 1.0e-4, rel.max()
    # far below the bf16 rounding (2^-9) that P then undergoes
    assert rel.max() < 2.0 ** -9 / 10


def test_underflow_and_clamp():
    y, _ = _exp2_poly(np.array([-np.inf, -1000.0, -126.0], dtype=np.float32), _kernel_coeffs())
    assert np.all(y >= 0) and np.all(y < 2.0 ** -125)
