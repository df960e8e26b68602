"""Error bound of the polynomial 2^x that the tensor-core kernel uses for part
of its softmax exponentials (exp2_poly.h), evaluated step by step in float32
the way the kernel does it, against numpy's float64 exp2."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "out_core_scheduling_b200", "csrc", "exp2_poly.h")


def coeffs():
    txt = open(HDR).read()
    c = {int(k): np.float32(v) for k, v in re.findall(r"CQSA_EXP2_C(\d) ([0-9.eE+-]+)f", txt)}
    return [c[i] for i in range(4)]


def exp2_poly_f32(x):
    """The kernel's steps: clamp at -126, y = x + 1.5*2^23 rounded down (the
    low mantissa bits hold floor(x)), f = x - (y - 1.5*2^23) in [0, 1), the
    polynomial by Horner in fp32, then floor(x) added to the exponent field."""
    c0, c1, c2, c3 = coeffs()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    y = (f32(12582912.0) + np.floor(x)).astype(f32)      # exact: an integer below 2^24
    f = (x - (y - f32(12582912.0)).astype(f32)).astype(f32)
    p = (c3 * f + c2).astype(f32)
    p = (p * f + c1).astype(f32)
    p = (p * f + c0).astype(f32)
    bits = p.view(np.int32) + (y.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_over_softmax_range():
    # Softmax arguments are at most 8 (lazy rescale) and decay to -inf.
    x = np.concatenate([np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32([-0.5, 0.5, 0.0, -1.0, 7.999])])
    got = exp2_poly_f32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.0e-4, rel.max()


def test_masked_and_tiny_arguments_are_negligible():
    x = np.float32([-np.inf, -1e30, -200.0, -127.0, -126.0, -125.5])
    got = exp2_poly_f32(x)
    assert np.all(got >= 0) and np.all(got < 1e-37)


def test_generator_reproduces_header():
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(os.path.dirname(HDR), "gen_exp2_poly.py")],
                         capture_output=True, text=True, check=True).stdout
    assert out == open(HDR).read()
