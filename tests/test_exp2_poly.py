"""The FMA-pipe 2^x used for part of the softmax exponentials: the constants
in sm100.cuh, evaluated the way the kernel does (float32, round-to-nearest
shifter range reduction, Horner with fused multiply-adds, exponent-field
add), agree with 2^x to the stated bound over the range the kernel feeds it,
stay normal floats for tiny arguments, and match the fit."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "io_aware_exact_33_b200", "csrc", "sm100.cuh")


def coefficients():
    body = open(HDR).read().split("void exp2_poly2(float x0, float x1, float& r0, float& r1) {")[1]
    body = body.split("\n}\n")[0]
    nums = [float(x.rstrip("f")) for x in re.findall(r"[-+]?\d\.\d+e[-+]\d+f", body)]
    # each coefficient appears twice (packed pair): c3, c3, c2, c2, c1, c1, c0, c0
    c3, c2, c1, c0 = nums[0::2]
    assert nums[1::2] == nums[0::2]
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def fma32(a, b, c):
    """float32 fused multiply-add: the float32 product is exact in float64."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly2(x):
    c0, c1, c2, c3 = (np.full(1, c, dtype=np.float32) for c in coefficients())
    shifter = np.float32(12582912.0)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    t = (x + shifter).astype(np.float32)          # round to nearest even
    n = (t - shifter).astype(np.float32)          # exact
    f = fma32(n, np.full_like(n, -1.0), x)        # x - n, exact
    p = fma32(np.broadcast_to(c3, f.shape), f, np.broadcast_to(c2, f.shape))
    p = fma32(p, f, np.broadcast_to(c1, f.shape))
    p = fma32(p, f, np.broadcast_to(c0, f.shape))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_reduction_is_round_to_nearest():
    x = np.array([-0.5, 0.49, 0.5, 0.51, -1.5, -124.6, 7.5], dtype=np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    assert np.array_equal(n, np.round(x))          # ties to even, like the hardware add
    assert np.all(np.abs(x - n) <= 0.5)


def test_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4, rel.max()   # bf16 P rounds at 2^-9, fp16 at 2^-12


def test_integers_and_tiny_arguments():
    got = exp2_poly2(np.array([0.0, 1.0, -3.0, 8.0], dtype=np.float32)).astype(np.float64)
    assert np.allclose(got, [1.0, 2.0, 0.125, 256.0], rtol=1e-4)
    tiny = exp2_poly2(np.array([-1e30, -200.0, -126.0], dtype=np.float32))
    assert np.all(tiny > 0) and np.all(tiny < 2.0 ** -124)
    assert np.all(np.isfinite(tiny)) and np.all(tiny >= np.finfo(np.float32).tiny)


def test_constants_match_the_fit():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "io_aware_exact_33_b200", "csrc",
                                                       "fit_exp2.py"), "3"],
                         capture_output=True, text=True, check=True).stdout
    fitted = [float(v) for v in re.findall(r"c\d = ([-+]?\d\.\d+e[-+]\d+)f", out)]
    assert np.allclose(fitted, [float(c) for c in coefficients()], rtol=1e-7)
