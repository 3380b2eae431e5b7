"""The FMA-pipe 2^x used for part of the softmax exponentials: the constants
in sm100.cuh, evaluated the way the kernel does (float32, floor range
reduction, Horner, exponent-field add), agree with 2^x to the stated bound,
give exactly 0 for masked (-inf) and tiny arguments, and match the fit."""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "io_aware_exact_33_b200", "csrc", "sm100.cuh")


def coefficients():
    body = open(HDR).read().split("float exp2_poly(float x) {")[1].split("}")[0]
    nums = [float(x.rstrip("f")) for x in re.findall(r"[-+]?\d\.\d+e[-+]\d+f", body)]
    # fmaf(c3, f, c2); fmaf(p, f, c1); fmaf(p, f, c0)
    c3, c2, c1, c0 = nums
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def exp2_poly(x):
    c0, c1, c2, c3 = coefficients()
    x = np.asarray(x, dtype=np.float32)
    xc = np.maximum(x, np.float32(-127.0))
    nf = np.floor(xc)
    f = (xc - nf).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (nf.astype(np.int32) << 23)
    out = bits.view(np.float32)
    return np.where(x < -126.0, np.float32(0.0), out)


def test_relative_error_bound():
    # down to -125: at -126 the result is subnormal and the exponent-field add
    # loses bits (such a P contributes nothing to the output)
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4, rel.max()   # bf16 P rounds at 2^-9, fp16 at 2^-12


def test_masked_and_tiny_arguments_give_zero():
    assert np.all(exp2_poly([-np.inf, -1e30, -127.0, -126.5]) == 0.0)
    assert exp2_poly([0.0])[0] > 0.9999 and abs(exp2_poly([8.0])[0] - 256.0) < 256 * 1e-4


def test_constants_match_the_fit():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "io_aware_exact_33_b200", "csrc",
                                                       "fit_exp2.py"), "3"],
                         capture_output=True, text=True, check=True).stdout
    fitted = [float(v) for v in re.findall(r"c\d = ([-+]?\d\.\d+e[-+]\d+)f", out)]
    assert np.allclose(fitted, [float(c) for c in coefficients()], rtol=1e-7)
