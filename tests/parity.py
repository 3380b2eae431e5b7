"""Comparison helpers: the CUDA library against the float64 oracle.

Tolerances (stated by the task's correctness target for inputs ~N(0,1) with
fp32 accumulation):
  * O:   |O - O_ref| <= 1e-2 + half an ulp of the output dtype at |O_ref|.
         The second term is the rounding of the exact value to bf16/fp16,
         which no kernel can avoid (for |O| in [4, 8) a bf16 half-ulp is
         0.0156); the raw maximum error and that floor are reported too.
  * LSE: |LSE - LSE_ref| <= 1e-3 on finite entries; -inf entries must match.
  * dQ, dK, dV: ||dX - dX_ref||_F / ||dX_ref||_F <= 1e-2.
"""
from __future__ import annotations

import math

import numpy as np
import torch

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_REL_TOL = 1e-2

_MANT_BITS = {torch.bfloat16: 7, torch.float16: 10}


def half_ulp(ref: np.ndarray, dtype) -> np.ndarray:
    """Half the spacing of ``dtype`` numbers at |ref| (normal range)."""
    mb = _MANT_BITS[dtype]
    a = np.abs(ref)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 0.5 * np.exp2(e - mb)


def check_o(o_gpu: torch.Tensor, o_ref: np.ndarray, what: str):
    og = o_gpu.detach().to("cpu", torch.float64).numpy()
    err = np.abs(og - o_ref)
    bound = O_TOL + half_ulp(o_ref, o_gpu.dtype)
    assert np.isfinite(og).all(), f"{what}: non-finite output"
    worst = np.unravel_index(np.argmax(err - bound), err.shape) if err.size else None
    floor = np.abs(torch.from_numpy(o_ref).to(o_gpu.dtype).double().numpy() - o_ref)
    info = (f"{what}: max|O-O_ref|={err.max() if err.size else 0:.3e} "
            f"rounding floor={floor.max() if floor.size else 0:.3e}")
    assert (err <= bound).all(), f"{info}; worst at {worst}: gpu={og[worst]} ref={o_ref[worst]}"
    return float(err.max()) if err.size else 0.0


def check_o_derived(o_gpu: torch.Tensor, o_ref: np.ndarray, pabs_ref: np.ndarray, what: str):
    """Tolerance derived from the kernel's arithmetic, for inputs outside the
    N(0,1) regime the flat 1e-2 is stated for: P enters the P.V product as a
    16-bit value (relative rounding <= 2^-8 for bf16, 2^-11 for fp16), so
    |dO| <= rel * sum_j P_ij |V_jc| (= ``pabs_ref``, the oracle's output on
    |V|), plus the output rounding and 1e-3 of fp32 slack."""
    og = o_gpu.detach().to("cpu", torch.float64).numpy()
    rel = 2.0 ** -8 if o_gpu.dtype == torch.bfloat16 else 2.0 ** -11
    bound = rel * pabs_ref + half_ulp(o_ref, o_gpu.dtype) + 1e-3
    err = np.abs(og - o_ref)
    assert np.isfinite(og).all(), f"{what}: non-finite output"
    assert (err <= bound).all(), f"{what}: max excess {np.max(err - bound):.3e}"
    return float(err.max())


def check_lse(lse_gpu: torch.Tensor, lse_ref: np.ndarray, what: str):
    lg = lse_gpu.detach().to("cpu", torch.float64).numpy()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lg), fin), f"{what}: -inf pattern differs"
    assert np.all(lg[~fin] == lse_ref[~fin]), f"{what}: infinite entries differ"
    err = np.abs(lg[fin] - lse_ref[fin]).max() if fin.any() else 0.0
    assert err <= LSE_TOL, f"{what}: max|LSE-LSE_ref|={err:.3e}"
    return float(err)


def rel_fro(x_gpu: torch.Tensor, x_ref: np.ndarray) -> float:
    xg = x_gpu.detach().to("cpu", torch.float64).numpy()
    assert np.isfinite(xg).all(), "non-finite gradient"
    den = np.linalg.norm(x_ref)
    num = np.linalg.norm(xg - x_ref)
    return float(num / den) if den > 0 else float(num)


def check_grad(x_gpu, x_ref, what):
    r = rel_fro(x_gpu, x_ref)
    assert r <= GRAD_REL_TOL, f"{what}: relative Frobenius error {r:.3e}"
    return r
