"""Seeded synthetic inputs for exact attention, shared by the oracle tests,
the GPU parity tests and the benchmark.

This module holds workload shapes and random-number generation only: no
attention arithmetic lives here.  Every tensor is drawn on the CPU from a
``torch.Generator`` seeded with ``manual_seed(seed)``, in the order Q, K, V,
dO, as float32 ``randn`` times ``sigma``, then rounded to the storage dtype
(bf16 or fp16).  The oracle widens exactly these rounded values to float64,
and the GPU receives a bit-identical copy, so both sides see the same inputs.

Layouts follow the ``(batch, seqlen, nheads, headdim)`` convention of the
integration example on "FlashAttention-2：下一代高效注意力机制的突破与实战解析"
(section "实操落地"); K and V carry ``nheads_kv`` heads (grouped-query
attention, named on "FlashAttention 四代演进", section "硬件边界与数据类型限制").
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, mask and input distribution."""

    name: str
    batch: int
    nheads: int
    nheads_kv: int
    seqlen_q: int
    seqlen_k: int
    headdim: int
    causal: bool
    window_left: int = -1
    window_right: int = -1
    dtype: str = "bf16"
    sigma: float = 1.0
    seed: int = 0
    passes: str = "fwd+bwd"
    softmax_scale: Optional[float] = None

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale is not None else 1.0 / math.sqrt(self.headdim)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads attention is measured and checked on.  The seed of each
# is its index in this list.
WORKLOADS: Dict[str, Workload] = {
    "tiny_b1_h2_n128_d64": Workload(
        "tiny_b1_h2_n128_d64", 1, 2, 2, 128, 128, 64, False, seed=0, passes="fwd+bwd"),
    "causal_b2_h32_n8192_d128": Workload(
        "causal_b2_h32_n8192_d128", 2, 32, 32, 8192, 8192, 128, True, seed=1, passes="fwd+bwd"),
    "full_b1_h16_n16384_d128": Workload(
        "full_b1_h16_n16384_d128", 1, 16, 16, 16384, 16384, 128, False, seed=2, passes="fwd+bwd"),
    "gqa_window_b4_h32_kv8_n4096_d128": Workload(
        "gqa_window_b4_h32_kv8_n4096_d128", 4, 32, 8, 4096, 4096, 128, True,
        window_left=1024, window_right=0, seed=3, passes="fwd+bwd"),
    "long_fp16_b1_h8_n65536_d256": Workload(
        "long_fp16_b1_h8_n65536_d256", 1, 8, 8, 65536, 65536, 256, True,
        dtype="fp16", sigma=0.5, seed=4, passes="fwd"),
}


# Workloads of the extra entry points (decode on the CUDA cores, FP8 forward):
# the decode case is 8 sequences each with one new query token against a
# 32,768-token key/value cache (GQA 32/8); the FP8 case is the headline
# causal shape, forward only, its inputs rounded to E4M3 with one scale per
# tensor.
EXTRA_WORKLOADS: Dict[str, Workload] = {
    "decode_b8_h32_kv8_n32768_d128": Workload(
        "decode_b8_h32_kv8_n32768_d128", 8, 32, 8, 1, 32768, 128, True, seed=12, passes="fwd"),
    "fp8_causal_b2_h32_n8192_d128": Workload(
        "fp8_causal_b2_h32_n8192_d128", 2, 32, 32, 8192, 8192, 128, True, seed=13, passes="fwd"),
}


@dataclasses.dataclass(frozen=True)
class VarlenWorkload:
    """Packed variable-length sequences: per-sequence query and key lengths
    (equal here), shared head counts, mask and input distribution."""

    name: str
    lens: tuple
    nheads: int
    nheads_kv: int
    headdim: int
    causal: bool
    window_left: int = -1
    window_right: int = -1
    dtype: str = "bf16"
    sigma: float = 1.0
    seed: int = 0
    passes: str = "fwd+bwd"
    softmax_scale: Optional[float] = None

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale is not None else 1.0 / math.sqrt(self.headdim)


def _uniform_lengths(n: int, lo: int, hi: int, seed: int) -> tuple:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


# A length mix for the packed entry points: 16 causal sequences of 256-1792
# tokens (uniform, seeded), about the token count of the causal N=8192 batch.
VARLEN_WORKLOADS: Dict[str, VarlenWorkload] = {
    "varlen_causal_16seq_h32_d128": VarlenWorkload(
        "varlen_causal_16seq_h32_d128", _uniform_lengths(16, 256, 1792, 11), 32, 32, 128, True,
        seed=11),
}


def make_inputs(w: Workload, with_dout: bool = True, device: str = "cpu"):
    """Draw (q, k, v, dout) for workload ``w``.

    Shapes: q, dout (B, Nq, H, d); k, v (B, Nk, Hkv, d).  Returns CPU tensors
    of the storage dtype unless ``device`` says otherwise (the copy is exact).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    dt = DTYPES[w.dtype]

    def draw(*shape):
        x = torch.randn(*shape, generator=g, dtype=torch.float32)
        return (x * w.sigma).to(dt)

    q = draw(w.batch, w.seqlen_q, w.nheads, w.headdim)
    k = draw(w.batch, w.seqlen_k, w.nheads_kv, w.headdim)
    v = draw(w.batch, w.seqlen_k, w.nheads_kv, w.headdim)
    dout = draw(w.batch, w.seqlen_q, w.nheads, w.headdim) if with_dout else None
    if device != "cpu":
        q, k, v = q.to(device), k.to(device), v.to(device)
        dout = dout.to(device) if dout is not None else None
    return q, k, v, dout


def make_varlen_inputs(lens_q, lens_k, nheads: int, nheads_kv: int, headdim: int,
                       dtype: str = "bf16", sigma: float = 1.0, seed: int = 0,
                       with_dout: bool = True, extra_q: int = 0, extra_k: int = 0):
    """Packed variable-length inputs: sequence b has ``lens_q[b]`` query and
    ``lens_k[b]`` key rows, stored back to back.  Returns (q (Tq, H, d),
    k, v (Tk, Hkv, d), dout (Tq, H, d) or None, cu_q, cu_k) with int32 offsets
    of len(lens) + 1 entries; ``extra_q`` / ``extra_k`` rows past the last
    sequence belong to none.  Drawn like ``make_inputs``: one generator seeded
    with ``seed``, in the order Q, K, V, dO, float32 randn * sigma rounded to
    the storage dtype."""
    if len(lens_q) != len(lens_k):
        raise ValueError("lens_q and lens_k must have one entry per sequence")
    cu_q = [0]
    cu_k = [0]
    for a, b in zip(lens_q, lens_k):
        cu_q.append(cu_q[-1] + int(a))
        cu_k.append(cu_k[-1] + int(b))
    tq, tk = cu_q[-1] + int(extra_q), cu_k[-1] + int(extra_k)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    dt = DTYPES[dtype]

    def draw(*shape):
        return (torch.randn(*shape, generator=g, dtype=torch.float32) * sigma).to(dt)

    q = draw(tq, nheads, headdim)
    k = draw(tk, nheads_kv, headdim)
    v = draw(tk, nheads_kv, headdim)
    dout = draw(tq, nheads, headdim) if with_dout else None
    return (q, k, v, dout, torch.tensor(cu_q, dtype=torch.int32),
            torch.tensor(cu_k, dtype=torch.int32))


def sample_rows(n: int, count: int, seed: int, must=()) -> torch.Tensor:
    """A sorted, duplicate-free set of row indices in [0, n): the first and
    last rows, any ``must`` rows, and ``count`` more drawn from ``seed``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7919)
    picks = set(int(i) for i in must if 0 <= int(i) < n)
    picks.update({0, n - 1} if n > 0 else set())
    if n > 0 and count > 0:
        picks.update(torch.randint(0, n, (count,), generator=g).tolist())
    return torch.tensor(sorted(picks), dtype=torch.int64)
