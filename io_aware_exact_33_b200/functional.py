"""Differentiable attention calls for PyTorch models.

``flash_attn_func`` / ``flash_attn_varlen_func`` take the arguments of the
integration example on "FlashAttention-2：下一代高效注意力机制的突破与实战解析"
(section "实操落地": ``(batch, seqlen, nheads, headdim)`` fp16/bf16 tensors,
``causal``, ``softmax_scale``; the FAQ adds ``alibi_slopes`` and the
variable-length form) and run the library's forward, saving Q, K, V, O and
the log-sum-exp; the backward pass calls the library's backward.  The LSE,
returned on request, is not differentiable.  With ``dropout_p`` > 0 the
drop decisions follow the library's generator contract; the seed is drawn
from torch's default generator (so ``torch.manual_seed`` makes a run
repeatable) unless given, and the backward reuses the forward's seed and
offset.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

import io_aware_exact_33_b200 as _lib


def _window(window_size) -> Tuple[int, int]:
    wl, wr = (int(window_size[0]), int(window_size[1]))
    if wl < -1 or wr < -1:
        raise ValueError("window_size entries must be >= -1 (-1 = unbounded)")
    return wl, wr


def _dropout(dropout_p: float, dropout_seed):
    """(p, seed, offset) for one call."""
    p = float(dropout_p)
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout_p must be in [0, 1)")
    if p == 0.0:
        return 0.0, 0, 0
    if dropout_seed is None:
        dropout_seed = int(torch.randint(0, 2 ** 62, (1,)).item())
    return p, int(dropout_seed), 0


class _Attn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, softmax_scale, causal, wl, wr, alibi_slopes, drop):
        o, lse = _lib.attn_fwd(q, k, v, softmax_scale, causal, wl, wr, alibi_slopes=alibi_slopes,
                               dropout_p=drop[0], dropout_seed=drop[1], dropout_offset=drop[2])
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.alibi_slopes = alibi_slopes
        ctx.drop = drop
        ctx.args = (softmax_scale, causal, wl, wr)
        ctx.mark_non_differentiable(lse)
        return o, lse

    @staticmethod
    def backward(ctx, do, _dlse):
        q, k, v, o, lse = ctx.saved_tensors
        p, seed, off = ctx.drop
        dq, dk, dv = _lib.attn_bwd(q, k, v, o, lse, do.contiguous(), *ctx.args,
                                   alibi_slopes=ctx.alibi_slopes, dropout_p=p, dropout_seed=seed,
                                   dropout_offset=off)
        return dq, dk, dv, None, None, None, None, None, None


class _AttnVarlen(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, softmax_scale, causal, wl, wr,
                alibi_slopes, drop):
        o, lse = _lib.attn_fwd_varlen(q, k, v, cu_q, cu_k, max_q, max_k, softmax_scale, causal,
                                      wl, wr, alibi_slopes=alibi_slopes, dropout_p=drop[0],
                                      dropout_seed=drop[1], dropout_offset=drop[2])
        ctx.save_for_backward(q, k, v, o, lse, cu_q, cu_k)
        ctx.alibi_slopes = alibi_slopes
        ctx.drop = drop
        ctx.args = (max_q, max_k, softmax_scale, causal, wl, wr)
        ctx.mark_non_differentiable(lse)
        return o, lse

    @staticmethod
    def backward(ctx, do, _dlse):
        q, k, v, o, lse, cu_q, cu_k = ctx.saved_tensors
        p, seed, off = ctx.drop
        dq, dk, dv = _lib.attn_bwd_varlen(q, k, v, o, lse, do.contiguous(), cu_q, cu_k, *ctx.args,
                                          alibi_slopes=ctx.alibi_slopes, dropout_p=p,
                                          dropout_seed=seed, dropout_offset=off)
        return dq, dk, dv, None, None, None, None, None, None, None, None, None, None


def flash_attn_func(q, k, v, dropout_p: float = 0.0, softmax_scale: Optional[float] = None,
                    causal: bool = False, window_size=(-1, -1), alibi_slopes=None,
                    return_lse: bool = False, dropout_seed: Optional[int] = None):
    """softmax(q k^T * scale + bias + mask) v for q (B, Nq, H, d), k and v
    (B, Nk, Hkv, d), differentiable in q, k and v.  ``window_size =
    (left, right)`` bounds the visible keys of query i to [i + off - left,
    i + off + right] (-1 = unbounded, off = Nk - Nq).  Returns ``out`` (B, Nq,
    H, d), or ``(out, lse)`` with lse (B, H, Nq) float32 when ``return_lse``."""
    drop = _dropout(dropout_p, dropout_seed)
    wl, wr = _window(window_size)
    out, lse = _Attn.apply(q, k, v, softmax_scale, bool(causal), wl, wr, alibi_slopes, drop)
    return (out, lse) if return_lse else out


def flash_attn_varlen_func(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                           max_seqlen_k: int, dropout_p: float = 0.0,
                           softmax_scale: Optional[float] = None, causal: bool = False,
                           window_size=(-1, -1), alibi_slopes=None, return_lse: bool = False,
                           dropout_seed: Optional[int] = None):
    """Packed variable-length form: q (total_q, H, d), k and v (total_k, Hkv,
    d), int32 offsets of batch + 1 entries.  Returns ``out`` (total_q, H, d),
    or ``(out, lse)`` with lse (H, total_q) float32 when ``return_lse``."""
    drop = _dropout(dropout_p, dropout_seed)
    wl, wr = _window(window_size)
    out, lse = _AttnVarlen.apply(q, k, v, cu_seqlens_q, cu_seqlens_k, int(max_seqlen_q),
                                 int(max_seqlen_k), softmax_scale, bool(causal), wl, wr,
                                 alibi_slopes, drop)
    return (out, lse) if return_lse else out
