"""Python access to the float64 CPU attention oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The CUDA
library and its Python binding never import it, and it never imports them.

Every function takes torch tensors in the storage dtype (bf16/fp16/fp32/fp64,
any device), widens them exactly to float64 on the CPU and returns float64
numpy arrays.  See ``attn_oracle.c`` for what is computed and which passages
of the pages each step follows.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class OracleParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen_q", ctypes.c_int64),
        ("seqlen_k", ctypes.c_int64),
        ("nheads", ctypes.c_int64),
        ("nheads_kv", ctypes.c_int64),
        ("headdim", ctypes.c_int64),
        ("softmax_scale", ctypes.c_double),
        ("causal", ctypes.c_int64),
        ("window_left", ctypes.c_int64),
        ("window_right", ctypes.c_int64),
        ("alibi_slopes", ctypes.c_void_p),
        ("dropout_threshold", ctypes.c_int64),
        ("dropout_seed", ctypes.c_uint64),
        ("dropout_offset", ctypes.c_int64),
        ("batch_base", ctypes.c_int64),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (float64, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Oracle:
    """Bindings to one compiled copy of the oracle (the default build, or a
    variant compiled elsewhere, as the mutation tests do)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        d = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.POINTER(ctypes.c_int64)
        P = ctypes.POINTER(OracleParams)
        lib.oracle_attn_fwd.argtypes = [P, d, d, d, d, d]
        lib.oracle_attn_fwd_rows.argtypes = [P, d, d, d, i64, ctypes.c_int64, d, d]
        lib.oracle_attn_bwd.argtypes = [P, d, d, d, d, d, d, d]
        lib.oracle_attn_bwd_rows.argtypes = [P, d, d, d, d, i64, ctypes.c_int64, d,
                                             i64, ctypes.c_int64, d, d]
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_rows, lib.oracle_attn_bwd,
                  lib.oracle_attn_bwd_rows):
            f.restype = ctypes.c_int
        lib.oracle_attn_merge.argtypes = [ctypes.c_int64] * 5 + [d, d, d, d]
        lib.oracle_attn_merge.restype = ctypes.c_int
        u32p = ctypes.POINTER(ctypes.c_uint32)
        lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_dropout_keep.argtypes = [P, ctypes.POINTER(ctypes.c_uint8)]
        lib.oracle_dropout_keep.restype = ctypes.c_int
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_quantize.argtypes = [d, ctypes.c_int64, ctypes.c_double,
                                             ctypes.POINTER(ctypes.c_uint8)]
        lib.oracle_e4m3_quantize.restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        self.lib = lib
        self.path = lib_path

    def attention_fwd(self, q, k, v, softmax_scale=None, causal=False, window_left=-1,
                      window_right=-1, alibi_slopes=None, dropout_p=0.0, dropout_seed=0,
                      dropout_offset=0):
        """O (B, Nq, H, d) and LSE (B, H, Nq), float64.  ``alibi_slopes``
        (H values, optional) adds -slope_h * |i + Nk - Nq - j| to the scores."""
        return self.attention_fwd_rows(q, k, v, None, softmax_scale, causal, window_left,
                                       window_right, alibi_slopes, dropout_p, dropout_seed,
                                       dropout_offset)

    def attention_fwd_rows(self, q, k, v, rows, softmax_scale=None, causal=False,
                           window_left=-1, window_right=-1, alibi_slopes=None, dropout_p=0.0,
                           dropout_seed=0, dropout_offset=0, batch_base=0):
        """O and LSE for the query positions ``rows`` only (all rows if None):
        O (B, len(rows), H, d), LSE (B, H, len(rows))."""
        qa, ka, va = _f64(q), _f64(k), _f64(v)
        p, _keep = _params(qa, ka, softmax_scale, causal, window_left, window_right, alibi_slopes,
                           dropout_p, dropout_seed, dropout_offset, batch_base)
        B, Nq, H, d = qa.shape
        if rows is None:
            n, rp = Nq, None
        else:
            ra = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            n, rp = ra.shape[0], _ptr(ra, ctypes.c_int64)
        o = np.zeros((B, n, H, d), dtype=np.float64)
        lse = np.zeros((B, H, n), dtype=np.float64)
        rc = self.lib.oracle_attn_fwd_rows(ctypes.byref(p), _ptr(qa), _ptr(ka), _ptr(va), rp,
                                           ctypes.c_int64(n), _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle_attn_fwd_rows rejected its arguments")
        return o, lse

    def attention_bwd(self, q, k, v, dout, softmax_scale=None, causal=False, window_left=-1,
                      window_right=-1, alibi_slopes=None, dropout_p=0.0, dropout_seed=0,
                      dropout_offset=0, batch_base=0):
        """dQ (B, Nq, H, d), dK and dV (B, Nk, Hkv, d), float64."""
        qa, ka, va, da = _f64(q), _f64(k), _f64(v), _f64(dout)
        p, _keep = _params(qa, ka, softmax_scale, causal, window_left, window_right, alibi_slopes,
                           dropout_p, dropout_seed, dropout_offset, batch_base)
        dq = np.zeros_like(qa)
        dk = np.zeros_like(ka)
        dv = np.zeros_like(va)
        rc = self.lib.oracle_attn_bwd(ctypes.byref(p), _ptr(qa), _ptr(ka), _ptr(va), _ptr(da),
                                      _ptr(dq), _ptr(dk), _ptr(dv))
        if rc != 0:
            raise ValueError("oracle_attn_bwd rejected its arguments")
        return dq, dk, dv

    def attention_bwd_rows(self, q, k, v, dout, qrows, krows, softmax_scale=None, causal=False,
                           window_left=-1, window_right=-1, alibi_slopes=None, dropout_p=0.0,
                           dropout_seed=0, dropout_offset=0):
        """dQ at query positions ``qrows`` (B, nq, H, d) and dK, dV at key
        positions ``krows`` (B, nk, Hkv, d), float64."""
        qa, ka, va, da = _f64(q), _f64(k), _f64(v), _f64(dout)
        p, _keep = _params(qa, ka, softmax_scale, causal, window_left, window_right, alibi_slopes,
                           dropout_p, dropout_seed, dropout_offset)
        qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64))
        kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int64))
        B, _, H, d = qa.shape
        Hkv = ka.shape[2]
        dq = np.zeros((B, qr.shape[0], H, d))
        dk = np.zeros((B, kr.shape[0], Hkv, d))
        dv = np.zeros((B, kr.shape[0], Hkv, d))
        rc = self.lib.oracle_attn_bwd_rows(ctypes.byref(p), _ptr(qa), _ptr(ka), _ptr(va),
                                           _ptr(da), _ptr(qr, ctypes.c_int64),
                                           ctypes.c_int64(qr.shape[0]), _ptr(dq),
                                           _ptr(kr, ctypes.c_int64), ctypes.c_int64(kr.shape[0]),
                                           _ptr(dk), _ptr(dv))
        if rc != 0:
            raise ValueError("oracle_attn_bwd_rows rejected its arguments")
        return dq, dk, dv


    # Packed variable-length sequences: each sequence is its own attention
    # problem (the varlen interface of "FlashAttention-2：下一代高效注意力机制
    # 的突破与实战解析", section "实操落地"), so the oracle runs the dense
    # definition on every sequence's rows.
    def attention_fwd_varlen(self, q, k, v, cu_q, cu_k, softmax_scale=None, causal=False,
                             window_left=-1, window_right=-1, alibi_slopes=None, dropout_p=0.0,
                             dropout_seed=0, dropout_offset=0):
        """q (Tq, H, d), k, v (Tk, Hkv, d), offsets cu_q, cu_k (batch + 1):
        O (Tq, H, d) and LSE (H, Tq), float64."""
        qa, ka, va = _f64(q), _f64(k), _f64(v)
        cq, ck = _offsets(cu_q), _offsets(cu_k)
        Tq, H, d = qa.shape
        o = np.zeros((Tq, H, d))
        lse = np.zeros((H, Tq))
        for b in range(len(cq) - 1):
            q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
            if q1 == q0:
                continue
            ob, lb = self.attention_fwd_rows(qa[None, q0:q1], ka[None, k0:k1], va[None, k0:k1],
                                             None, softmax_scale, causal, window_left,
                                             window_right, alibi_slopes, dropout_p, dropout_seed,
                                             dropout_offset, batch_base=b)
            o[q0:q1] = ob[0]
            lse[:, q0:q1] = lb[0]
        return o, lse

    def attention_bwd_varlen(self, q, k, v, dout, cu_q, cu_k, softmax_scale=None, causal=False,
                             window_left=-1, window_right=-1, alibi_slopes=None, dropout_p=0.0,
                             dropout_seed=0, dropout_offset=0):
        """dQ (Tq, H, d), dK and dV (Tk, Hkv, d), float64, per sequence."""
        qa, ka, va, da = _f64(q), _f64(k), _f64(v), _f64(dout)
        cq, ck = _offsets(cu_q), _offsets(cu_k)
        dq, dk, dv = np.zeros_like(qa), np.zeros_like(ka), np.zeros_like(va)
        for b in range(len(cq) - 1):
            q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
            if q1 == q0 or k1 == k0:
                continue
            g = self.attention_bwd(qa[None, q0:q1], ka[None, k0:k1], va[None, k0:k1],
                                   da[None, q0:q1], softmax_scale, causal, window_left,
                                   window_right, alibi_slopes, dropout_p, dropout_seed,
                                   dropout_offset, batch_base=b)
            dq[q0:q1], dk[k0:k1], dv[k0:k1] = g[0][0], g[1][0], g[2][0]
        return dq, dk, dv


    def philox4x32_10(self, counter, key):
        """The generator's four output words for a counter of four 32-bit
        words and a key of two."""
        c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in counter])
        k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        out = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, k, out)
        return list(out)

    def dropout_keep(self, batch, nheads, seqlen_q, seqlen_k, dropout_p, dropout_seed=0,
                     dropout_offset=0, batch_base=0):
        """The keep mask (B, H, Nq, Nk) uint8 of the dropout contract: 1 kept,
        0 dropped (independent of the attention mask)."""
        p = OracleParams(batch, seqlen_q, seqlen_k, nheads, 1, 1, 1.0, 0, -1, -1, None,
                         dropout_threshold(dropout_p), int(dropout_seed) & (2 ** 64 - 1),
                         int(dropout_offset) & 0xFFFFFFFF, int(batch_base))
        keep = np.zeros((batch, nheads, seqlen_q, seqlen_k), dtype=np.uint8)
        rc = self.lib.oracle_dropout_keep(ctypes.byref(p),
                                          keep.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
        if rc != 0:
            raise ValueError("oracle_dropout_keep rejected its arguments")
        return keep

    def e4m3_quantize(self, x, scale=1.0):
        """E4M3 codes (uint8, x's shape) of x / scale: round to nearest even,
        saturating at +-448."""
        xa = _f64(x)
        codes = np.zeros(xa.shape, dtype=np.uint8)
        self.lib.oracle_e4m3_quantize(_ptr(xa), ctypes.c_int64(xa.size), ctypes.c_double(scale),
                                      codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
        return codes

    def e4m3_dequantize(self, codes, scale=1.0):
        """float64 values scale * e4m3(code) of uint8 codes."""
        table = np.array([self.lib.oracle_e4m3_value(c) for c in range(256)])
        return table[np.asarray(codes, dtype=np.uint8)] * scale

    def attention_merge(self, o_parts, lse_parts):
        """Merge partial results over disjoint key sets: o_parts (S, B, Nq,
        H, d), lse_parts (S, B, H, Nq) -> O (B, Nq, H, d), LSE (B, H, Nq),
        float64."""
        op, lp = _f64(o_parts), _f64(lse_parts)
        S, B, Nq, H, d = op.shape
        if lp.shape != (S, B, H, Nq):
            raise ValueError("lse_parts must be (splits, batch, nheads, seqlen_q)")
        o = np.zeros((B, Nq, H, d))
        lse = np.zeros((B, H, Nq))
        rc = self.lib.oracle_attn_merge(S, B, Nq, H, d, _ptr(op), _ptr(lp), _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle_attn_merge rejected its arguments")
        return o, lse


def default() -> Oracle:
    """The oracle built from ``attn_oracle.c`` beside this file."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def num_threads() -> int:
    return int(default().lib.oracle_num_threads())


def set_num_threads(n: int) -> None:
    default().lib.oracle_set_num_threads(int(n))


def _f64(t) -> np.ndarray:
    import torch
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float64)
    return np.ascontiguousarray(t.detach().to("cpu", torch.float64).numpy())


def _offsets(cu) -> list:
    import torch
    if isinstance(cu, torch.Tensor):
        cu = cu.detach().cpu().tolist()
    cu = [int(x) for x in cu]
    if not cu or cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("sequence offsets must start at 0 and not decrease")
    return cu


def _ptr(a: np.ndarray, ty=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ty))


def dropout_threshold(dropout_p: float) -> int:
    """The drop threshold t = round(256 p) of the dropout contract (an
    element is dropped iff its random byte is below t); p' = t / 256 is the
    rate actually applied.  p must lie in [0, 1) with t <= 255."""
    p = float(dropout_p)
    t = int(math.floor(256.0 * p + 0.5))
    if not (0.0 <= p < 1.0) or t > 255:
        raise ValueError(f"dropout_p must be in [0, 255.5/256), got {dropout_p}")
    return t


def _params(q, k, softmax_scale, causal, window_left, window_right, alibi_slopes=None,
            dropout_p=0.0, dropout_seed=0, dropout_offset=0, batch_base=0):
    """The C parameter block and the slopes array it points to (keep both
    alive for the call)."""
    B, Nq, H, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if Bk != B or dk != d or H % Hkv != 0:
        raise ValueError("inconsistent shapes")
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    slopes = None
    if alibi_slopes is not None:
        slopes = np.ascontiguousarray(
            _f64(alibi_slopes if hasattr(alibi_slopes, "shape") else np.asarray(alibi_slopes))
            .reshape(-1))
        if slopes.shape[0] != H:
            raise ValueError("alibi_slopes needs one slope per query head")
    ptr = slopes.ctypes.data if slopes is not None else None
    return OracleParams(B, Nq, Nk, H, Hkv, d, scale, int(bool(causal)),
                        int(window_left), int(window_right), ptr, dropout_threshold(dropout_p),
                        int(dropout_seed) & (2 ** 64 - 1), int(dropout_offset) & 0xFFFFFFFF,
                        int(batch_base)), slopes


def attention_fwd(*a, **kw):
    return default().attention_fwd(*a, **kw)


def attention_fwd_rows(*a, **kw):
    return default().attention_fwd_rows(*a, **kw)


def attention_bwd(*a, **kw):
    return default().attention_bwd(*a, **kw)


def attention_bwd_rows(*a, **kw):
    return default().attention_bwd_rows(*a, **kw)


def attention_fwd_varlen(*a, **kw):
    return default().attention_fwd_varlen(*a, **kw)


def attention_bwd_varlen(*a, **kw):
    return default().attention_bwd_varlen(*a, **kw)


def attention_merge(*a, **kw):
    return default().attention_merge(*a, **kw)


def philox4x32_10(*a, **kw):
    return default().philox4x32_10(*a, **kw)


def dropout_keep(*a, **kw):
    return default().dropout_keep(*a, **kw)


def e4m3_quantize(*a, **kw):
    return default().e4m3_quantize(*a, **kw)


def e4m3_dequantize(*a, **kw):
    return default().e4m3_dequantize(*a, **kw)
