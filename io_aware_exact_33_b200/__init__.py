"""Python binding of libattn.so, the sm_100a exact-attention library.

Argument marshalling only: torch supplies device memory and the current CUDA
stream, and every step of the attention computation runs in the library's
kernels.  The entry points carry the C ABI's names (``include/attn.h``):
``attn_fwd``, ``attn_bwd``, ``attn_fwd_workspace_size``,
``attn_bwd_workspace_size``, ``attn_check_params``, ``attn_status_string``,
``attn_get_device_status`` and ``attn_version``.

There is no fallback: if the compiled library is missing, the first call
raises an ImportError that says how to build it.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

ATTN_BF16, ATTN_FP16 = 0, 1
STATUS = {
    0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED_HEADDIM",
    3: "ATTN_ERR_UNSUPPORTED_DTYPE", 4: "ATTN_ERR_MISALIGNED", 5: "ATTN_ERR_WORKSPACE_TOO_SMALL",
    6: "ATTN_ERR_CUDA", 7: "ATTN_ERR_TIMEOUT", 8: "ATTN_ERR_DEVICE_STATUS",
}
EXPORTED = ("attn_fwd", "attn_bwd", "attn_bwd_prepare", "attn_bwd_accumulate", "attn_bwd_finalize",
            "attn_fwd_workspace_size", "attn_bwd_workspace_size", "attn_check_params",
            "attn_status_string", "attn_get_device_status", "attn_version", "attn_bwd_noalloc",
            "attn_selftest_bounded_wait", "attn_check_varlen_params", "attn_fwd_varlen",
            "attn_fwd_e4m3", "attn_fwd_decode", "attn_fwd_decode_workspace_size",
            "attn_bwd_varlen_workspace_size", "attn_bwd_varlen", "attn_merge",
            "attn_bwd_accumulate_f32", "attn_f32_to_16")


class AttnParams(ctypes.Structure):
    """Mirror of ``attn_params`` in include/attn.h."""
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("seqlen_q", ctypes.c_int32),
        ("seqlen_k", ctypes.c_int32),
        ("nheads", ctypes.c_int32),
        ("nheads_kv", ctypes.c_int32),
        ("headdim", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("causal", ctypes.c_int32),
        ("window_left", ctypes.c_int32),
        ("window_right", ctypes.c_int32),
        ("alibi_slopes", ctypes.c_void_p),
        ("dropout_p", ctypes.c_float),
        ("dropout_offset", ctypes.c_uint32),
        ("dropout_seed", ctypes.c_uint64),
        ("pos_offset", ctypes.c_int32),
        ("reserved0", ctypes.c_int32),
    ]


class AttnVarlenParams(ctypes.Structure):
    """Mirror of ``attn_varlen_params`` in include/attn.h."""
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("total_q", ctypes.c_int32),
        ("total_k", ctypes.c_int32),
        ("max_seqlen_q", ctypes.c_int32),
        ("max_seqlen_k", ctypes.c_int32),
        ("nheads", ctypes.c_int32),
        ("nheads_kv", ctypes.c_int32),
        ("headdim", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("causal", ctypes.c_int32),
        ("window_left", ctypes.c_int32),
        ("window_right", ctypes.c_int32),
        ("alibi_slopes", ctypes.c_void_p),
        ("dropout_p", ctypes.c_float),
        ("dropout_offset", ctypes.c_uint32),
        ("dropout_seed", ctypes.c_uint64),
    ]


class AttnMergeParams(ctypes.Structure):
    """Mirror of ``attn_merge_params`` in include/attn.h."""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("splits", "batch", "seqlen_q", "nheads", "headdim", "dtype")]


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({attn_status_string(status)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m io_aware_exact_33_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, P = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(AttnParams)
    lib.attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.attn_fwd.restype = ctypes.c_int
    lib.attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.attn_bwd.restype = ctypes.c_int
    lib.attn_bwd_prepare.argtypes = [P, vp, vp, vp, vp, sz, vp]
    lib.attn_bwd_prepare.restype = ctypes.c_int
    lib.attn_bwd_accumulate.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.attn_bwd_accumulate.restype = ctypes.c_int
    lib.attn_bwd_finalize.argtypes = [P, vp, vp, sz, vp]
    lib.attn_bwd_finalize.restype = ctypes.c_int
    lib.attn_bwd_accumulate_f32.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.attn_bwd_accumulate_f32.restype = ctypes.c_int
    lib.attn_f32_to_16.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_int, vp]
    lib.attn_f32_to_16.restype = ctypes.c_int
    lib.attn_bwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.attn_bwd_noalloc.restype = ctypes.c_int
    lib.attn_fwd_workspace_size.argtypes = [P]
    lib.attn_fwd_workspace_size.restype = sz
    lib.attn_bwd_workspace_size.argtypes = [P]
    lib.attn_bwd_workspace_size.restype = sz
    lib.attn_check_params.argtypes = [P, ctypes.c_int]
    lib.attn_check_params.restype = ctypes.c_int
    lib.attn_status_string.argtypes = [ctypes.c_int]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.attn_get_device_status.restype = ctypes.c_int
    VP = ctypes.POINTER(AttnVarlenParams)
    lib.attn_check_varlen_params.argtypes = [VP, ctypes.c_int]
    lib.attn_check_varlen_params.restype = ctypes.c_int
    lib.attn_bwd_varlen_workspace_size.argtypes = [VP]
    lib.attn_bwd_varlen_workspace_size.restype = sz
    lib.attn_fwd_varlen.argtypes = [VP, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.attn_fwd_varlen.restype = ctypes.c_int
    lib.attn_bwd_varlen.argtypes = [VP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.attn_bwd_varlen.restype = ctypes.c_int
    lib.attn_merge.argtypes = [ctypes.POINTER(AttnMergeParams), vp, vp, vp, vp, vp]
    lib.attn_merge.restype = ctypes.c_int
    lib.attn_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp, vp]
    lib.attn_selftest_bounded_wait.restype = ctypes.c_int
    lib.attn_version.argtypes = []
    lib.attn_version.restype = ctypes.c_char_p
    return lib


_handle = None


class _Lazy:
    """Loads libattn.so on first use; raises ImportError if it was not built."""

    def __getattr__(self, name):
        global _handle
        if _handle is None:
            _handle = _load()
        return getattr(_handle, name)


_lib = _Lazy()


def make_params(batch, seqlen_q, seqlen_k, nheads, nheads_kv, headdim, dtype=ATTN_BF16,
                softmax_scale=None, causal=False, window_left=-1, window_right=-1,
                alibi_slopes=None, dropout_p=0.0, dropout_seed=0, dropout_offset=0,
                pos_offset=0) -> AttnParams:
    """``alibi_slopes``: None, or the device address (int) of nheads float32
    slopes.  Dropout: rate ``dropout_p`` (applied as round(256 p) / 256), the
    generator's 64-bit seed and 32-bit offset (see include/attn.h).
    ``pos_offset`` moves the query rows relative to the keys for the masks and
    the positional bias (0 = bottom-right alignment; include/attn.h)."""
    scale = 1.0 / math.sqrt(headdim) if softmax_scale is None else float(softmax_scale)
    return AttnParams(int(batch), int(seqlen_q), int(seqlen_k), int(nheads), int(nheads_kv),
                      int(headdim), int(dtype), scale, int(bool(causal)), int(window_left),
                      int(window_right), alibi_slopes, float(dropout_p),
                      int(dropout_offset) & 0xFFFFFFFF, int(dropout_seed) & (2 ** 64 - 1),
                      int(pos_offset), 0)


def _slopes_ptr(alibi_slopes, nheads, device):
    """Device address of a (nheads,) float32 CUDA tensor of slopes, or None."""
    if alibi_slopes is None:
        return None
    import torch
    if (not isinstance(alibi_slopes, torch.Tensor) or not alibi_slopes.is_cuda or
            alibi_slopes.dtype != torch.float32 or not alibi_slopes.is_contiguous() or
            alibi_slopes.numel() != nheads or alibi_slopes.device != device):
        raise ValueError("alibi_slopes must be a contiguous float32 tensor of nheads values "
                         "on the inputs' device")
    return alibi_slopes.data_ptr()


def attn_status_string(status: int) -> str:
    return _lib.attn_status_string(int(status)).decode()


def attn_version() -> str:
    return _lib.attn_version().decode()


def attn_check_params(p: AttnParams, pass_: int = 0) -> int:
    return int(_lib.attn_check_params(ctypes.byref(p), int(pass_)))


def attn_fwd_workspace_size(p: AttnParams) -> int:
    return int(_lib.attn_fwd_workspace_size(ctypes.byref(p)))


def attn_bwd_workspace_size(p: AttnParams) -> int:
    return int(_lib.attn_bwd_workspace_size(ctypes.byref(p)))


def attn_get_device_status(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream().cuda_stream if stream is None else int(stream)
    code = ctypes.c_int(0)
    st = _lib.attn_get_device_status(ctypes.c_void_p(s), ctypes.byref(code))
    if st != 0:
        raise AttnError(st, "attn_get_device_status")
    return int(code.value)


def attn_selftest_bounded_wait(wait_limit_us: int, result=None, stream=None) -> None:
    """Launch the bounded-wait self-test: a kernel whose two waiters give up
    after ``wait_limit_us`` microseconds on a barrier nothing arrives at.
    ``result`` (optional) is a CUDA int32 tensor of 2 elements receiving 1 per
    waiter that gave up.  Afterwards ``attn_get_device_status()`` returns
    ATTN_ERR_TIMEOUT.  Raises AttnError on a bad limit or a launch failure."""
    rp = None
    if result is not None:
        if result.numel() < 2 or not result.is_cuda or result.dtype.itemsize != 4:
            raise ValueError("result must be a CUDA int32 tensor with 2 elements")
        rp = ctypes.c_void_p(result.data_ptr())
    st = _lib.attn_selftest_bounded_wait(ctypes.c_uint(int(wait_limit_us) & 0xffffffff), rp,
                                         _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_selftest_bounded_wait")


# ----------------------------------------------------------------- torch side
def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    if t.dtype == torch.float16:
        return ATTN_FP16
    raise TypeError(f"attention inputs must be bf16 or fp16, got {t.dtype}")


def _check(t, name, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _stream(stream):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream if stream is None else int(stream))


def params_for(q, k, softmax_scale=None, causal=False, window_left=-1, window_right=-1,
               alibi_slopes=None, dropout_p=0.0, dropout_seed=0, dropout_offset=0,
               pos_offset=0):
    B, Nq, H, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("q and k disagree on batch or head dim")
    return make_params(B, Nq, Nk, H, Hkv, d, _dtype_code(q), softmax_scale, causal, window_left,
                       window_right, _slopes_ptr(alibi_slopes, H, q.device), dropout_p,
                       dropout_seed, dropout_offset, pos_offset)


def attn_fwd(q, k, v, softmax_scale: Optional[float] = None, causal: bool = False,
             window_left: int = -1, window_right: int = -1, out=None, lse=None,
             stream=None, alibi_slopes=None, dropout_p: float = 0.0, dropout_seed: int = 0,
             dropout_offset: int = 0, pos_offset: int = 0) -> Tuple["torch.Tensor", "torch.Tensor"]:
    """O = softmax(q k^T * scale + bias + mask) v and the per-row natural-log LSE.

    q (B, Nq, H, d), k and v (B, Nk, Hkv, d), bf16 or fp16, contiguous CUDA
    tensors; ``alibi_slopes`` (optional, (H,) float32) adds
    -slope_h * |i + Nk - Nq - j|.  ``dropout_p`` > 0 drops attention
    probabilities by the generator contract of include/attn.h (seed, offset);
    the backward needs the same three values.  ``pos_offset`` moves the query
    rows relative to the keys (include/attn.h).  Returns (out (B, Nq, H, d),
    lse (B, H, Nq) float32)."""
    import torch
    p = params_for(q, k, softmax_scale, causal, window_left, window_right, alibi_slopes,
                   dropout_p, dropout_seed, dropout_offset, pos_offset)
    B, Nq, H, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
        if t.dtype != q.dtype:
            raise TypeError("q, k, v must share a dtype")
    _check(v, "v", k.shape)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check(out, "out", q.shape)
    _check(lse, "lse", (B, H, Nq))
    ws_bytes = attn_fwd_workspace_size(p)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device) if ws_bytes else None
    st = _lib.attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                       _ptr(ws), ctypes.c_size_t(ws_bytes), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_fwd")
    return out, lse


def attn_fwd_e4m3(q, k, v, q_scale: float, k_scale: float, v_scale: float,
                  softmax_scale: Optional[float] = None, causal: bool = False,
                  window_left: int = -1, window_right: int = -1, out_dtype=None, out=None,
                  lse=None, stream=None) -> Tuple["torch.Tensor", "torch.Tensor"]:
    """Attention over E4M3 inputs: q (B, Nq, H, 128), k and v (B, Nk, Hkv,
    128) hold E4M3 codes (uint8 or float8_e4m3fn CUDA tensors), element ~
    scale * e4m3(code) with one scale per tensor.  Returns (out (B, Nq, H,
    128) in ``out_dtype`` (bf16 by default, or fp16), lse (B, H, Nq)
    float32)."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
        if t.element_size() != 1:
            raise TypeError(f"{n} must hold one-byte E4M3 codes")
    _check(v, "v", k.shape)
    B, Nq, H, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("q and k disagree on batch or head dim")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    code = {torch.bfloat16: ATTN_BF16, torch.float16: ATTN_FP16}.get(out_dtype)
    if code is None:
        raise TypeError("out_dtype must be bfloat16 or float16")
    p = make_params(B, Nq, Nk, H, Hkv, d, code, softmax_scale, causal, window_left, window_right)
    if out is None:
        out = torch.empty((B, Nq, H, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check(out, "out", (B, Nq, H, d))
    _check(lse, "lse", (B, H, Nq))
    fn = _lib.attn_fwd_e4m3
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(AttnParams), vp, vp, vp, ctypes.c_float, ctypes.c_float,
                   ctypes.c_float, vp, vp, vp]
    fn.restype = ctypes.c_int
    st = fn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), float(q_scale), float(k_scale),
            float(v_scale), _ptr(out), _ptr(lse), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_fwd_e4m3")
    return out, lse


def attn_fwd_decode(q, k, v, softmax_scale: Optional[float] = None, causal: bool = False,
                    window_left: int = -1, window_right: int = -1, out=None, lse=None,
                    workspace=None, stream=None) -> Tuple["torch.Tensor", "torch.Tensor"]:
    """``attn_fwd`` for decoding: a few query rows ((H / Hkv) * Nq <= 16)
    against a long key / value sequence, on the CUDA cores with the keys
    split over blocks.  Same arguments, layouts and results as ``attn_fwd``
    (no positional slopes)."""
    import torch
    p = params_for(q, k, softmax_scale, causal, window_left, window_right)
    B, Nq, H, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
        if t.dtype != q.dtype:
            raise TypeError("q, k, v must share a dtype")
    _check(v, "v", k.shape)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out, "out", q.shape)
    _check(lse, "lse", (B, H, Nq))
    fn = _lib.attn_fwd_decode_workspace_size
    fn.argtypes = [ctypes.POINTER(AttnParams)]
    fn.restype = ctypes.c_size_t
    ws_bytes = int(fn(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    vp = ctypes.c_void_p
    call = _lib.attn_fwd_decode
    call.argtypes = [ctypes.POINTER(AttnParams), vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    call.restype = ctypes.c_int
    st = call(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(workspace),
              ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_fwd_decode")
    return out, lse


def _bwd_tensors(q, k, v, out, lse, dout, dq, dk, dv):
    """Checks every tensor of a backward call before any pointer reaches the
    library (CUDA, contiguous, shapes, one 16-bit dtype; lse float32) and
    allocates the gradients the caller did not pass.  Raises ValueError or
    TypeError, so a wrong tensor never becomes an out-of-bounds access."""
    import torch
    B, Nq, H, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, n)
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, out, dout must share a dtype")
    _check(v, "v", k.shape)
    _check(out, "out", q.shape)
    _check(dout, "dout", q.shape)
    _check(lse, "lse", (B, H, Nq))
    if lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n, shape in ((dq, "dq", q.shape), (dk, "dk", k.shape), (dv, "dv", k.shape)):
        _check(t, n, shape)
        if t.dtype != q.dtype:
            raise TypeError(f"{n} must have the inputs' dtype")
    return dq, dk, dv


def attn_bwd(q, k, v, out, lse, dout, softmax_scale: Optional[float] = None, causal: bool = False,
             window_left: int = -1, window_right: int = -1, dq=None, dk=None, dv=None,
             workspace=None, stream=None, alibi_slopes=None, dropout_p: float = 0.0,
             dropout_seed: int = 0, dropout_offset: int = 0, pos_offset: int = 0):
    """Gradients (dq, dk, dv) of sum(out * dout) for attention with the same
    arguments as ``attn_fwd``; ``out`` and ``lse`` are its results."""
    import torch
    p = params_for(q, k, softmax_scale, causal, window_left, window_right, alibi_slopes,
                   dropout_p, dropout_seed, dropout_offset, pos_offset)
    dq, dk, dv = _bwd_tensors(q, k, v, out, lse, dout, dq, dk, dv)
    ws_bytes = attn_bwd_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    st = _lib.attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                       _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                       ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def attn_bwd_prepare(p: AttnParams, out, lse, dout, workspace, stream=None) -> None:
    """First backward stage (rowsum(dout*out), lse in base 2, zeroed dQ
    accumulator) on already-validated torch tensors and a params struct."""
    st = _lib.attn_bwd_prepare(ctypes.byref(p), _ptr(out), _ptr(lse), _ptr(dout), _ptr(workspace),
                               ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd_prepare")


def attn_bwd_accumulate(p: AttnParams, q, k, v, dout, dk, dv, workspace, stream=None) -> None:
    """Second backward stage: dk, dv and the fp32 dQ accumulator."""
    st = _lib.attn_bwd_accumulate(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk),
                                  _ptr(dv), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                  _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd_accumulate")


def attn_bwd_accumulate_f32(p: AttnParams, q, k, v, dout, dk_acc, dv_acc, workspace,
                            stream=None) -> None:
    """Second backward stage with the key gradients added in float32:
    dk_acc += scale * dS^T Q, dv_acc += P^T dout (float32 tensors of k's
    shape), plus the dQ share into the workspace accumulator."""
    for t, n in ((dk_acc, "dk_acc"), (dv_acc, "dv_acc")):
        _check(t, n, k.shape)
        if t.element_size() != 4 or not t.is_floating_point():
            raise TypeError(f"{n} must be float32")
    st = _lib.attn_bwd_accumulate_f32(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                      _ptr(dk_acc), _ptr(dv_acc), _ptr(workspace),
                                      ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd_accumulate_f32")


def attn_f32_to_16(src, dst, stream=None) -> None:
    """dst (bf16 or fp16) = src (float32, same number of elements) rounded
    to nearest even, on the GPU."""
    _check(src, "src")
    _check(dst, "dst")
    if src.numel() != dst.numel() or src.element_size() != 4:
        raise ValueError("src must be float32 with dst's number of elements")
    st = _lib.attn_f32_to_16(_ptr(src), _ptr(dst), ctypes.c_longlong(src.numel()),
                             _dtype_code(dst), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_f32_to_16")


def attn_bwd_finalize(p: AttnParams, dq, workspace, stream=None) -> None:
    """Third backward stage: dq = scale * accumulator in the input dtype."""
    st = _lib.attn_bwd_finalize(ctypes.byref(p), _ptr(dq), _ptr(workspace),
                                ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd_finalize")


def attn_bwd_noalloc(q, k, v, out, lse, dout, softmax_scale: Optional[float] = None,
                     causal: bool = False, window_left: int = -1, window_right: int = -1,
                     dq=None, dk=None, dv=None, stream=None, alibi_slopes=None,
                     dropout_p: float = 0.0, dropout_seed: int = 0, dropout_offset: int = 0,
                     pos_offset: int = 0):
    """Like ``attn_bwd`` but the library uses its own fixed device scratch
    (ATTN_NOALLOC_SCRATCH_BYTES) instead of a caller workspace, for callers
    that cannot allocate device memory at call time.  The output tensors are
    the caller's (allocated here only when not given).  Calls that overlap on
    the GPU share that scratch and must be serialised by the caller."""
    p = params_for(q, k, softmax_scale, causal, window_left, window_right, alibi_slopes,
                   dropout_p, dropout_seed, dropout_offset, pos_offset)
    dq, dk, dv = _bwd_tensors(q, k, v, out, lse, dout, dq, dk, dv)
    st = _lib.attn_bwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                               _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd_noalloc")
    return dq, dk, dv


# ----------------------------------------------------------------- packed sequences
def make_varlen_params(batch, total_q, total_k, max_seqlen_q, max_seqlen_k, nheads, nheads_kv,
                       headdim, dtype=ATTN_BF16, softmax_scale=None, causal=False,
                       window_left=-1, window_right=-1, alibi_slopes=None, dropout_p=0.0,
                       dropout_seed=0, dropout_offset=0) -> AttnVarlenParams:
    scale = 1.0 / math.sqrt(headdim) if softmax_scale is None else float(softmax_scale)
    return AttnVarlenParams(int(batch), int(total_q), int(total_k), int(max_seqlen_q),
                            int(max_seqlen_k), int(nheads), int(nheads_kv), int(headdim),
                            int(dtype), scale, int(bool(causal)), int(window_left),
                            int(window_right), alibi_slopes, float(dropout_p),
                            int(dropout_offset) & 0xFFFFFFFF, int(dropout_seed) & (2 ** 64 - 1))


def attn_check_varlen_params(p: AttnVarlenParams, pass_: int = 0) -> int:
    return int(_lib.attn_check_varlen_params(ctypes.byref(p), int(pass_)))


def attn_bwd_varlen_workspace_size(p: AttnVarlenParams) -> int:
    return int(_lib.attn_bwd_varlen_workspace_size(ctypes.byref(p)))


def _varlen_params(q, k, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, softmax_scale,
                   causal, window_left, window_right, alibi_slopes=None, dropout_p=0.0,
                   dropout_seed=0, dropout_offset=0):
    import torch
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed q must be (total_q, nheads, d) and k (total_k, nheads_kv, d)")
    Tq, H, d = q.shape
    Tk, Hkv, dk = k.shape
    if dk != d:
        raise ValueError("q and k disagree on head dim")
    for t, n in ((cu_seqlens_q, "cu_seqlens_q"), (cu_seqlens_k, "cu_seqlens_k")):
        _check(t, n)
        if t.dtype != torch.int32 or t.dim() != 1:
            raise TypeError(f"{n} must be a 1-D int32 CUDA tensor")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have batch + 1 entries")
    return make_varlen_params(cu_seqlens_q.numel() - 1, Tq, Tk, max_seqlen_q, max_seqlen_k, H, Hkv,
                              d, _dtype_code(q), softmax_scale, causal, window_left, window_right,
                              _slopes_ptr(alibi_slopes, H, q.device), dropout_p, dropout_seed,
                              dropout_offset)


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    softmax_scale: Optional[float] = None, causal: bool = False,
                    window_left: int = -1, window_right: int = -1, out=None, lse=None,
                    stream=None, alibi_slopes=None, dropout_p: float = 0.0, dropout_seed: int = 0,
                    dropout_offset: int = 0):
    """Attention over packed variable-length sequences.

    q (total_q, H, d), k and v (total_k, Hkv, d); sequence b owns rows
    cu_seqlens_q[b]:cu_seqlens_q[b+1] of q and cu_seqlens_k[b]:cu_seqlens_k[b+1]
    of k, v (int32 CUDA tensors of batch + 1 offsets).  Returns (out
    (total_q, H, d), lse (H, total_q) float32)."""
    import torch
    p = _varlen_params(q, k, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                       softmax_scale, causal, window_left, window_right, alibi_slopes,
                       dropout_p, dropout_seed, dropout_offset)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
        if t.dtype != q.dtype:
            raise TypeError("q, k, v must share a dtype")
    _check(v, "v", k.shape)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    _check(out, "out", q.shape)
    _check(lse, "lse", (q.shape[1], q.shape[0]))
    st = _lib.attn_fwd_varlen(ctypes.byref(p), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(q),
                              _ptr(k), _ptr(v), _ptr(out), _ptr(lse), None, ctypes.c_size_t(0),
                              _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_fwd_varlen")
    return out, lse


def attn_bwd_varlen(q, k, v, out, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                    max_seqlen_k: int, softmax_scale: Optional[float] = None,
                    causal: bool = False, window_left: int = -1, window_right: int = -1,
                    dq=None, dk=None, dv=None, workspace=None, stream=None, alibi_slopes=None,
                    dropout_p: float = 0.0, dropout_seed: int = 0, dropout_offset: int = 0):
    """Gradients (dq, dk, dv) of sum(out * dout) for ``attn_fwd_varlen`` with
    the same arguments; ``out`` and ``lse`` are its results."""
    import torch
    p = _varlen_params(q, k, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                       softmax_scale, causal, window_left, window_right, alibi_slopes,
                       dropout_p, dropout_seed, dropout_offset)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, n)
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, out, dout must share a dtype")
    _check(v, "v", k.shape)
    _check(out, "out", q.shape)
    _check(dout, "dout", q.shape)
    _check(lse, "lse", (q.shape[1], q.shape[0]))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws_bytes = attn_bwd_varlen_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    st = _lib.attn_bwd_varlen(ctypes.byref(p), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), _ptr(q),
                              _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                              _ptr(dk), _ptr(dv), _ptr(workspace),
                              ctypes.c_size_t(workspace.numel()), _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_bwd_varlen")
    return dq, dk, dv


# ----------------------------------------------------------------- merge of partial results
def attn_merge(o_parts, lse_parts, out=None, lse=None, stream=None):
    """Merge partial results over disjoint key sets (split-KV): o_parts
    (S, B, Nq, H, d) 16-bit, lse_parts (S, B, H, Nq) float32, both CUDA and
    contiguous.  Returns (out (B, Nq, H, d), lse (B, H, Nq))."""
    import torch
    _check(o_parts, "o_parts")
    _check(lse_parts, "lse_parts")
    if o_parts.dim() != 5 or lse_parts.dtype != torch.float32:
        raise ValueError("o_parts must be (splits, B, Nq, H, d); lse_parts float32 (splits, B, H, Nq)")
    S, B, Nq, H, d = o_parts.shape
    if tuple(lse_parts.shape) != (S, B, H, Nq):
        raise ValueError(f"lse_parts has shape {tuple(lse_parts.shape)}, expected {(S, B, H, Nq)}")
    out = torch.empty(o_parts.shape[1:], dtype=o_parts.dtype, device=o_parts.device) if out is None else out
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=o_parts.device) if lse is None else lse
    _check(out, "out", o_parts.shape[1:])
    _check(lse, "lse", (B, H, Nq))
    p = AttnMergeParams(S, B, Nq, H, d, _dtype_code(o_parts))
    st = _lib.attn_merge(ctypes.byref(p), _ptr(o_parts), _ptr(lse_parts), _ptr(out), _ptr(lse),
                         _stream(stream))
    if st != 0:
        raise AttnError(st, "attn_merge")
    return out, lse
