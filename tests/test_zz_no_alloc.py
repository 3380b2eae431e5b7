"""attn_bwd_noalloc: the backward entry point for callers that cannot allocate
device memory (a host framework that owns the GPU's memory pool, or a
latency-critical path that cannot afford cudaMalloc's device synchronisation
and possible failure).  It uses a fixed scratch array inside libattn.so
instead of a caller workspace.

Called here straight through the C ABI (ctypes on libattn.so) and compared
with attn_bwd, the entry point that takes a caller workspace, on two calls in
a row: the second call must not see the first call's leftovers in the shared
scratch.  Both calls are also checked against the float64 oracle directly,
and the Python wrapper of the same name is run once (its results against the
oracle, its argument checks against tensors of the wrong shape or layout).
This file is collected last so that a run stopping at its first failure has
already run every other test; it passes alone in a fresh process as well as
after the others.
"""
import ctypes

import pytest
import torch

import oracle
from attn_inputs import Workload, make_inputs
from parity import check_grad, rel_fro

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # ATTN_NOALLOC_SCRATCH_BYTES in include/attn.h


@pytest.fixture(scope="module")
def abi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    lib = ctypes.CDLL(m.LIB_PATH)
    vp, P = ctypes.c_void_p, ctypes.POINTER(m.AttnParams)
    lib.attn_bwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.attn_bwd_noalloc.restype = ctypes.c_int
    lib.attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.attn_bwd.restype = ctypes.c_int
    lib.attn_bwd_workspace_size.argtypes = [P]
    lib.attn_bwd_workspace_size.restype = ctypes.c_size_t
    return m, lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


CASES = [
    Workload("noalloc_d128_causal_gqa", 1, 4, 2, 300, 300, 128, True, seed=300),
    Workload("noalloc_d64_window", 2, 2, 2, 200, 260, 64, False, 40, 17, seed=301),
    Workload("noalloc_d256_causal", 1, 2, 1, 200, 200, 256, True, seed=302),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point_twice(abi, w):
    m, lib = abi
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    args = (w.scale, w.causal, w.window_left, w.window_right)
    o, lse = m.attn_fwd(q, k, v, *args)
    p = m.params_for(q, k, *args)
    assert lib.attn_bwd_workspace_size(ctypes.byref(p)) <= NOALLOC_SCRATCH_BYTES
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    ref = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    ws_bytes = lib.attn_bwd_workspace_size(ctypes.byref(p))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    st = lib.attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                      *(_ptr(t) for t in ref), _ptr(ws), ctypes.c_size_t(ws_bytes), stream)
    assert st == 0

    dq_r, dk_r, dv_r = oracle.attention_bwd(*(t.cpu() for t in (q, k, v, do)), w.scale, w.causal,
                                            w.window_left, w.window_right)
    for call in range(2):
        out = [torch.full_like(q, float("nan")), torch.full_like(k, float("nan")),
               torch.full_like(v, float("nan"))]
        st = lib.attn_bwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                  _ptr(do), *(_ptr(t) for t in out), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert m.attn_get_device_status() == 0
        for name, got, want, exact in zip(("dq", "dk", "dv"), out, ref, (dq_r, dk_r, dv_r)):
            check_grad(got.cpu(), want.double().cpu().numpy(), f"{w.name} call {call} {name}")
            assert rel_fro(got.cpu(), want.double().cpu().numpy()) <= 1e-2
            check_grad(got.cpu(), exact, f"{w.name} call {call} {name} vs the oracle")


def test_noalloc_python_wrapper(abi):
    m, _ = abi
    w = CASES[0]
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    args = (w.scale, w.causal, w.window_left, w.window_right)
    o, lse = m.attn_fwd(q, k, v, *args)
    dq, dk, dv = m.attn_bwd_noalloc(q, k, v, o, lse, do, *args)
    torch.cuda.synchronize()
    assert m.attn_get_device_status() == 0
    exact = oracle.attention_bwd(*(t.cpu() for t in (q, k, v, do)), *args)
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), exact):
        check_grad(got.cpu(), want, f"wrapper {name} vs the oracle")
    # tensors of the wrong shape or layout are refused before the library sees them
    with pytest.raises(ValueError):
        m.attn_bwd_noalloc(q, k, v, o, lse, do, *args, dq=torch.empty_like(q)[:, :-1])
    with pytest.raises(ValueError):
        m.attn_bwd_noalloc(q, k, v, o, lse, do.transpose(1, 2).contiguous().transpose(1, 2),
                           *args)
    with pytest.raises(ValueError):
        m.attn_bwd_noalloc(q, k, v[:, :-1].contiguous(), o, lse, do, *args)
    with pytest.raises(ValueError):
        m.attn_bwd_noalloc(q, k, v, o, lse[..., :-1].contiguous(), do, *args)


def test_noalloc_rejects_sizes_beyond_its_scratch(abi):
    m, lib = abi
    # dQ accumulator alone: 1 x 16384 x 8 x 128 x 4 bytes = 64 MiB > 32 MiB
    p = m.make_params(1, 16384, 16384, 8, 8, 128, m.ATTN_BF16, None, True)
    null = ctypes.c_void_p(0)
    st = lib.attn_bwd_noalloc(ctypes.byref(p), *([null] * 9), ctypes.c_void_p(0))
    assert st == 5  # ATTN_ERR_WORKSPACE_TOO_SMALL, returned before any launch
