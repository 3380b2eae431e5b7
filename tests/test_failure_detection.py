"""Failure detection without a GPU fault.

Every on-chip barrier wait in the kernels is bounded: on expiry the kernel
records ATTN_ERR_TIMEOUT in a device status word and returns instead of
spinning.  The GPU test drives that path with the library's self-test kernel,
whose waiters wait on a barrier nothing ever arrives at (with a 20 ms limit),
then checks the status word and that the context still runs attention
correctly.  The CPU tests cover the host-side argument checks of the entry
point."""
import time

import pytest

import oracle
from attn_inputs import WORKLOADS, make_inputs
from parity import check_lse, check_o


@pytest.fixture(scope="module")
def attn():
    from io_aware_exact_33_b200 import build
    build.build()
    import io_aware_exact_33_b200 as m
    return m


@pytest.mark.parametrize("limit_us", [0, 1000001, 2**32 - 1])
def test_selftest_rejects_bad_limit_without_launch(attn, limit_us):
    with pytest.raises(attn.AttnError) as e:
        attn.attn_selftest_bounded_wait(limit_us, stream=0)
    assert e.value.status == 1  # ATTN_ERR_INVALID_ARG, checked on the host


@pytest.mark.gpu
def test_bounded_wait_expires_and_context_survives(attn):
    import torch
    dev = torch.device("cuda:0")
    assert attn.attn_get_device_status() == 0
    result = torch.full((2,), -1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    attn.attn_selftest_bounded_wait(20000, result)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert result.tolist() == [1, 1]            # both waiters gave up
    assert elapsed >= 0.019                     # ... not before the limit
    assert elapsed < 5.0
    assert attn.attn_get_device_status() == 7   # ATTN_ERR_TIMEOUT recorded
    assert attn.attn_get_device_status() == 0   # and cleared by the read

    # The context is still usable: a normal forward call after the timeout.
    w = WORKLOADS["tiny_b1_h2_n128_d64"]
    q, k, v, _ = make_inputs(w, with_dout=False)
    o, lse = attn.attn_fwd(q.to(dev), k.to(dev), v.to(dev), w.scale, w.causal, w.window_left,
                           w.window_right)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.scale, w.causal, w.window_left,
                                          w.window_right)
    check_o(o.cpu(), o_ref, "after timeout")
    check_lse(lse.cpu(), lse_ref, "after timeout")
    assert attn.attn_get_device_status() == 0
