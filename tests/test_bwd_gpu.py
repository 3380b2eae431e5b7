"""Backward parity: dQ, dK, dV from the sm_100a kernels against the float64
oracle's analytic gradients on the same seeded inputs (full tensors at small
sizes; sampled rows plus exact identities at the full workload sizes)."""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import WORKLOADS, Workload, make_inputs, sample_rows
from parity import check_grad, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def W(name, B, H, Hkv, Nq, Nk, d, causal=False, wl=-1, wr=-1, dtype="bf16", seed=200, sigma=1.0):
    return Workload(name, B, H, Hkv, Nq, Nk, d, causal, wl, wr, dtype, sigma, seed)


def run_bwd(attn, w: Workload):
    q, k, v, do = make_inputs(w)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    args = (w.scale, w.causal, w.window_left, w.window_right)
    o, lse = attn.attn_fwd(qc, kc, vc, *args)
    dq, dk, dv = attn.attn_bwd(qc, kc, vc, o, lse, doc, *args)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    return (q, k, v, do), (dq.cpu(), dk.cpu(), dv.cpu())


SMALL = [
    W("d64_n128", 1, 2, 2, 128, 128, 64),
    W("d128_n128", 1, 2, 2, 128, 128, 128),
    W("d128_ragged", 2, 2, 2, 300, 300, 128, seed=201),
    W("d64_ragged", 1, 3, 3, 200, 200, 64, seed=202),
    W("d128_causal", 1, 4, 4, 513, 513, 128, causal=True, seed=203),
    W("d64_causal", 2, 2, 2, 260, 260, 64, causal=True, seed=204),
    W("d128_fp16_causal", 1, 2, 2, 384, 384, 128, causal=True, dtype="fp16", seed=205),
    W("d64_fp16", 1, 2, 1, 256, 256, 64, dtype="fp16", seed=206),
    W("gqa4_window", 2, 8, 2, 700, 700, 128, causal=True, wl=129, wr=0, seed=207),
    W("gqa8_window_edge", 1, 8, 1, 640, 640, 128, causal=True, wl=127, seed=208),
    W("window_both_sides", 1, 2, 2, 500, 500, 128, wl=100, wr=60, seed=209),
    W("nq_lt_nk_causal", 1, 2, 2, 100, 390, 128, causal=True, seed=210),
    W("nq_gt_nk_causal_empty_rows", 1, 2, 2, 300, 130, 128, causal=True, seed=211),
    W("nq_gt_nk_d64", 1, 2, 1, 257, 65, 64, seed=212),
    W("single_row", 1, 1, 1, 1, 1, 128, seed=213),
    # head dim 256: three kernels (dV, dK key-stationary; dQ query-stationary)
    W("d256_n128", 1, 2, 2, 128, 128, 256, seed=220),
    W("d256_ragged_gqa_causal", 2, 4, 2, 333, 333, 256, causal=True, seed=221),
    W("d256_fp16_nq_lt_nk", 1, 2, 1, 200, 330, 256, dtype="fp16", seed=222),
    W("d256_window", 1, 4, 4, 600, 600, 256, causal=True, wl=129, seed=223),
    W("d256_window_both_sides", 1, 2, 2, 500, 500, 256, wl=100, wr=60, seed=224),
    W("d256_nq_gt_nk_empty_rows", 1, 2, 2, 300, 130, 256, causal=True, seed=225),
    W("d256_gqa8_causal", 1, 8, 1, 257, 257, 256, causal=True, seed=226),
    W("d256_single_row", 1, 1, 1, 1, 1, 256, seed=227),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_bwd_small_full(attn, w):
    (q, k, v, do), (dq, dk, dv) = run_bwd(attn, w)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do, w.scale, w.causal, w.window_left,
                                            w.window_right)
    check_grad(dq, dq_r, w.name + " dQ")
    check_grad(dk, dk_r, w.name + " dK")
    check_grad(dv, dv_r, w.name + " dV")


def test_bwd_tiny_workload(attn):
    w = WORKLOADS["tiny_b1_h2_n128_d64"]
    (q, k, v, do), (dq, dk, dv) = run_bwd(attn, w)
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do, w.scale, w.causal)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


def _identities(w, do, dk, dv):
    """sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i (over each GQA group) for
    every (batch, kv head): rows of dS sum to zero and rows of P to one, for
    every query that sees at least one key (true for all queries here)."""
    B, Nq, H, d = do.shape
    Hkv = dk.shape[2]
    g = H // Hkv
    sdv = dv.double().sum(dim=1)  # (B, Hkv, d)
    sdo = do.double().sum(dim=1).reshape(B, Hkv, g, d).sum(dim=2)
    rel = ((sdv - sdo).norm() / sdo.norm()).item()
    assert rel <= 1e-2, f"sum dV vs sum dO: {rel:.3e}"
    sdk = dk.double().sum(dim=1)
    scale_ref = dk.double().abs().sum(dim=1).norm().item()
    assert sdk.norm().item() <= 1e-2 * scale_ref, "sum dK is not ~0"


# The two largest workloads are checked on many more rows, with their raw
# errors recorded, in test_parity_configs_gpu.py (which also runs the
# identities below on them).
@pytest.mark.parametrize("name", ["tiny_b1_h2_n128_d64", "gqa_window_b4_h32_kv8_n4096_d128"])
def test_bwd_full_size_sampled(attn, name):
    w = WORKLOADS[name]
    (q, k, v, do), (dq, dk, dv) = run_bwd(attn, w)
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    _identities(w, do, dk, dv)
    must = [1, 127, 128, 129, w.seqlen_q // 2]
    if w.window_left >= 0:
        must += [w.window_left, w.window_left + 1]
    qrows = sample_rows(w.seqlen_q, 6, w.seed, must=must)
    krows = sample_rows(w.seqlen_k, 6, w.seed + 1, must=must)
    dq_r, dk_r, dv_r = oracle.attention_bwd_rows(q, k, v, do, qrows, krows, w.scale, w.causal,
                                                 w.window_left, w.window_right)
    check_grad(dq[:, qrows], dq_r, name + " dQ rows")
    check_grad(dk[:, krows], dk_r, name + " dK rows")
    check_grad(dv[:, krows], dv_r, name + " dV rows")


def test_bwd_empty_sides(attn):
    q = torch.randn(1, 20, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(1, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(q)
    lse = torch.full((1, 2, 20), float("-inf"), device="cuda")
    dq, dk, dv = attn.attn_bwd(q, k, k.clone(), o, lse, torch.randn_like(q))
    torch.cuda.synchronize()
    assert (dq == 0).all() and dk.numel() == 0


def test_bwd_headdim_256_rejects_dropout(attn):
    q = torch.randn(1, 16, 2, 256, dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd(q, q.clone(), q.clone())
    with pytest.raises(attn.AttnError) as e:
        attn.attn_bwd(q, q, q, o, lse, q, dropout_p=0.1, dropout_seed=1)
    assert e.value.status == 2


def test_bwd_d256_accumulates(attn):
    """attn_bwd_accumulate adds its dQ share to the accumulator (twice gives
    twice the gradient), as for the other head dims."""
    w = W("d256_acc", 1, 2, 2, 200, 200, 256, causal=True, seed=228)
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    o, lse = attn.attn_fwd(q, k, v, w.scale, True)
    p = attn.params_for(q, k, w.scale, True)
    ws = torch.empty(attn.attn_bwd_workspace_size(p), dtype=torch.uint8, device="cuda")
    dq1, dq2 = torch.empty_like(q), torch.empty_like(q)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    attn.attn_bwd_prepare(p, o, lse, do, ws)
    attn.attn_bwd_accumulate(p, q, k, v, do, dk, dv, ws)
    attn.attn_bwd_finalize(p, dq1, ws)
    attn.attn_bwd_accumulate(p, q, k, v, do, dk, dv, ws)
    attn.attn_bwd_finalize(p, dq2, ws)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    assert torch.allclose(dq2.float(), 2 * dq1.float(), rtol=1e-2, atol=1e-3)


def test_bwd_workspace_too_small(attn):
    q = torch.randn(1, 64, 2, 128, dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd(q, q, q)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(attn.AttnError) as e:
        attn.attn_bwd(q, q, q, o, lse, q, workspace=ws)
    assert e.value.status == 5
