"""Per-head positional slopes (alibi_slopes) on the GPU against the float64
oracle with the same slopes: forward and backward for head dims 64, 128 and
256, every mask kind, GQA, Nq != Nk, fp16, packed sequences,
and zero slopes against no slopes."""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import Workload, make_inputs, make_varlen_inputs
from parity import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def slopes_for(h):
    """The geometric slopes of the usual positional-bias recipe, 2^(-8k/H)."""
    return torch.tensor([2.0 ** (-8.0 * (k + 1) / h) for k in range(h)], dtype=torch.float32)


def W(name, B, H, Hkv, Nq, Nk, d, causal=False, wl=-1, wr=-1, dtype="bf16", seed=500):
    return Workload(name, B, H, Hkv, Nq, Nk, d, causal, wl, wr, dtype, 1.0, seed)


CASES = [
    (W("d128", 1, 4, 4, 300, 300, 128, seed=501), True),
    (W("d128_causal", 2, 4, 2, 513, 513, 128, causal=True, seed=502), True),
    (W("d128_window", 1, 8, 2, 700, 700, 128, causal=True, wl=129, seed=503), True),
    (W("d128_both_sides", 1, 2, 2, 400, 400, 128, wl=100, wr=60, seed=504), True),
    (W("d128_nq_lt_nk", 1, 2, 2, 100, 390, 128, causal=True, seed=505), True),
    (W("d128_nq_gt_nk", 1, 2, 1, 260, 130, 128, seed=506), True),
    (W("d64_fp16", 1, 4, 4, 256, 256, 64, dtype="fp16", seed=507), True),
    (W("d64_causal", 2, 2, 2, 260, 260, 64, causal=True, seed=508), True),
    (W("d256_causal", 1, 2, 2, 300, 300, 256, causal=True, dtype="fp16", seed=509), True),
    (W("d256", 1, 2, 1, 200, 330, 256, seed=510), True),
    (W("d256_window", 1, 4, 2, 450, 450, 256, causal=True, wl=129, seed=512), True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_alibi_parity(attn, case):
    w, bwd = case
    q, k, v, do = make_inputs(w)
    sl = slopes_for(w.nheads)
    args = (w.scale, w.causal, w.window_left, w.window_right)
    qc, kc, vc, doc, slc = q.cuda(), k.cuda(), v.cuda(), do.cuda(), sl.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, *args, alibi_slopes=slc)
    grads = attn.attn_bwd(qc, kc, vc, o, lse, doc, *args, alibi_slopes=slc) if bwd else None
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, *args, alibi_slopes=sl.double())
    check_o(o.cpu(), o_ref, w.name)
    check_lse(lse.cpu(), lse_ref, w.name)
    if bwd:
        refs = oracle.attention_bwd(q, k, v, do, *args, alibi_slopes=sl.double())
        for g, r, n in zip(grads, refs, ("dQ", "dK", "dV")):
            check_grad(g.cpu(), r, f"{w.name} {n}")


def test_alibi_zero_slopes_match_no_slopes(attn):
    w = W("zero", 1, 4, 4, 384, 384, 128, causal=True, seed=511)
    q, k, v, do = (t.cuda() for t in make_inputs(w))
    zero = torch.zeros(4, dtype=torch.float32, device="cuda")
    o0, l0 = attn.attn_fwd(q, k, v, None, True, alibi_slopes=zero)
    o1, l1 = attn.attn_fwd(q, k, v, None, True)
    g0 = attn.attn_bwd(q, k, v, o0, l0, do, None, True, alibi_slopes=zero)
    g1 = attn.attn_bwd(q, k, v, o1, l1, do, None, True)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
    assert torch.equal(g0[1], g1[1]) and torch.equal(g0[2], g1[2])


def test_alibi_packed_sequences(attn):
    lens_q, lens_k = [200, 1, 129, 330], [260, 64, 129, 300]
    H, Hkv, d = 4, 2, 128
    q, k, v, do, cu_q, cu_k = make_varlen_inputs(lens_q, lens_k, H, Hkv, d, seed=512)
    sl = slopes_for(H)
    args = (1.0 / np.sqrt(d), True, -1, -1)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = attn.attn_fwd_varlen(qc, kc, vc, cu_q.cuda(), cu_k.cuda(), max(lens_q), max(lens_k),
                                  *args, alibi_slopes=sl.cuda())
    grads = attn.attn_bwd_varlen(qc, kc, vc, o, lse, doc, cu_q.cuda(), cu_k.cuda(), max(lens_q),
                                 max(lens_k), *args, alibi_slopes=sl.cuda())
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd_varlen(q, k, v, cu_q, cu_k, *args,
                                                 alibi_slopes=sl.double())
    check_o(o.cpu(), o_ref, "packed alibi")
    check_lse(lse.cpu(), lse_ref, "packed alibi")
    refs = oracle.attention_bwd_varlen(q, k, v, do, cu_q, cu_k, *args, alibi_slopes=sl.double())
    for g, r, n in zip(grads, refs, ("dQ", "dK", "dV")):
        check_grad(g.cpu(), r, f"packed alibi {n}")


@pytest.mark.parametrize("causal", [False, True])
def test_alibi_steep_slopes(attn, causal):
    """Slopes above ~0.35 make the bias vary by more than 64 (log2 units)
    across a key tile; the forward then takes the exact biased row max
    instead of its upper bound.  Mixed heads exercise both."""
    w = W("steep", 1, 4, 4, 300, 300, 128, causal=causal, seed=513)
    q, k, v, do = make_inputs(w)
    sl = torch.tensor([2.0, 0.5, 0.02, 1.0], dtype=torch.float32)
    args = (w.scale, w.causal, -1, -1)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, *args, alibi_slopes=sl.cuda())
    grads = attn.attn_bwd(qc, kc, vc, o, lse, doc, *args, alibi_slopes=sl.cuda())
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, *args, alibi_slopes=sl.double())
    check_o(o.cpu(), o_ref, "steep")
    check_lse(lse.cpu(), lse_ref, "steep")
    refs = oracle.attention_bwd(q, k, v, do, *args, alibi_slopes=sl.double())
    for g, r, n in zip(grads, refs, ("dQ", "dK", "dV")):
        check_grad(g.cpu(), r, f"steep {n}")
