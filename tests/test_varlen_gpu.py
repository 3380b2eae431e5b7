"""Packed variable-length sequences: attn_fwd_varlen / attn_bwd_varlen against
the float64 oracle run on every sequence alone (the oracle's own per-sequence
entry points), over ragged lengths that start and end inside tiles, empty
query and key sequences, query and key lengths that differ per sequence,
every mask kind, GQA, both dtypes and all head dimensions; rows that belong
to no sequence must keep their contents (dq gets zeros there)."""
import random

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_varlen_inputs
from parity import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def _lens(n, lo, hi, seed):
    r = random.Random(seed)
    return [r.randint(lo, hi) for _ in range(n)]


CASES = [
    # name, lens_q, lens_k, H, Hkv, d, dtype, mask kwargs, backward?
    ("ragged_d128", [1, 127, 128, 129, 300, 0, 513], [1, 127, 128, 129, 300, 0, 513], 4, 2, 128,
     "bf16", dict(causal=False), True),
    ("ragged_causal_nq_ne_nk", [100, 257, 64, 3, 200], [390, 257, 200, 0, 70], 4, 4, 128, "bf16",
     dict(causal=True), True),
    ("window_gqa", [700, 33, 1000], [700, 33, 1000], 8, 2, 128, "bf16",
     dict(causal=True, window_left=129, window_right=0), True),
    ("window_both_sides", [500, 260], [480, 300], 2, 2, 128, "bf16",
     dict(causal=False, window_left=100, window_right=60), True),
    ("d64_fp16", [65, 200, 128, 1, 77], [65, 200, 128, 1, 77], 2, 1, 64, "fp16",
     dict(causal=False), True),
    ("d64_causal", [260, 129], [260, 129], 2, 2, 64, "bf16", dict(causal=True), True),
    ("d128_fp16_causal", [384, 17, 255], [384, 17, 255], 2, 2, 128, "fp16", dict(causal=True),
     True),
    ("d256_fp16_causal", [300, 129, 64], [300, 129, 64], 2, 2, 256, "fp16",
     dict(causal=True), True),
    ("d256_bf16", [65, 250], [200, 250], 2, 1, 256, "bf16", dict(causal=False), True),
    ("d256_window_gqa", [400, 0, 190], [400, 0, 190], 4, 2, 256, "bf16",
     dict(causal=True, window_left=100, window_right=0), True),
    ("many_causal", _lens(12, 1, 2000, 5), None, 8, 8, 128, "bf16", dict(causal=True), True),
]


def _run(attn, name, lens_q, lens_k, H, Hkv, d, dtype, mask, bwd, seed, extra=(0, 0)):
    lens_k = lens_q if lens_k is None else lens_k
    q, k, v, do, cu_q, cu_k = make_varlen_inputs(lens_q, lens_k, H, Hkv, d, dtype, seed=seed,
                                                 extra_q=extra[0], extra_k=extra[1])
    scale = 1.0 / np.sqrt(d)
    args = (scale, mask.get("causal", False), mask.get("window_left", -1),
            mask.get("window_right", -1))
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    cqc, ckc = cu_q.cuda(), cu_k.cuda()
    mq, mk = max(lens_q), max(lens_k)
    sentinel = 7.0
    o = torch.full_like(qc, sentinel)
    lse = torch.full((H, q.shape[0]), sentinel, dtype=torch.float32, device="cuda")
    attn.attn_fwd_varlen(qc, kc, vc, cqc, ckc, mq, mk, *args, out=o, lse=lse)
    grads = None
    if bwd:
        dk = torch.full_like(kc, sentinel)
        dv = torch.full_like(vc, sentinel)
        grads = attn.attn_bwd_varlen(qc, kc, vc, o, lse, doc, cqc, ckc, mq, mk, *args, dk=dk,
                                     dv=dv)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    return (q, k, v, do, cu_q, cu_k, args), o.cpu(), lse.cpu(), grads


@pytest.mark.parametrize("idx", range(len(CASES)), ids=[c[0] for c in CASES])
def test_varlen_parity(attn, idx):
    name, lens_q, lens_k, H, Hkv, d, dtype, mask, bwd = CASES[idx]
    (q, k, v, do, cu_q, cu_k, args), o, lse, grads = _run(
        attn, name, lens_q, lens_k, H, Hkv, d, dtype, mask, bwd, seed=300 + idx)
    o_ref, lse_ref = oracle.attention_fwd_varlen(q, k, v, cu_q, cu_k, *args)
    check_o(o, o_ref, name)
    check_lse(lse, lse_ref, name)
    if bwd:
        dq_r, dk_r, dv_r = oracle.attention_bwd_varlen(q, k, v, do, cu_q, cu_k, *args)
        dq, dk, dv = (g.cpu() for g in grads)
        check_grad(dq, dq_r, name + " dQ")
        check_grad(dk, dk_r, name + " dK")
        check_grad(dv, dv_r, name + " dV")


def test_varlen_rows_outside_sequences(attn):
    """Rows past the last sequence: o, lse, dk, dv keep their contents and
    dq is zero there; the sequences themselves match the oracle."""
    lens = [130, 70]
    (q, k, v, do, cu_q, cu_k, args), o, lse, grads = _run(
        attn, "outside", lens, lens, 2, 2, 128, "bf16", dict(causal=True), True, seed=41,
        extra=(50, 40))
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    assert torch.all(o[tq:].float() == 7.0) and torch.all(lse[:, tq:] == 7.0)
    dq, dk, dv = (g.cpu() for g in grads)
    assert torch.all(dq[tq:].float() == 0.0)
    assert torch.all(dk[tk:].float() == 7.0) and torch.all(dv[tk:].float() == 7.0)
    o_ref, lse_ref = oracle.attention_fwd_varlen(q, k, v, cu_q, cu_k, *args)
    check_o(o[:tq], o_ref[:tq], "outside")
    check_lse(lse[:, :tq], lse_ref[:, :tq], "outside")


def test_varlen_equals_dense_batch(attn):
    """Equal-length packed sequences give the dense entry point's results:
    bit for bit where the order of the arithmetic is fixed (O, LSE, dK, dV),
    to rounding for dQ (its partial sums are added into the accumulator in
    whatever order the key tiles finish)."""
    B, N, H, d = 3, 384, 4, 128
    q, k, v, do, cu_q, cu_k = make_varlen_inputs([N] * B, [N] * B, H, H, d, seed=43)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o_p, lse_p = attn.attn_fwd_varlen(qc, kc, vc, cu_q.cuda(), cu_k.cuda(), N, N, None, True)
    o_d, lse_d = attn.attn_fwd(qc.view(B, N, H, d), kc.view(B, N, H, d), vc.view(B, N, H, d),
                               None, True)
    torch.cuda.synchronize()
    assert torch.equal(o_p.view(B, N, H, d), o_d)
    assert torch.equal(lse_p.view(H, B, N).permute(1, 0, 2), lse_d)
    g_p = attn.attn_bwd_varlen(qc, kc, vc, o_p, lse_p, doc, cu_q.cuda(), cu_k.cuda(), N, N, None,
                               True)
    g_d = attn.attn_bwd(qc.view(B, N, H, d), kc.view(B, N, H, d), vc.view(B, N, H, d), o_d, lse_d,
                        doc.view(B, N, H, d), None, True)
    torch.cuda.synchronize()
    assert torch.equal(g_p[1].view(g_d[1].shape), g_d[1])
    assert torch.equal(g_p[2].view(g_d[2].shape), g_d[2])
    dq_p, dq_d = g_p[0].view(g_d[0].shape).double(), g_d[0].double()
    assert float((dq_p - dq_d).norm() / dq_d.norm()) < 1e-3
