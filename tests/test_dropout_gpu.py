"""Dropout on the GPU against the float64 oracle with the same rate, seed and
offset (the generator contract of include/attn.h): forward output and LSE,
backward gradients, for head dims 64 and 128, causal, windowed and full
masks, GQA, Nq != Nk, fp16, positional slopes and packed sequences; runs
repeat exactly and other offsets give other masks; the headdim-256 forward
refuses dropout."""
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


def W(name, B, H, Hkv, Nq, Nk, d, causal=False, wl=-1, wr=-1, dtype="bf16", seed=900):
    return Workload(name, B, H, Hkv, Nq, Nk, d, causal, wl, wr, dtype, 1.0, seed)


# (workload, dropout_p, generator seed, offset, positional slopes)
CASES = [
    (W("d128_causal", 2, 4, 2, 300, 300, 128, causal=True, seed=901), 0.3, 0x1234, 0, False),
    (W("d128_full", 1, 4, 4, 257, 257, 128, seed=902), 0.1, 2 ** 64 - 3, 5, False),
    (W("d128_window", 1, 4, 2, 520, 520, 128, causal=True, wl=129, seed=903), 0.5, 77, 2, False),
    (W("d128_nq_lt_nk", 1, 2, 2, 100, 390, 128, causal=True, seed=904), 0.2, 99, 1, False),
    (W("d128_slopes", 1, 4, 4, 256, 256, 128, causal=True, seed=905), 0.3, 3, 0, True),
    (W("d64_fp16_nq_gt_nk", 1, 4, 2, 333, 200, 64, dtype="fp16", seed=906), 0.1, 11, 7, False),
    (W("d64_causal", 2, 2, 2, 260, 260, 64, causal=True, seed=907), 0.4, 12, 0, False),
]


def _slopes(h):
    return torch.tensor([2.0 ** (-8.0 * (k + 1) / h) for k in range(h)], dtype=torch.float32)


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_dropout_parity(attn, case):
    w, p, seed, off, with_slopes = case
    q, k, v, do = make_inputs(w)
    args = (w.scale, w.causal, w.window_left, w.window_right)
    drop = dict(dropout_p=p, dropout_seed=seed, dropout_offset=off)
    sl = _slopes(w.nheads) if with_slopes else None
    slc = sl.cuda() if with_slopes else None
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, *args, alibi_slopes=slc, **drop)
    dq, dk, dv = attn.attn_bwd(qc, kc, vc, o, lse, doc, *args, alibi_slopes=slc, **drop)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    ref_sl = sl.double() if with_slopes else None
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, *args, alibi_slopes=ref_sl, **drop)
    check_o(o.cpu(), o_ref, w.name)
    check_lse(lse.cpu(), lse_ref, w.name)
    g_ref = oracle.attention_bwd(q, k, v, do, *args, alibi_slopes=ref_sl, **drop)
    for x, r, n in zip((dq, dk, dv), g_ref, ("dQ", "dK", "dV")):
        check_grad(x.cpu(), r, f"{w.name} {n}")


def test_dropout_packed_sequences(attn):
    lens = [130, 0, 257, 64]
    q, k, v, do, cu_q, cu_k = make_varlen_inputs(lens, lens, 4, 2, 128, seed=910)
    drop = dict(dropout_p=0.25, dropout_seed=4242, dropout_offset=3)
    dev = [t.cuda() for t in (q, k, v, do, cu_q, cu_k)]
    o, lse = attn.attn_fwd_varlen(dev[0], dev[1], dev[2], dev[4], dev[5], max(lens), max(lens),
                                  None, True, **drop)
    g = attn.attn_bwd_varlen(dev[0], dev[1], dev[2], o, lse, dev[3], dev[4], dev[5], max(lens),
                             max(lens), None, True, **drop)
    torch.cuda.synchronize()
    scale = 128 ** -0.5
    o_ref, lse_ref = oracle.attention_fwd_varlen(q, k, v, cu_q, cu_k, scale, True, **drop)
    check_o(o.cpu(), o_ref, "varlen dropout")
    check_lse(lse.cpu(), lse_ref, "varlen dropout")
    g_ref = oracle.attention_bwd_varlen(q, k, v, do, cu_q, cu_k, scale, True, **drop)
    for x, r, n in zip(g, g_ref, ("dQ", "dK", "dV")):
        check_grad(x.cpu(), r, "varlen dropout " + n)


def test_dropout_repeatable_and_offset_sensitive(attn):
    w = W("rep", 1, 2, 2, 256, 256, 128, causal=True, seed=911)
    q, k, v, _ = (t.cuda() for t in make_inputs(w))
    a, _ = attn.attn_fwd(q, k, v, None, True, dropout_p=0.3, dropout_seed=8, dropout_offset=0)
    b, _ = attn.attn_fwd(q, k, v, None, True, dropout_p=0.3, dropout_seed=8, dropout_offset=0)
    c, _ = attn.attn_fwd(q, k, v, None, True, dropout_p=0.3, dropout_seed=8, dropout_offset=1)
    assert torch.equal(a, b)
    assert not torch.equal(a, c)


def test_dropout_headdim_256_refused(attn):
    q = torch.zeros(1, 128, 2, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_fwd(q, q, q, dropout_p=0.1)
