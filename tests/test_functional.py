"""The differentiable wrappers (functional.py): their autograd plumbing on
the CPU, with the library calls replaced by the float64 oracle (argument
pass-through, gradient routing, the upstream gradient reaching the backward,
LSE not differentiable, the dropout seed shared by both passes); and the real
library on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import Workload, make_inputs, make_varlen_inputs


@pytest.fixture
def fake_lib(monkeypatch):
    import io_aware_exact_33_b200 as attn
    calls = []

    def fwd(q, k, v, scale, causal, wl, wr, alibi_slopes=None, **drop):
        calls.append(("fwd", scale, causal, wl, wr, alibi_slopes, drop))
        o, lse = oracle.attention_fwd(q, k, v, scale, causal, wl, wr, alibi_slopes=alibi_slopes,
                                      **drop)
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(lse).float()

    def bwd(q, k, v, o, lse, do, scale, causal, wl, wr, alibi_slopes=None, **drop):
        calls.append(("bwd", scale, causal, wl, wr, alibi_slopes, drop))
        g = oracle.attention_bwd(q, k, v, do, scale, causal, wl, wr, alibi_slopes=alibi_slopes,
                                 **drop)
        return tuple(torch.from_numpy(x).to(q.dtype) for x in g)

    def fwd_varlen(q, k, v, cu_q, cu_k, mq, mk, scale, causal, wl, wr, alibi_slopes=None, **drop):
        calls.append(("fwd_varlen", mq, mk, scale, causal, wl, wr, drop))
        o, lse = oracle.attention_fwd_varlen(q, k, v, cu_q, cu_k, scale, causal, wl, wr,
                                             alibi_slopes=alibi_slopes, **drop)
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(lse).float()

    def bwd_varlen(q, k, v, o, lse, do, cu_q, cu_k, mq, mk, scale, causal, wl, wr,
                   alibi_slopes=None, **drop):
        calls.append(("bwd_varlen", mq, mk, scale, causal, wl, wr, drop))
        g = oracle.attention_bwd_varlen(q, k, v, do, cu_q, cu_k, scale, causal, wl, wr,
                                        alibi_slopes=alibi_slopes, **drop)
        return tuple(torch.from_numpy(x).to(q.dtype) for x in g)

    monkeypatch.setattr(attn, "attn_fwd", fwd)
    monkeypatch.setattr(attn, "attn_bwd", bwd)
    monkeypatch.setattr(attn, "attn_fwd_varlen", fwd_varlen)
    monkeypatch.setattr(attn, "attn_bwd_varlen", bwd_varlen)
    return calls


def _leaf(t):
    return t.double().clone().requires_grad_(True)


def test_autograd_plumbing(fake_lib):
    from io_aware_exact_33_b200.functional import flash_attn_func
    w = Workload("f", 2, 4, 2, 9, 11, 8, True, 3, -1, "bf16", 1.0, 700)
    q, k, v, do = (_leaf(t) for t in make_inputs(w))
    slopes = torch.tensor([0.5, 0.25, 0.1, 0.0], dtype=torch.float64)
    out, lse = flash_attn_func(q, k, v, softmax_scale=0.3, causal=True, window_size=(3, -1),
                               alibi_slopes=slopes, return_lse=True)
    assert not lse.requires_grad
    (out * do.detach()).sum().backward()
    assert [c[:5] for c in fake_lib] == [("fwd", 0.3, True, 3, -1), ("bwd", 0.3, True, 3, -1)]
    o_r, _ = oracle.attention_fwd(q.detach(), k.detach(), v.detach(), 0.3, True, 3, -1,
                                  alibi_slopes=slopes)
    g_r = oracle.attention_bwd(q.detach(), k.detach(), v.detach(), do.detach(), 0.3, True, 3, -1,
                               alibi_slopes=slopes)
    assert np.array_equal(out.detach().numpy(), o_r)
    for t, r in zip((q, k, v), g_r):
        assert np.array_equal(t.grad.numpy(), r)


def test_varlen_autograd_plumbing(fake_lib):
    from io_aware_exact_33_b200.functional import flash_attn_varlen_func
    q, k, v, do, cu_q, cu_k = make_varlen_inputs([5, 0, 9], [7, 4, 9], 4, 2, 8, seed=701)
    q, k, v = _leaf(q), _leaf(k), _leaf(v)
    out = flash_attn_varlen_func(q, k, v, cu_q, cu_k, 9, 9, softmax_scale=0.4, causal=True)
    (out * do.double()).sum().backward()
    assert [c[0] for c in fake_lib] == ["fwd_varlen", "bwd_varlen"]
    g_r = oracle.attention_bwd_varlen(q.detach(), k.detach(), v.detach(), do, cu_q, cu_k, 0.4,
                                      True)
    for t, r in zip((q, k, v), g_r):
        assert np.array_equal(t.grad.numpy(), r)


def test_dropout_and_window_arguments():
    from io_aware_exact_33_b200.functional import flash_attn_func
    q = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError):
        flash_attn_func(q, q, q, dropout_p=1.0)
    with pytest.raises(ValueError):
        flash_attn_func(q, q, q, window_size=(-2, 0))


def test_dropout_seed_shared_by_both_passes(fake_lib):
    """The forward draws one seed (repeatable under torch.manual_seed) and
    the backward gets the same seed and offset; the gradients are those of
    the oracle with that mask."""
    from io_aware_exact_33_b200.functional import flash_attn_func
    w = Workload("fd", 1, 2, 1, 8, 8, 8, True, -1, -1, "bf16", 1.0, 703)
    q, k, v, do = (_leaf(t) for t in make_inputs(w))
    torch.manual_seed(5)
    out = flash_attn_func(q, k, v, dropout_p=0.3, softmax_scale=0.5, causal=True)
    (out * do.detach()).sum().backward()
    (f, b) = fake_lib
    assert f[0] == "fwd" and b[0] == "bwd" and f[6] == b[6]
    drop = f[6]
    assert drop["dropout_p"] == 0.3 and drop["dropout_offset"] == 0
    torch.manual_seed(5)
    out2 = flash_attn_func(q.detach(), k.detach(), v.detach(), dropout_p=0.3, softmax_scale=0.5,
                           causal=True)
    assert torch.equal(out.detach(), out2) and fake_lib[2][6] == drop
    g = oracle.attention_bwd(q.detach(), k.detach(), v.detach(), do.detach(), 0.5, True, **drop)
    for t, r in zip((q, k, v), g):
        assert np.array_equal(t.grad.numpy(), r)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
def test_functional_on_gpu(d):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_33_b200.functional import flash_attn_func
    from parity import check_grad, check_o
    w = Workload("fg", 2, 4, 2, 300, 300, d, True, -1, -1, "bf16", 1.0, 702)
    q0, k0, v0, do0 = make_inputs(w)
    q, k, v = (t.cuda().requires_grad_(True) for t in (q0, k0, v0))
    out = flash_attn_func(q, k, v, causal=True)
    out.backward(do0.cuda())
    torch.cuda.synchronize()
    o_r, _ = oracle.attention_fwd(q0, k0, v0, w.scale, True)
    check_o(out.detach().cpu(), o_r, "functional")
    for t, r, n in zip((q, k, v), oracle.attention_bwd(q0, k0, v0, do0, w.scale, True),
                       ("dQ", "dK", "dV")):
        check_grad(t.grad.cpu(), r, "functional " + n)
