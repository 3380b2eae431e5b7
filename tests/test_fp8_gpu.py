"""The E4M3 (FP8) forward on the GPU against the float64 oracle over the
dequantized inputs (codes made by the oracle's E4M3 codec with one scale per
tensor).

Tolerance, derived from the kernel's arithmetic: the products q8 k8 are
exact in the f32 accumulator and l sums the unrounded P, so the output's
error comes from P rounded to E4M3 before the P V product: at most 2^-4
relative for P >= 2^-6 and 2^-10 absolute below, in the kernel's units where
the row's largest P is >= 1.  Hence, per element,
    |O - O_ref| <= 2^-4 sum_j P_ij |V_j| + 2^-10 n_i max|V| / l_i
                   + half an ulp of the output + 1e-3,
with P, l_i = sum_j exp(s_ij - max_j s_ij) and the n_i visible keys taken
from the dequantized inputs.  The LSE uses unrounded values: 1e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import Workload, make_inputs
from oracle_pins import mask_matrix
from parity import check_lse, half_ulp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def W(name, B, H, Hkv, Nq, Nk, causal=False, wl=-1, wr=-1, seed=950):
    return Workload(name, B, H, Hkv, Nq, Nk, 128, causal, wl, wr, "bf16", 1.0, seed)


CASES = [
    (W("causal_gqa", 2, 4, 2, 300, 300, causal=True, seed=951), "bf16"),
    (W("full_fp16_out", 1, 4, 4, 520, 520, seed=952), "fp16"),
    (W("window", 1, 4, 2, 700, 700, causal=True, wl=129, seed=953), "bf16"),
    (W("nq_lt_nk", 1, 2, 2, 100, 390, causal=True, seed=954), "bf16"),
    (W("nq_gt_nk", 1, 2, 1, 260, 130, seed=955), "bf16"),
]


def quantize(x):
    """Codes and scale (amax / 448) of one tensor, by the oracle's codec."""
    scale = float(x.double().abs().max()) / 448.0
    codes = oracle.e4m3_quantize(x, scale)
    return torch.from_numpy(codes), scale, oracle.e4m3_dequantize(codes, scale)


def bound(qd, kd, vd, w):
    """The derived per-element tolerance (module docstring) in (B, Nq, H, d)."""
    q, k, v = (torch.from_numpy(a) for a in (qd, kd, vd))
    g = w.nheads // w.nheads_kv
    k = k.repeat_interleave(g, dim=2)
    v = v.repeat_interleave(g, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", q, k) * w.scale
    vis = torch.from_numpy(mask_matrix(w.seqlen_q, w.seqlen_k, causal=w.causal,
                                       window_left=w.window_left, window_right=w.window_right))
    s = s.masked_fill(~vis, -math.inf)
    mx = s.amax(-1, keepdim=True).clamp_min(-1e300)
    e = torch.exp(s - mx)
    l = e.sum(-1, keepdim=True)
    prob = e / l
    pabs = torch.einsum("bhij,bjhd->bihd", prob, v.abs())
    n_vis = vis.sum(-1).double()  # (Nq,)
    sub = (2.0 ** -10) * n_vis[None, None, :] * float(v.abs().max()) / l[..., 0]  # (B, H, Nq)
    return (2.0 ** -4) * pabs.numpy() + sub.permute(0, 2, 1)[..., None].numpy()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_e4m3_forward_parity(attn, case):
    w, out = case
    q, k, v, _ = make_inputs(w, with_dout=False)
    (q8, qs, qd), (k8, ks, kd), (v8, vs, vd) = quantize(q), quantize(k), quantize(v)
    out_dtype = torch.float16 if out == "fp16" else torch.bfloat16
    o, lse = attn.attn_fwd_e4m3(q8.cuda(), k8.cuda(), v8.cuda(), qs, ks, vs, w.scale, w.causal,
                                w.window_left, w.window_right, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd(qd, kd, vd, w.scale, w.causal, w.window_left,
                                          w.window_right)
    og = o.cpu().double().numpy()
    tol = bound(qd, kd, vd, w) + half_ulp(o_ref, out_dtype) + 1e-3
    err = np.abs(og - o_ref)
    assert np.isfinite(og).all()
    assert (err <= tol).all(), f"{w.name}: max excess {np.max(err - tol):.3e}"
    # the rounding of P is unbiased: the mean error is far below the bound
    assert err.mean() <= 0.25 * tol.mean(), (err.mean(), tol.mean())
    check_lse(lse.cpu(), lse_ref, w.name)


def test_e4m3_forward_matches_bf16_kernel(attn):
    """Power-of-two scales make the dequantized inputs exact in bf16: the
    16-bit kernel on them and the E4M3 kernel differ only by P's rounding."""
    w = W("pow2", 1, 4, 4, 256, 256, causal=True, seed=956)
    q, k, v, _ = make_inputs(w, with_dout=False)
    outs = []
    for x in (q, k, v):
        scale = 2.0 ** math.ceil(math.log2(float(x.double().abs().max()) / 448.0))
        codes = oracle.e4m3_quantize(x, scale)
        outs.append((torch.from_numpy(codes), scale,
                     torch.from_numpy(oracle.e4m3_dequantize(codes, scale))))
    (q8, qs, qd), (k8, ks, kd), (v8, vs, vd) = outs
    assert all(torch.equal(t.to(torch.bfloat16).double(), t) for t in (qd, kd, vd))
    o8, l8 = attn.attn_fwd_e4m3(q8.cuda(), k8.cuda(), v8.cuda(), qs, ks, vs, w.scale, True)
    o16, l16 = attn.attn_fwd(qd.to(torch.bfloat16).cuda(), kd.to(torch.bfloat16).cuda(),
                             vd.to(torch.bfloat16).cuda(), w.scale, True)
    torch.cuda.synchronize()
    assert (l8 - l16).abs().max().item() <= 1e-3
    tol = bound(qd.numpy(), kd.numpy(), vd.numpy(), w) + 2e-2
    assert ((o8.double() - o16.double()).abs().cpu().numpy() <= tol).all()


def test_e4m3_no_keys_and_rejects(attn):
    q8 = torch.zeros(1, 64, 2, 128, dtype=torch.uint8, device="cuda")
    k8 = torch.zeros(1, 0, 2, 128, dtype=torch.uint8, device="cuda")
    o, lse = attn.attn_fwd_e4m3(q8, k8, k8, 1.0, 1.0, 1.0)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isinf(lse))
    q64 = torch.zeros(1, 64, 2, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_e4m3(q64, q64, q64, 1.0, 1.0, 1.0)
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_e4m3(q8, q8, q8, 0.0, 1.0, 1.0)
