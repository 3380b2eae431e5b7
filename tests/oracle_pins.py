"""Checks that pin the float64 oracle to facts outside itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with a closed form, a hand-worked value, brute-force
finite differences, an independent library routine, or an invariant of the
definition.  ``test_oracle_pins.py`` runs them on the oracle; the mutation
test runs them on copies of the oracle with a planted mistake and requires
each copy to fail at least one.

Passages: the definition Softmax(QK^T/sqrt(d))V ("FlashAttention ...
transformer optimization", technical deep dive); causal and sliding-window
masks (FlashAttention-2 page, section 3 and the sparse-attention extension);
MQA/GQA (page 5, hardware/dtype section); the backward pass recomputes scores
(page 2, item 2) and so has the analytic gradient of the definition.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

MASKS = [
    dict(causal=False, window_left=-1, window_right=-1),
    dict(causal=True, window_left=-1, window_right=-1),
    dict(causal=True, window_left=3, window_right=-1),
    dict(causal=False, window_left=2, window_right=1),
    dict(causal=False, window_left=-1, window_right=0),
    dict(causal=False, window_left=0, window_right=2),
]


def _visible(i, j, nq, nk, causal, window_left, window_right):
    ii = i + nk - nq
    if causal and j > ii:
        return False
    if window_left >= 0 and j < ii - window_left:
        return False
    if window_right >= 0 and j > ii + window_right:
        return False
    return True


def mask_matrix(nq, nk, **m):
    """Boolean visibility matrix built from the mask reading, by brute force."""
    return np.array([[_visible(i, j, nq, nk, **m) for j in range(nk)] for i in range(nq)])


def rand(shape, seed, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64).to(dtype)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), f"{what}: non-finite pattern differs"
    assert np.array_equal(a[~fin], b[~fin]), f"{what}: infinities differ"
    err = np.max(np.abs(a[fin] - b[fin])) if fin.any() else 0.0
    assert err <= tol, f"{what}: max err {err:.3e} > {tol:.1e}"


# --- closed forms -----------------------------------------------------------

def pin_golden_handworked(orc):
    """Values worked by hand from the definition (tests/golden/handworked_2x2.txt)."""
    vals = {}
    with open(os.path.join(GOLDEN, "handworked_2x2.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                key, *nums = line.split()
                vals[key] = [float(x) for x in nums]
    B, H, Hkv, Nq, Nk, d = (int(x) for x in vals["shape"])
    scale = vals["scale"][0]
    q = torch.tensor(vals["q"], dtype=torch.float64).reshape(B, Nq, H, d)
    k = torch.tensor(vals["k"], dtype=torch.float64).reshape(B, Nk, Hkv, d)
    v = torch.tensor(vals["v"], dtype=torch.float64).reshape(B, Nk, Hkv, d)
    do = torch.tensor(vals["dout"], dtype=torch.float64).reshape(B, Nq, H, d)
    for name, causal in (("noncausal", False), ("causal", True)):
        o, lse = orc.attention_fwd(q, k, v, scale, causal)
        dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, causal)
        _close(o.ravel(), vals[name + ".o"], 1e-12, name + ".o")
        _close(lse.ravel(), vals[name + ".lse"], 1e-12, name + ".lse")
        _close(dq.ravel(), vals[name + ".dq"], 1e-12, name + ".dq")
        _close(dk.ravel(), vals[name + ".dk"], 1e-12, name + ".dk")
        _close(dv.ravel(), vals[name + ".dv"], 1e-12, name + ".dv")


def pin_identical_keys(orc):
    """All keys equal: every visible key has the same score s, so the softmax
    is uniform: O_i = mean of the visible V_j and LSE_i = s + ln(count)."""
    B, H, Hkv, Nq, Nk, d = 2, 4, 2, 7, 9, 5
    q = rand((B, Nq, H, d), 1)
    kvec = rand((B, 1, Hkv, d), 2)
    k = kvec.expand(B, Nk, Hkv, d).contiguous()
    v = rand((B, Nk, Hkv, d), 3)
    scale = 0.37
    for m in MASKS:
        o, lse = orc.attention_fwd(q, k, v, scale, **m)
        vis = mask_matrix(Nq, Nk, **m)
        for b in range(B):
            for h in range(H):
                g = h // (H // Hkv)
                for i in range(Nq):
                    js = np.nonzero(vis[i])[0]
                    if len(js) == 0:
                        exp_o, exp_l = np.zeros(d), -math.inf
                    else:
                        exp_o = v[b, js, g].numpy().mean(axis=0)
                        s = scale * float(q[b, i, h] @ kvec[b, 0, g])
                        exp_l = s + math.log(len(js))
                    _close(o[b, i, h], exp_o, 1e-12, f"identical keys O {m}")
                    _close([lse[b, h, i]], [exp_l], 1e-12, f"identical keys LSE {m}")


def pin_constant_values(orc):
    """V_j = c for every key: the weights sum to one, so O_i = c on every row
    with a visible key."""
    B, H, Hkv, Nq, Nk, d = 1, 2, 1, 6, 6, 4
    q, k = rand((B, Nq, H, d), 4), rand((B, Nk, Hkv, d), 5)
    c = torch.tensor([1.5, -2.0, 0.25, 3.0], dtype=torch.float64)
    v = c.expand(B, Nk, Hkv, d).contiguous()
    for m in MASKS:
        o, _ = orc.attention_fwd(q, k, v, 0.8, **m)
        vis = mask_matrix(Nq, Nk, **m)
        for i in range(Nq):
            exp = c.numpy() if vis[i].any() else np.zeros(d)
            _close(o[0, i], np.broadcast_to(exp, (H, d)), 1e-13, f"constant V {m}")


def pin_causal_first_row(orc):
    """Under the causal mask, query 0 sees key 0 only: O_0 = V_0 exactly and
    LSE_0 = scale * q_0 . k_0."""
    B, H, N, d = 2, 3, 8, 6
    q, k, v = rand((B, N, H, d), 6), rand((B, N, H, d), 7), rand((B, N, H, d), 8)
    o, lse = orc.attention_fwd(q, k, v, 0.5, causal=True)
    assert np.array_equal(o[:, 0], v[:, 0].numpy())
    s00 = 0.5 * torch.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]).numpy()
    _close(lse[:, :, 0], s00, 1e-14, "causal LSE_0")


def pin_window_zero(orc):
    """Causal with window_left = 0: each query sees only its own key, so
    O_i = V_i; and a window at least N wide reduces to plain causal."""
    B, H, N, d = 1, 2, 9, 4
    q, k, v = rand((B, N, H, d), 9), rand((B, N, H, d), 10), rand((B, N, H, d), 11)
    o, _ = orc.attention_fwd(q, k, v, 1.1, causal=True, window_left=0)
    assert np.array_equal(o, v.numpy())
    o1, l1 = orc.attention_fwd(q, k, v, 1.1, causal=True, window_left=N)
    o2, l2 = orc.attention_fwd(q, k, v, 1.1, causal=True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# --- a different algorithm --------------------------------------------------

def _online_softmax_attention(q, k, v, scale, vis, block):
    """Blockwise single pass with a running max and running sum, written here
    independently of the oracle: the online softmax the pages describe
    (FlashAttention-2 page; page 2's "running maximum and normalisation
    factor"), in float64, one head."""
    nq, nk = vis.shape
    o = np.zeros((nq, v.shape[1]))
    lse = np.full(nq, -np.inf)
    for i in range(nq):
        m, l, acc = -np.inf, 0.0, np.zeros(v.shape[1])
        for j0 in range(0, nk, block):
            js = [j for j in range(j0, min(nk, j0 + block)) if vis[i, j]]
            if not js:
                continue
            s = scale * (k[js] @ q[i])
            m_new = max(m, s.max())
            alpha = math.exp(m - m_new) if m > -np.inf else 0.0
            p = np.exp(s - m_new)
            l = l * alpha + p.sum()
            acc = acc * alpha + p @ v[js]
            m = m_new
        if l > 0:
            o[i] = acc / l
            lse[i] = m + math.log(l)
    return o, lse


def pin_online_equals_two_pass(orc):
    B, H, Hkv, Nq, Nk, d = 1, 2, 1, 11, 13, 6
    q, k, v = rand((B, Nq, H, d), 12), rand((B, Nk, Hkv, d), 13), rand((B, Nk, Hkv, d), 14)
    q = q * 3.0  # wide score range exercises the rescaling
    for m in MASKS:
        o, lse = orc.attention_fwd(q, k, v, 0.6, **m)
        vis = mask_matrix(Nq, Nk, **m)
        for block in (1, 7, 128):
            for h in range(H):
                eo, el = _online_softmax_attention(q[0, :, h].numpy(), k[0, :, 0].numpy(),
                                                   v[0, :, 0].numpy(), 0.6, vis, block)
                _close(o[0, :, h], eo, 1e-12, f"online O {m} block {block}")
                _close(lse[0, h], el, 1e-12, f"online LSE {m} block {block}")


# --- an independent library routine -------------------------------------------

def pin_torch_sdpa(orc):
    """torch's scaled_dot_product_attention on the CPU in float64 with an
    explicit boolean mask and repeat-interleaved K/V, and its autograd
    gradients, on rows that see at least one key."""
    import torch.nn.functional as F
    B, H, Hkv, Nq, Nk, d = 2, 4, 2, 10, 10, 8
    q, k, v = rand((B, Nq, H, d), 15), rand((B, Nk, Hkv, d), 16), rand((B, Nk, Hkv, d), 17)
    do = rand((B, Nq, H, d), 18)
    scale = 0.3
    for m in MASKS:
        vis = mask_matrix(Nq, Nk, **m)
        if not vis.any(axis=1).all():
            continue
        qt = q.permute(0, 2, 1, 3).clone().requires_grad_(True)
        kt = k.permute(0, 2, 1, 3).clone().requires_grad_(True)
        vt = v.permute(0, 2, 1, 3).clone().requires_grad_(True)
        rep = H // Hkv
        out = F.scaled_dot_product_attention(
            qt, kt.repeat_interleave(rep, dim=1), vt.repeat_interleave(rep, dim=1),
            attn_mask=torch.from_numpy(vis), scale=scale)
        (out * do.permute(0, 2, 1, 3)).sum().backward()
        o, _ = orc.attention_fwd(q, k, v, scale, **m)
        dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, **m)
        _close(o, out.detach().permute(0, 2, 1, 3).numpy(), 1e-10, f"sdpa O {m}")
        _close(dq, qt.grad.permute(0, 2, 1, 3).numpy(), 1e-10, f"sdpa dQ {m}")
        _close(dk, kt.grad.permute(0, 2, 1, 3).numpy(), 1e-10, f"sdpa dK {m}")
        _close(dv, vt.grad.permute(0, 2, 1, 3).numpy(), 1e-10, f"sdpa dV {m}")


# --- brute force -------------------------------------------------------------

def pin_finite_differences(orc):
    """Central differences of L = sum(O o dO) with respect to every element of
    Q, K and V agree with the analytic gradients (tiny shapes, every mask,
    Nq != Nk, MHA and GQA)."""
    h = 1e-6
    for (Hkv, Nq, Nk, d, seed) in ((2, 5, 5, 3, 20), (1, 4, 7, 2, 21), (1, 7, 4, 3, 22)):
        B, H = 1, 2
        q, k, v = rand((B, Nq, H, d), seed), rand((B, Nk, Hkv, d), seed + 1), rand((B, Nk, Hkv, d), seed + 2)
        do = rand((B, Nq, H, d), seed + 3)
        for m in MASKS:
            dq, dk, dv = orc.attention_bwd(q, k, v, do, 0.7, **m)

            def loss(qq, kk, vv):
                o, _ = orc.attention_fwd(qq, kk, vv, 0.7, **m)
                return float((o * do.numpy()).sum())

            for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
                fd = np.zeros(x.shape)
                flat = x.reshape(-1)
                for idx in range(flat.numel()):
                    xp, xm = flat.clone(), flat.clone()
                    xp[idx] += h
                    xm[idx] -= h
                    args = {"q": q, "k": k, "v": v}
                    args[name] = xp.reshape(x.shape)
                    lp = loss(args["q"], args["k"], args["v"])
                    args[name] = xm.reshape(x.shape)
                    lm = loss(args["q"], args["k"], args["v"])
                    fd.reshape(-1)[idx] = (lp - lm) / (2 * h)
                scale_ref = max(1.0, np.abs(fd).max())
                err = np.abs(fd - g).max() / scale_ref
                assert err <= 1e-6, f"finite differences d{name} {m} Nq={Nq} Nk={Nk}: {err:.2e}"


# --- invariants --------------------------------------------------------------

def pin_invariants(orc):
    """Adding a constant to every score of a row leaves O unchanged and shifts
    LSE by it; permuting keys and values together leaves O unchanged (no mask);
    the rows of P sum to one (O of a one-hot V picks out a column of P whose
    sum over V's columns is one)."""
    B, H, N, d = 1, 2, 8, 4
    q, k, v = rand((B, N, H, d), 30), rand((B, N, H, d), 31), rand((B, N, H, d), 32)
    scale = 0.9
    # shift: an extra feature with q = 1 and k = c for every key adds scale*c.
    c = 2.5
    q2 = torch.cat([q, torch.ones(B, N, H, 1, dtype=torch.float64)], dim=-1)
    k2 = torch.cat([k, torch.full((B, N, H, 1), c, dtype=torch.float64)], dim=-1)
    v2 = torch.cat([v, torch.zeros(B, N, H, 1, dtype=torch.float64)], dim=-1)
    for m in MASKS:
        o1, l1 = orc.attention_fwd(q, k, v, scale, **m)
        o2, l2 = orc.attention_fwd(q2, k2, v2, scale, **m)
        _close(o2[..., :d], o1, 1e-12, f"shift O {m}")
        fin = np.isfinite(l1)
        _close(l2[fin], l1[fin] + scale * c, 1e-12, f"shift LSE {m}")
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(33))
    o1, l1 = orc.attention_fwd(q, k, v, scale)
    o2, l2 = orc.attention_fwd(q, k[:, perm], v[:, perm], scale)
    _close(o2, o1, 1e-12, "permutation O")
    _close(l2, l1, 1e-12, "permutation LSE")
    # one-hot values (head dim = N, so q and k are drawn at that width too)
    q3, k3 = rand((B, N, H, N), 34), rand((B, N, H, N), 35)
    eye = torch.eye(N, dtype=torch.float64).reshape(1, N, 1, N).expand(B, N, H, N).contiguous()
    for m in MASKS:
        pmat, _ = orc.attention_fwd(q3, k3, eye, scale, **m)
        vis = mask_matrix(N, N, **m)
        rows = pmat.sum(axis=-1)
        _close(rows, np.where(vis.any(axis=1), 1.0, 0.0)[None, :, None].repeat(H, axis=2), 1e-13,
               f"rows of P {m}")
        for h in range(H):
            assert np.all(pmat[0, :, h, :][~vis] == 0.0), f"masked entries of P {m}"


def pin_gqa_equals_repeated_mha(orc):
    """GQA equals MHA on K/V repeated per query head; dK/dV of a kv head is
    the sum over its query heads."""
    B, H, Hkv, N, d = 2, 6, 2, 7, 4
    q, k, v = rand((B, N, H, d), 40), rand((B, N, Hkv, d), 41), rand((B, N, Hkv, d), 42)
    do = rand((B, N, H, d), 43)
    rep = H // Hkv
    kr, vr = k.repeat_interleave(rep, dim=2), v.repeat_interleave(rep, dim=2)
    for m in MASKS:
        o1, l1 = orc.attention_fwd(q, k, v, 0.5, **m)
        o2, l2 = orc.attention_fwd(q, kr, vr, 0.5, **m)
        _close(o1, o2, 0.0, f"gqa O {m}")
        _close(l1, l2, 0.0, f"gqa LSE {m}")
        dq1, dk1, dv1 = orc.attention_bwd(q, k, v, do, 0.5, **m)
        dq2, dk2, dv2 = orc.attention_bwd(q, kr, vr, do, 0.5, **m)
        _close(dq1, dq2, 1e-14, f"gqa dQ {m}")
        _close(dk1, dk2.reshape(B, N, Hkv, rep, d).sum(axis=3), 1e-13, f"gqa dK {m}")
        _close(dv1, dv2.reshape(B, N, Hkv, rep, d).sum(axis=3), 1e-13, f"gqa dV {m}")


def pin_empty_rows(orc):
    """A query with no visible key (causal with Nq > Nk) gets O = 0,
    LSE = -inf and zero gradients; its dO contributes nothing."""
    B, H, Nq, Nk, d = 1, 1, 6, 3, 2
    q, k, v = rand((B, Nq, H, d), 50), rand((B, Nk, H, d), 51), rand((B, Nk, H, d), 52)
    do = rand((B, Nq, H, d), 53)
    o, lse = orc.attention_fwd(q, k, v, 1.0, causal=True)
    # off = Nk - Nq = -3: rows 0..2 see nothing.
    assert np.all(o[:, :3] == 0.0) and np.all(lse[:, :, :3] == -np.inf)
    assert np.all(np.isfinite(lse[:, :, 3:]))
    dq, dk, dv = orc.attention_bwd(q, k, v, do, 1.0, causal=True)
    assert np.all(dq[:, :3] == 0.0)
    do2 = do.clone()
    do2[:, :3] = 100.0
    _, dk2, dv2 = orc.attention_bwd(q, k, v, do2, 1.0, causal=True)
    assert np.array_equal(dk, dk2) and np.array_equal(dv, dv2)


def pin_rows_match_full(orc):
    """The sampled-row entry points return exactly the full entry points'
    rows, with and without positional slopes."""
    B, H, Hkv, Nq, Nk, d = 2, 4, 2, 9, 11, 3
    q, k, v = rand((B, Nq, H, d), 60), rand((B, Nk, Hkv, d), 61), rand((B, Nk, Hkv, d), 62)
    do = rand((B, Nq, H, d), 63)
    qrows, krows = [0, 3, 8], [1, 10, 5]
    for slopes in (None, [0.5, 0.1, 0.02, 1.5]):
        for m in MASKS:
            kw = dict(m, alibi_slopes=slopes)
            o, lse = orc.attention_fwd(q, k, v, 0.4, **kw)
            o_r, lse_r = orc.attention_fwd_rows(q, k, v, qrows, 0.4, **kw)
            assert np.array_equal(o[:, qrows], o_r) and np.array_equal(lse[:, :, qrows], lse_r)
            dq, dk, dv = orc.attention_bwd(q, k, v, do, 0.4, **kw)
            dq_r, dk_r, dv_r = orc.attention_bwd_rows(q, k, v, do, qrows, krows, 0.4, **kw)
            _close(dq_r, dq[:, qrows], 1e-13, f"rows dQ {m} {slopes}")
            _close(dk_r, dk[:, krows], 1e-13, f"rows dK {m} {slopes}")
            _close(dv_r, dv[:, krows], 1e-13, f"rows dV {m} {slopes}")


def pin_varlen_per_sequence(orc):
    """Packed sequences: every sequence's rows equal torch's scaled dot
    product attention (float64, explicit bottom-right mask, autograd
    gradients) run on that sequence alone, with query and key lengths that
    differ per sequence, an empty query sequence and an empty key sequence;
    rows of a sequence with no keys get O = 0, LSE = -inf and zero
    gradients."""
    import torch.nn.functional as F
    H, Hkv, d, scale = 4, 2, 8, 0.35
    lq = [5, 0, 9, 3, 7]
    lk = [7, 4, 9, 0, 2]
    cq = np.concatenate([[0], np.cumsum(lq)]).tolist()
    ck = np.concatenate([[0], np.cumsum(lk)]).tolist()
    q, k, v = rand((cq[-1], H, d), 70), rand((ck[-1], Hkv, d), 71), rand((ck[-1], Hkv, d), 72)
    do = rand((cq[-1], H, d), 73)
    for m in MASKS:
        o, lse = orc.attention_fwd_varlen(q, k, v, cq, ck, scale, **m)
        dq, dk, dv = orc.attention_bwd_varlen(q, k, v, do, cq, ck, scale, **m)
        assert o.shape == (cq[-1], H, d) and lse.shape == (H, cq[-1])
        for b in range(len(lq)):
            q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
            if q1 == q0:
                continue
            if k1 == k0:
                assert np.all(o[q0:q1] == 0.0) and np.all(lse[:, q0:q1] == -np.inf)
                assert np.all(dq[q0:q1] == 0.0)
                continue
            vis = mask_matrix(q1 - q0, k1 - k0, **m)
            seen = vis.any(axis=1)
            qt = q[q0:q1].permute(1, 0, 2)[None].clone().requires_grad_(True)
            kt = k[k0:k1].permute(1, 0, 2)[None].clone().requires_grad_(True)
            vt = v[k0:k1].permute(1, 0, 2)[None].clone().requires_grad_(True)
            rep = H // Hkv
            # rows with no visible key are left out of the library call
            out = F.scaled_dot_product_attention(
                qt[:, :, seen], kt.repeat_interleave(rep, dim=1),
                vt.repeat_interleave(rep, dim=1), attn_mask=torch.from_numpy(vis[seen]),
                scale=scale)
            (out * do[q0:q1][seen].permute(1, 0, 2)[None]).sum().backward()
            _close(o[q0:q1][seen], out.detach()[0].permute(1, 0, 2).numpy(), 1e-10,
                   f"varlen O seq {b} {m}")
            assert np.all(o[q0:q1][~seen] == 0.0)
            _close(dq[q0:q1], qt.grad[0].permute(1, 0, 2).numpy(), 1e-10, f"varlen dQ {b} {m}")
            _close(dk[k0:k1], kt.grad[0].permute(1, 0, 2).numpy(), 1e-10, f"varlen dK {b} {m}")
            _close(dv[k0:k1], vt.grad[0].permute(1, 0, 2).numpy(), 1e-10, f"varlen dV {b} {m}")


def alibi_bias(nq, nk, slopes):
    """-slope_h * |i + Nk - Nq - j| for every head, query and key (H, Nq, Nk),
    written out by brute force."""
    out = np.zeros((len(slopes), nq, nk))
    for h, sl in enumerate(slopes):
        for i in range(nq):
            for j in range(nk):
                out[h, i, j] = -sl * abs(i + nk - nq - j)
    return out


def pin_alibi_sdpa(orc):
    """Per-head positional slopes: torch's scaled dot product attention with
    the bias written into a float mask (-inf where hidden), and its autograd
    gradients, for every mask, GQA and Nq != Nk; zero slopes give exactly
    the unbiased result."""
    import torch.nn.functional as F
    B, H, Hkv, d, scale = 2, 4, 2, 8, 0.3
    slopes = [0.5, 0.25, 0.125, 0.0625]
    for nq, nk in ((10, 10), (6, 11), (9, 7)):
        q, k, v = rand((B, nq, H, d), 80), rand((B, nk, Hkv, d), 81), rand((B, nk, Hkv, d), 82)
        do = rand((B, nq, H, d), 83)
        bias = alibi_bias(nq, nk, slopes)
        for m in MASKS:
            vis = mask_matrix(nq, nk, **m)
            seen = vis.any(axis=1)
            o, lse = orc.attention_fwd(q, k, v, scale, alibi_slopes=slopes, **m)
            dq, dk, dv = orc.attention_bwd(q, k, v, do, scale, alibi_slopes=slopes, **m)
            if not seen.any():
                continue
            qt = q.permute(0, 2, 1, 3)[:, :, seen].clone().requires_grad_(True)
            kt = k.permute(0, 2, 1, 3).clone().requires_grad_(True)
            vt = v.permute(0, 2, 1, 3).clone().requires_grad_(True)
            rep = H // Hkv
            fmask = torch.from_numpy(np.where(vis[seen][None], bias[:, seen], -np.inf))
            out = F.scaled_dot_product_attention(
                qt, kt.repeat_interleave(rep, dim=1), vt.repeat_interleave(rep, dim=1),
                attn_mask=fmask[None], scale=scale)
            (out * do.permute(0, 2, 1, 3)[:, :, seen]).sum().backward()
            what = f"alibi {nq}x{nk} {m}"
            _close(o[:, seen], out.detach().permute(0, 2, 1, 3).numpy(), 1e-10, what + " O")
            assert np.all(o[:, ~seen] == 0.0)
            _close(dq[:, seen], qt.grad.permute(0, 2, 1, 3).numpy(), 1e-10, what + " dQ")
            _close(dk, kt.grad.permute(0, 2, 1, 3).numpy(), 1e-10, what + " dK")
            _close(dv, vt.grad.permute(0, 2, 1, 3).numpy(), 1e-10, what + " dV")
            o0, lse0 = orc.attention_fwd(q, k, v, scale, alibi_slopes=[0.0] * H, **m)
            o1, lse1 = orc.attention_fwd(q, k, v, scale, **m)
            assert np.array_equal(o0, o1) and np.array_equal(lse0, lse1)


def pin_merge_of_key_chunks(orc):
    """Merging the oracle's results over disjoint key chunks (one of them
    empty) equals the oracle over all keys: non-causal with GQA, and the
    causal split-KV decoding shape (queries at the end of the keys, causal
    only in the last chunk, which holds them)."""
    B, H, Hkv, d = 2, 4, 2, 8
    for nq, nk, causal, cuts in ((7, 23, False, (0, 5, 5, 16, 23)),
                                 (3, 29, True, (0, 11, 20, 29))):
        q, k, v = rand((B, nq, H, d), 90), rand((B, nk, Hkv, d), 91), rand((B, nk, Hkv, d), 92)
        o_full, lse_full = orc.attention_fwd(q, k, v, 0.37, causal=causal)
        parts_o, parts_l = [], []
        for a, z in zip(cuts, cuts[1:]):
            last = z == nk
            o_p, l_p = orc.attention_fwd(q, k[:, a:z], v[:, a:z], 0.37, causal=causal and last)
            parts_o.append(o_p)
            parts_l.append(l_p)
        o_m, lse_m = orc.attention_merge(np.stack(parts_o), np.stack(parts_l))
        _close(o_m, o_full, 1e-12, f"merge O causal={causal}")
        _close(lse_m, lse_full, 1e-12, f"merge LSE causal={causal}")
    # a row no part sees: O = 0, LSE = -inf
    o_m, lse_m = orc.attention_merge(np.zeros((2, 1, 1, 1, 4)), np.full((2, 1, 1, 1), -np.inf))
    assert np.all(o_m == 0.0) and np.all(lse_m == -np.inf)


ALL_PINS = [
    pin_golden_handworked,
    pin_identical_keys,
    pin_constant_values,
    pin_causal_first_row,
    pin_window_zero,
    pin_online_equals_two_pass,
    pin_torch_sdpa,
    pin_finite_differences,
    pin_invariants,
    pin_gqa_equals_repeated_mha,
    pin_empty_rows,
    pin_rows_match_full,
    pin_varlen_per_sequence,
    pin_alibi_sdpa,
    pin_merge_of_key_chunks,
]
