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


# --- dropout -----------------------------------------------------------------
# Dropout on the attention probabilities is named on page 5 (hardware/dtype
# section) without a formula; the oracle's reading is inverted dropout with
# the drop decisions of a Philox4x32-10 counter-based generator (see
# attn_oracle.c).  The generator is pinned to cuRAND's host-side Philox
# generator (run, not read); the arithmetic to unbiasedness, finite
# differences and the no-dropout special case.

def _curand_philox_groups(seed, ngroups):
    """cuRAND's host generator (PHILOX4_32_10, default ordering) for a 64-bit
    seed: its first ngroups blocks of four 32-bit outputs."""
    import ctypes
    lib = ctypes.CDLL("libcurand.so")
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0  # PHILOX4_32_10
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        buf = (ctypes.c_uint32 * (4 * ngroups))()
        assert lib.curandGenerate(gen, buf, ctypes.c_size_t(4 * ngroups)) == 0
        out = list(buf)
    finally:
        lib.curandDestroyGenerator(gen)
    return [out[4 * g:4 * g + 4] for g in range(ngroups)]


def pin_philox_against_curand(orc):
    """The oracle's Philox4x32-10 equals cuRAND's host generator, whose g-th
    block of four outputs is the generator at counter (0, 0, g, 0) under key
    (seed low word, seed high word)."""
    for seed in (0x123456789ABCDEF0, 0, 42, 2 ** 64 - 1, 0x0F1E2D3C4B5A6978):
        key = (seed & 0xFFFFFFFF, seed >> 32)
        for g, want in enumerate(_curand_philox_groups(seed, 48)):
            got = orc.philox4x32_10((0, 0, g, 0), key)
            assert got == want, f"philox seed={seed:#x} counter word2={g}: {got} != {want}"


def _contract_keep(orc, B, H, Nq, Nk, t, seed, offset):
    """The keep mask evaluated from the generator by the counter layout."""
    key = (seed & 0xFFFFFFFF, seed >> 32)
    keep = np.zeros((B, H, Nq, Nk), dtype=np.uint8)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, Nq, 4):
                for j0 in range(0, Nk, 4):
                    words = orc.philox4x32_10((j0 // 4, i0 // 4, b * H + h, offset), key)
                    for i in range(i0, min(i0 + 4, Nq)):
                        for j in range(j0, min(j0 + 4, Nk)):
                            u = (words[i % 4] >> (8 * (j % 4))) & 0xFF
                            keep[b, h, i, j] = u >= t
    return keep


def pin_dropout_mask(orc):
    """The keep mask: it follows the counter layout from the generator; the
    drop rate is t / 256 at several thresholds (a uniform byte); neighbours
    along rows, columns and diagonals, other offsets and other heads are
    uncorrelated (|corr| within 5 / sqrt(n))."""
    B, H, N = 2, 3, 256
    seed = 0xDEADBEEF12345
    keep = orc.dropout_keep(B, H, 9, 13, 0.3, seed, 7)
    assert np.array_equal(keep, _contract_keep(orc, B, H, 9, 13, orc_threshold(0.3), seed, 7))
    n = B * H * N * N
    for p in (1 / 256, 0.1, 0.5, 255 / 256):
        t = orc_threshold(p)
        drop = 1.0 - orc.dropout_keep(B, H, N, N, p, seed, 3).astype(np.float64)
        rate = t / 256
        sd = math.sqrt(rate * (1 - rate) / n)
        assert abs(drop.mean() - rate) <= 5 * sd + 1e-12, f"drop rate {drop.mean()} vs {rate}"
    k = orc.dropout_keep(B, H, N, N, 0.5, seed, 3).astype(np.float64) - 0.5
    k2 = orc.dropout_keep(B, H, N, N, 0.5, seed, 4).astype(np.float64) - 0.5

    def corr(a, b):
        return float((a * b).mean() / math.sqrt((a * a).mean() * (b * b).mean()))

    pairs = {"row": (k[..., :, 1:], k[..., :, :-1]), "col": (k[..., 1:, :], k[..., :-1, :]),
             "diag": (k[..., 1:, 1:], k[..., :-1, :-1]), "offset": (k, k2),
             "head": (k[:, 1:], k[:, :-1]), "batch": (k[1:], k[:-1])}
    for what, (a, b) in pairs.items():
        assert abs(corr(a, b)) <= 5 / math.sqrt(a.size), f"keep bits correlated along {what}"


def orc_threshold(p):
    import oracle
    return oracle.dropout_threshold(p)


def pin_dropout_special_cases(orc):
    """p = 0 and any p below 1/512 (threshold 0) are exactly no dropout; a
    threshold of 1 changes the output; the mask ignores the attention mask."""
    B, H, Hkv, Nq, Nk, d = 1, 2, 1, 6, 9, 3
    q, k, v = rand((B, Nq, H, d), 90), rand((B, Nk, Hkv, d), 91), rand((B, Nk, Hkv, d), 92)
    do = rand((B, Nq, H, d), 93)
    o0, l0 = orc.attention_fwd(q, k, v, 0.5, True)
    g0 = orc.attention_bwd(q, k, v, do, 0.5, True)
    for p in (0.0, 1.0 / 1024):
        o, l = orc.attention_fwd(q, k, v, 0.5, True, dropout_p=p, dropout_seed=5)
        g = orc.attention_bwd(q, k, v, do, 0.5, True, dropout_p=p, dropout_seed=5)
        assert np.array_equal(o, o0) and np.array_equal(l, l0)
        assert all(np.array_equal(a, b) for a, b in zip(g, g0))
    o, l = orc.attention_fwd(q, k, v, 0.5, True, dropout_p=0.5, dropout_seed=5)
    assert np.array_equal(l, l0), "dropout must not change the LSE"
    assert not np.allclose(o, o0)


def pin_dropout_unbiased(orc):
    """Inverted dropout keeps the expectation: the mean of O over many
    offsets converges to O without dropout (within 5 standard errors per
    element), for p = 0.25 and p = 0.6, causal and full."""
    B, H, Hkv, Nq, Nk, d = 1, 2, 1, 5, 11, 3
    q, k, v = rand((B, Nq, H, d), 94), rand((B, Nk, Hkv, d), 95), rand((B, Nk, Hkv, d), 96)
    K = 1500
    for p, causal in ((0.25, True), (0.6, False)):
        o_ref, _ = orc.attention_fwd(q, k, v, 0.8, causal)
        samples = np.stack([orc.attention_fwd(q, k, v, 0.8, causal, dropout_p=p,
                                              dropout_seed=77, dropout_offset=off)[0]
                            for off in range(K)])
        mean, se = samples.mean(0), samples.std(0) / math.sqrt(K)
        assert np.all(np.abs(mean - o_ref) <= 5 * se + 1e-12), \
            f"dropout mean off by {np.max(np.abs(mean - o_ref) / (se + 1e-300)):.1f} s.e."


def pin_dropout_finite_differences(orc):
    """With the drop decisions fixed (seed and offset), O is a smooth
    function of Q, K and V: central differences of sum(O o dO) agree with
    the backward, and the sampled-row backward equals the full one."""
    h = 1e-6
    B, H, Hkv, Nq, Nk, d = 1, 2, 1, 6, 8, 3
    q, k, v = rand((B, Nq, H, d), 97), rand((B, Nk, Hkv, d), 98), rand((B, Nk, Hkv, d), 99)
    do = rand((B, Nq, H, d), 100)
    for m in (dict(causal=False), dict(causal=True)):
        kw = dict(m, dropout_p=0.35, dropout_seed=1234, dropout_offset=9)
        dq, dk, dv = orc.attention_bwd(q, k, v, do, 0.6, **kw)

        def loss(qq, kk, vv):
            return float((orc.attention_fwd(qq, kk, vv, 0.6, **kw)[0] * do.numpy()).sum())

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            fd = np.zeros(x.shape)
            flat = x.reshape(-1)
            for idx in range(flat.numel()):
                args = {"q": q, "k": k, "v": v}
                xp, xm = flat.clone(), flat.clone()
                xp[idx] += h
                xm[idx] -= h
                args[name] = xp.reshape(x.shape)
                lp = loss(args["q"], args["k"], args["v"])
                args[name] = xm.reshape(x.shape)
                lm = loss(args["q"], args["k"], args["v"])
                fd.reshape(-1)[idx] = (lp - lm) / (2 * h)
            err = np.abs(fd - g).max() / max(1.0, np.abs(fd).max())
            assert err <= 1e-6, f"dropout finite differences d{name} {m}: {err:.2e}"
        qrows, krows = [0, 5, 2], [7, 0, 3]
        dq_r, dk_r, dv_r = orc.attention_bwd_rows(q, k, v, do, qrows, krows, 0.6, **kw)
        _close(dq_r, dq[:, qrows], 1e-13, "dropout rows dQ")
        _close(dk_r, dk[:, krows], 1e-13, "dropout rows dK")
        _close(dv_r, dv[:, krows], 1e-13, "dropout rows dV")
        o_r, _ = orc.attention_fwd_rows(q, k, v, qrows, 0.6, **kw)
        assert np.array_equal(o_r, orc.attention_fwd(q, k, v, 0.6, **kw)[0][:, qrows])


def pin_dropout_varlen_numbering(orc):
    """Packed sequences number their drop decisions by sequence index: equal
    lengths packed give the dense batched result."""
    B, H, N, d = 3, 2, 7, 3
    q, k, v = rand((B, N, H, d), 101), rand((B, N, H, d), 102), rand((B, N, H, d), 103)
    do = rand((B, N, H, d), 104)
    kw = dict(dropout_p=0.4, dropout_seed=99, dropout_offset=1)
    cu = [0, N, 2 * N, 3 * N]
    o, lse = orc.attention_fwd(q, k, v, 0.5, True, **kw)
    ov, lv = orc.attention_fwd_varlen(q.reshape(B * N, H, d), k.reshape(B * N, H, d),
                                      v.reshape(B * N, H, d), cu, cu, 0.5, True, **kw)
    _close(ov, o.reshape(B * N, H, d), 1e-14, "varlen dropout O")
    g = orc.attention_bwd(q, k, v, do, 0.5, True, **kw)
    gv = orc.attention_bwd_varlen(q.reshape(B * N, H, d), k.reshape(B * N, H, d),
                                  v.reshape(B * N, H, d), do.reshape(B * N, H, d), cu, cu, 0.5,
                                  True, **kw)
    for a, b_, n in zip(gv, g, ("dQ", "dK", "dV")):
        _close(a, b_.reshape(B * N, H, d), 1e-14, "varlen dropout " + n)


# --- FP8 (E4M3) --------------------------------------------------------------

def pin_e4m3_codec(orc):
    """The oracle's E4M3 codec against torch's float8_e4m3fn (run, not read):
    the value of every one of the 256 codes; the code of every finite bf16
    number within +-448 and of every midpoint between neighbouring codes
    (ties to the even mantissa); every finite code round-trips; beyond 448
    the oracle saturates where torch gives NaN."""
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3_dequantize(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(mine[fin], ref[fin]), "E4M3 values"
    assert np.array_equal(np.signbit(mine[fin]), np.signbit(ref[fin]))

    def torch_codes(x32):
        return x32.to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    bf = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    x = bf.float()
    x = x[torch.isfinite(x) & (x.abs() <= 448)]
    assert np.array_equal(orc.e4m3_quantize(x), torch_codes(x)), "E4M3 codes of bf16 values"
    pos = mine[:0x7F]
    mids = torch.tensor((pos[:-1] + pos[1:]) / 2, dtype=torch.float32)
    for m in (mids, -mids):
        assert np.array_equal(orc.e4m3_quantize(m), torch_codes(m)), "E4M3 ties"
    assert np.array_equal(orc.e4m3_quantize(mine[fin]), codes[fin]), "E4M3 round trip"
    sat = orc.e4m3_quantize(np.array([449.0, 464.0, 1e6, -500.0, np.inf]))
    assert sat.tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E], sat
    scaled = orc.e4m3_quantize(np.array([3.0, -1.5]), scale=0.5)
    assert scaled.tolist() == torch_codes(torch.tensor([6.0, -3.0])).tolist()


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
    pin_philox_against_curand,
    pin_dropout_mask,
    pin_dropout_special_cases,
    pin_dropout_unbiased,
    pin_dropout_finite_differences,
    pin_dropout_varlen_numbering,
    pin_e4m3_codec,
]
