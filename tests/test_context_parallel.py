"""Context-parallel attention (context_parallel.py).

CPU: the chunk layouts and the ring schedule checked by brute force (every
visible pair of chunks computed exactly once, zigzag balanced), and the ring
itself run as gloo ranks (world sizes 1-3) with the library's kernels
replaced by fakes: the forward by the float64 oracle on each chunk pair, the
merge by the oracle's merge, the staged backward by the textbook gradient
formulas against the given O and LSE.  The whole-sequence result is then
compared with the oracle over the whole sequence.  GPU: one process (the
ring of one rank, two zigzag chunks) on the real kernels."""
import math
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from attn_inputs import Workload, make_inputs
from oracle_pins import mask_matrix
from parity import check_grad, check_lse, check_o


# ------------------------------------------------------------------ layouts and schedule
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (True, 7, -1),
                                          (False, 5, 9), (False, -1, 0), (True, 0, -1)])
def test_schedule_covers_every_visible_pair_once(layout, world, causal, wl, wr):
    """Every (query chunk, key chunk) pair with a visible element (brute
    force over the whole sequence's mask) is scheduled exactly once, with the
    chunk distance that becomes its position offset."""
    from io_aware_exact_33_b200 import context_parallel as cp
    n = 4
    nc = cp.num_chunks(world, layout)
    owned = sorted(g for r in range(world) for g in cp.chunk_ids(r, world, layout))
    assert owned == list(range(nc))
    seen = {}
    for r in range(world):
        mine = cp.chunk_ids(r, world, layout)
        for s, step in enumerate(cp.schedule(r, world, layout, causal, wl, wr, n)):
            theirs = cp.chunk_ids((r - s) % world, world, layout)
            for c, kc, dg in step:
                key = (mine[c], theirs[kc])
                assert key not in seen and dg == key[0] - key[1]
                seen[key] = dg
    vis = mask_matrix(nc * n, nc * n, causal=causal, window_left=wl, window_right=wr)
    want = {(a, b) for a in range(nc) for b in range(nc)
            if vis[a * n:(a + 1) * n, b * n:(b + 1) * n].any()}
    assert set(seen) == want


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_causal_steps_are_balanced(world):
    """Work per rank and step in units of one full n x n pair (a causal
    diagonal pair is half of one): two units everywhere."""
    from io_aware_exact_33_b200 import context_parallel as cp
    for r in range(world):
        for step in cp.schedule(r, world, "zigzag", True):
            assert sum(0.5 if dg == 0 else 1.0 for _, _, dg in step) == 2.0


def test_shard_unshard_roundtrip():
    from io_aware_exact_33_b200 import context_parallel as cp
    x = torch.arange(2 * 24 * 3).reshape(2, 24, 3)
    for layout in ("contiguous", "zigzag"):
        for world in (1, 2, 3):
            shards = [cp.shard(x, r, world, layout) for r in range(world)]
            assert all(s.is_contiguous() for s in shards)
            assert torch.equal(cp.unshard(shards, layout), x)
    z = cp.shard(x, 0, 3, "zigzag")  # chunks 0 and 5 of 6
    assert torch.equal(z[0], x[:, 0:4]) and torch.equal(z[1], x[:, 20:24])
    with pytest.raises(ValueError):
        cp.shard(torch.zeros(1, 10, 1), 0, 3, "zigzag")


# ------------------------------------------------------------------ fakes of the kernels
_STATE = {}


def _fake_scores(q, k, scale, causal, wl, wr, pos_offset):
    """float64 scaled scores (B, H, nq, nk) of one pair with the masks of the
    kernels' reading at off = nk - nq + pos_offset (-inf where hidden)."""
    g = q.shape[2] // k.shape[2]
    kd = k.double().repeat_interleave(g, dim=2)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    s = torch.einsum("bihd,bjhd->bhij", q.double(), kd) * scale
    n, m = s.shape[-2:]
    dist = torch.arange(n)[:, None] + (m - n + pos_offset) - torch.arange(m)[None, :]  # i + off - j
    vis = torch.ones(n, m, dtype=torch.bool)
    if causal:
        vis &= dist >= 0
    if wl >= 0:
        vis &= dist <= wl
    if wr >= 0:
        vis &= dist >= -wr
    return s.masked_fill(~vis, -math.inf)


def _fake_fwd(q, k, v, softmax_scale=None, causal=False, window_left=-1, window_right=-1,
              out=None, lse=None, stream=None, alibi_slopes=None, pos_offset=0):
    """One pair's partial output and LSE over its keys (float64, explicit
    masks), as attn_fwd computes them; a row that sees no key gets O = 0 and
    LSE = -inf."""
    for t in (q, k, v, out, lse):
        assert t.is_contiguous()
    assert q.shape[1] == k.shape[1] and alibi_slopes is None
    s = _fake_scores(q, k, softmax_scale, causal, window_left, window_right, pos_offset)
    mx = s.amax(-1, keepdim=True)
    e = torch.exp(s - mx.clamp_min(-1e300))
    l = e.sum(-1, keepdim=True)
    g = q.shape[2] // k.shape[2]
    vd = v.double().repeat_interleave(g, dim=2)
    o = torch.einsum("bhij,bjhd->bihd", e / l.clamp_min(1e-300), vd)
    out.copy_(o)
    lse.copy_((mx + torch.log(l))[..., 0])
    return out, lse


def _fake_merge(o_parts, lse_parts, out=None, lse=None, stream=None):
    for t in (o_parts, lse_parts, out, lse):
        assert t.is_contiguous()
    o, l = oracle.attention_merge(o_parts, lse_parts)
    out.copy_(torch.from_numpy(o))
    lse.copy_(torch.from_numpy(l))
    return out, lse


def _fake_ws_size(p):
    return 64


def _fake_prepare(p, out, lse, dout, workspace, stream=None):
    _STATE[workspace.data_ptr()] = dict(o=out.double(), lse=lse.double(), do=dout.double(),
                                        dq=torch.zeros(out.shape, dtype=torch.float64))


def _fake_accumulate_f32(p, q, k, v, dout, dk_acc, dv_acc, workspace, stream=None):
    """Gradient shares of one key block, probabilities taken against the
    given (global) LSE and D = rowsum(dO o O) from the given (global) O; the
    key gradients are added into the float32 sums."""
    st = _STATE[workspace.data_ptr()]
    assert p.seqlen_q == q.shape[1] and p.seqlen_k == k.shape[1]
    g = p.nheads // p.nheads_kv
    qd = q.double()
    kd = k.double().repeat_interleave(g, dim=2)
    vd = v.double().repeat_interleave(g, dim=2)
    s = _fake_scores(q, k, p.softmax_scale, p.causal, p.window_left, p.window_right,
                     p.pos_offset)
    prob = torch.exp(s - st["lse"][..., None])
    dvec = (st["do"] * st["o"]).sum(-1).transpose(1, 2)  # (B, H, n)
    dp = torch.einsum("bihd,bjhd->bhij", st["do"], vd)
    ds = prob * (dp - dvec[..., None])
    st["dq"] += torch.einsum("bhij,bjhd->bihd", ds, kd) * p.softmax_scale
    dkh = torch.einsum("bhij,bihd->bjhd", ds, qd) * p.softmax_scale
    dvh = torch.einsum("bhij,bihd->bjhd", prob, st["do"])
    B, m, hkv, d = k.shape
    assert dk_acc.dtype == torch.float32 and dv_acc.dtype == torch.float32
    dk_acc += dkh.reshape(B, m, hkv, g, d).sum(3).float()
    dv_acc += dvh.reshape(B, m, hkv, g, d).sum(3).float()


def _fake_f32_to_16(src, dst, stream=None):
    assert src.dtype == torch.float32 and src.shape == dst.shape
    dst.copy_(src)


def _fake_finalize(p, dq, workspace, stream=None):
    dq.copy_(_STATE.pop(workspace.data_ptr())["dq"])


def _install_fakes():
    import io_aware_exact_33_b200 as attn
    attn.attn_fwd = _fake_fwd
    attn.attn_merge = _fake_merge
    attn.attn_bwd_workspace_size = _fake_ws_size
    attn.attn_bwd_prepare = _fake_prepare
    attn.attn_bwd_accumulate_f32 = _fake_accumulate_f32
    attn.attn_f32_to_16 = _fake_f32_to_16
    attn.attn_bwd_finalize = _fake_finalize


@pytest.fixture
def fakes(monkeypatch):
    import io_aware_exact_33_b200 as attn
    for name, f in (("attn_fwd", _fake_fwd), ("attn_merge", _fake_merge),
                    ("attn_bwd_workspace_size", _fake_ws_size),
                    ("attn_bwd_prepare", _fake_prepare),
                    ("attn_bwd_accumulate_f32", _fake_accumulate_f32),
                    ("attn_f32_to_16", _fake_f32_to_16),
                    ("attn_bwd_finalize", _fake_finalize)):
        monkeypatch.setattr(attn, name, f)


# ------------------------------------------------------------------ the ring on gloo ranks
def _ring_rank(rank, world, store_path, w, layout, queue):
    import torch.distributed as dist
    from io_aware_exact_33_b200 import context_parallel as cp
    # rendezvous through a file: no port to race for
    dist.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank,
                            world_size=world)
    try:
        _install_fakes()
        q, k, v, do = (cp.shard(t, rank, world, layout) for t in make_inputs(w))
        win = dict(window_left=w.window_left, window_right=w.window_right)
        o, lse = cp.ring_attn_fwd(q, k, v, w.softmax_scale, w.causal, layout, **win)
        dq, dk, dv = cp.ring_attn_bwd(q, k, v, o, lse, do, w.softmax_scale, w.causal, layout,
                                      **win)
        # the autograd wrapper runs the same two passes
        ql, kl, vl = (t.clone().requires_grad_(True) for t in (q, k, v))
        out = cp.ring_flash_attn_func(ql, kl, vl, w.softmax_scale, w.causal, layout,
                                      window_size=(w.window_left, w.window_right))
        out.backward(do)
        # the backward fakes use torch's CPU matrix products, whose last bits
        # may depend on memory alignment: allow one bf16 rounding step
        near = lambda a, b: torch.allclose(a.float(), b.float(), rtol=2 ** -7, atol=2 ** -12)
        same = (torch.equal(out.detach(), o) and near(ql.grad, dq) and near(kl.grad, dk) and
                near(vl.grad, dv))
        # plain arrays, pickled by value: a tensor would travel through shared
        # memory that needs this process alive until the parent has it
        queue.put((rank, *(t.float().numpy() for t in (o, lse, dq, dk, dv)), same))
    finally:
        dist.destroy_process_group()


def _run_ring(world, w, layout, tmp_path):
    oracle.build()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    store = str(tmp_path / "rendezvous")
    procs = [ctx.Process(target=_ring_rank, args=(r, world, store, w, layout, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((queue.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0, f"rank exit code {p.exitcode}"
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    return [(r, bf(o), torch.from_numpy(lse), bf(dq), bf(dk), bf(dv), same)
            for r, o, lse, dq, dk, dv, same in res]


def _compare_whole(res, w, layout, what, slopes=None):
    from io_aware_exact_33_b200 import context_parallel as cp
    q, k, v, do = make_inputs(w)
    args = (w.softmax_scale, w.causal, w.window_left, w.window_right)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, *args, alibi_slopes=slopes)
    g_ref = oracle.attention_bwd(q, k, v, do, *args, alibi_slopes=slopes)
    o = cp.unshard([r[1] for r in res], layout)
    lse = cp.unshard([r[2] for r in res], layout, dim=2)
    check_o(o, o_ref, what + " O")
    check_lse(lse, lse_ref, what + " LSE")
    for i, name in enumerate(("dQ", "dK", "dV")):
        check_grad(cp.unshard([r[3 + i] for r in res], layout), g_ref[i], f"{what} {name}")
    assert all(r[6] for r in res), f"{what}: autograd wrapper differs from the direct calls"


@pytest.mark.parametrize("world,layout,causal,wl,wr", [
    (2, "zigzag", True, -1, -1), (3, "zigzag", True, -1, -1), (2, "contiguous", True, -1, -1),
    (3, "contiguous", False, -1, -1), (2, "zigzag", False, -1, -1),
    (3, "zigzag", True, 7, -1), (2, "contiguous", False, 5, 9),
])
def test_ring_on_gloo_ranks(world, layout, causal, wl, wr, tmp_path):
    from io_aware_exact_33_b200 import context_parallel as cp
    n = 6  # rows per chunk
    N = n * cp.num_chunks(world, layout)
    w = Workload("cp", 2, 4, 2, N, N, 8, causal, wl, wr, "bf16", 1.0, 800 + world,
                 softmax_scale=0.4)
    res = _run_ring(world, w, layout, tmp_path)
    _compare_whole(res, w, layout, f"ring W={world} {layout} causal={causal} window={wl},{wr}")


def test_ring_of_one_process(fakes):
    """Without a process group the ring is this process alone; zigzag then
    holds chunks 0 and 1, and key chunk 0 collects dK / dV from both query
    chunks."""
    from io_aware_exact_33_b200 import context_parallel as cp
    w = Workload("cp1", 1, 2, 1, 10, 10, 8, True, -1, -1, "bf16", 1.0, 810)
    q, k, v, do = (cp.shard(t, 0, 1) for t in make_inputs(w))
    o, lse = cp.ring_attn_fwd(q, k, v, None, True)
    dq, dk, dv = cp.ring_attn_bwd(q, k, v, o, lse, do, None, True)
    _compare_whole([(0, o, lse, dq, dk, dv, True)], w, "zigzag", "ring W=1")


def test_ring_rejects_bad_layouts(fakes):
    from io_aware_exact_33_b200 import context_parallel as cp
    q = torch.zeros(1, 1, 4, 2, 8, dtype=torch.bfloat16)  # one chunk, zigzag wants two
    with pytest.raises(ValueError):
        cp.ring_attn_fwd(q, q, q, causal=True)
    with pytest.raises(ValueError):
        cp.chunk_ids(0, 2, "striped")


# ------------------------------------------------------------------ GPU
@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
def test_ring_of_one_process_on_gpu(d):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_33_b200 import context_parallel as cp
    w = Workload("cpg", 2, 4, 2, 400, 400, d, True, -1, -1, "bf16", 1.0, 811)
    q, k, v, do = (cp.shard(t, 0, 1).cuda() for t in make_inputs(w))
    o, lse = cp.ring_attn_fwd(q, k, v, None, True)
    dq, dk, dv = cp.ring_attn_bwd(q, k, v, o, lse, do, None, True)
    torch.cuda.synchronize()
    res = [(0, o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu(), True)]
    _compare_whole(res, w, "zigzag", "ring W=1 on GPU")


@pytest.mark.gpu
@pytest.mark.parametrize("wl,wr,with_slopes", [(150, -1, False), (-1, -1, True), (90, -1, True)])
def test_ring_window_and_slopes_on_gpu(wl, wr, with_slopes):
    """Sliding windows and positional slopes across chunks: every pair call
    carries pos_offset = (query chunk - key chunk) x n, and the merged result
    equals the oracle over the whole sequence (zigzag, two chunks of 200:
    with a window of 150 or 90 the far pair is partly or wholly hidden)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from io_aware_exact_33_b200 import context_parallel as cp
    w = Workload("cpw", 2, 4, 2, 400, 400, 128, True, wl, wr, "bf16", 1.0, 813)
    slopes = (torch.tensor([2.0 ** (-2 * (h + 1)) for h in range(4)], dtype=torch.float32)
              if with_slopes else None)
    sl = slopes.cuda() if with_slopes else None
    q, k, v, do = (cp.shard(t, 0, 1).cuda() for t in make_inputs(w))
    o, lse = cp.ring_attn_fwd(q, k, v, None, True, window_left=wl, window_right=wr,
                              alibi_slopes=sl)
    dq, dk, dv = cp.ring_attn_bwd(q, k, v, o, lse, do, None, True, window_left=wl,
                                  window_right=wr, alibi_slopes=sl)
    torch.cuda.synchronize()
    res = [(0, o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu(), True)]
    _compare_whole(res, w, "zigzag", f"ring W=1 window={wl} slopes={with_slopes}", slopes)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 256])
def test_accumulate_f32_adds_key_gradients(d):
    """attn_bwd_accumulate_f32 adds dK (x scale) and dV in float32 into the
    caller's sums: two calls on zeroed sums give twice the oracle's key
    gradients, and twice the dQ share in the workspace accumulator; the
    float32-to-16-bit conversion rounds like torch.  Head dim 256 runs the
    three-kernel backward."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as attn
    w = Workload("accf32", 2, 4, 2, 300, 260, d, True, 64, -1, "bf16", 1.0, 812)
    q, k, v, do = make_inputs(w)
    qc, kc, vc, doc = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    args = (w.softmax_scale, w.causal, w.window_left, w.window_right)
    o, lse = attn.attn_fwd(qc, kc, vc, *args)
    p = attn.params_for(qc, kc, *args)
    ws = torch.empty(attn.attn_bwd_workspace_size(p), dtype=torch.uint8, device="cuda")
    attn.attn_bwd_prepare(p, o, lse, doc, ws)
    dk_acc = torch.zeros(k.shape, dtype=torch.float32, device="cuda")
    dv_acc = torch.zeros(k.shape, dtype=torch.float32, device="cuda")
    for _ in range(2):
        attn.attn_bwd_accumulate_f32(p, qc, kc, vc, doc, dk_acc, dv_acc, ws)
    dq = torch.empty_like(qc)
    attn.attn_bwd_finalize(p, dq, ws)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    dq_r, dk_r, dv_r = oracle.attention_bwd(q, k, v, do, *args)
    check_grad(dk_acc.cpu() / 2, dk_r, "dK sum / 2")
    check_grad(dv_acc.cpu() / 2, dv_r, "dV sum / 2")
    check_grad(dq.cpu().double() / 2, dq_r, "dQ (two shares) / 2")
    half = torch.empty(k.shape, dtype=torch.bfloat16, device="cuda")
    attn.attn_f32_to_16(dk_acc, half)
    torch.cuda.synchronize()
    assert torch.equal(half.cpu(), dk_acc.cpu().to(torch.bfloat16))
