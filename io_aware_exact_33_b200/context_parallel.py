"""Context (sequence) parallel attention: one long sequence split over ranks.

Each rank holds some chunks of the sequence's queries, keys and values.  The
key/value blocks travel once around a ring of ranks (point-to-point sends
and receives of ``torch.distributed``, NCCL over NVLink on GPUs); every rank
runs the library's attention kernels on its own queries against each block
as it passes, and the results are combined exactly:

- forward: every (query chunk, key chunk) pair gives a partial output and
  LSE over that key chunk, written by ``attn_fwd`` into one slot of a parts
  buffer; ``attn_merge`` then combines the parts of each query chunk
  (LSE = log sum exp LSE_s, O = sum exp(LSE_s - LSE) O_s, the rescale that
  the online softmax applies tile by tile);
- backward: the staged backward of the library.  ``attn_bwd_prepare`` runs
  once per query chunk on the merged O and LSE, every pair's
  ``attn_bwd_accumulate_f32`` adds its dQ share into that chunk's float32
  accumulator (exact across pairs: softmax probabilities are taken against
  the global LSE) and its dK / dV into a float32 buffer that travels round
  the ring behind its key/value block and arrives at its owner after the
  last step, and ``attn_bwd_finalize`` writes dQ.

The pages name faster communication across devices as the way to longer
contexts (FA2-Guide, "对未来Transformer架构的深远影响") without fixing a scheme;
this is the plainest exact one.  Every pair is one kernel call over local
indices with ``pos_offset`` = (query chunk - key chunk) x chunk length, so
the kernels apply the whole sequence's causal mask, sliding window and
positional slopes to the pair; pairs that no mask lets through are skipped.
With a causal mask, equal-size chunks make every pair either fully visible
(key chunk before the query chunk), causal with Nq = Nk (the same chunk) or
skipped (key chunk after).  The "zigzag" layout gives rank r of W the chunks
r and 2W - 1 - r of 2W, so every rank does the same causal work at every
step; "contiguous" gives rank r chunk r of W (balanced without a mask only).

Layouts: a rank's tensors are chunk-major, q (C, B, n, H, d), k and v
(C, B, n, Hkv, d), lse (C, B, H, n), C = chunks per rank in ``chunk_ids``
order, so each chunk is one contiguous (B, n, ...) tensor.  ``shard`` and
``unshard`` convert from and to whole-sequence tensors.

Not supported here: packed variable-length batches and dropout.  Every
rank must call these functions with the same shapes and arguments, in the
same order (they are collective).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

import io_aware_exact_33_b200 as _lib

LAYOUTS = ("contiguous", "zigzag")
FULL, CAUSAL, SKIP = 0, 1, 2


def chunk_ids(rank: int, world: int, layout: str = "zigzag") -> Tuple[int, ...]:
    """Global indices of the sequence chunks that rank ``rank`` holds, in
    the order of its chunk-major tensors."""
    if layout == "contiguous":
        return (rank,)
    if layout == "zigzag":
        return (rank, 2 * world - 1 - rank)
    raise ValueError(f"layout must be one of {LAYOUTS}, got {layout!r}")


def num_chunks(world: int, layout: str = "zigzag") -> int:
    """Chunks the whole sequence is cut into."""
    return len(chunk_ids(0, world, layout)) * world


def pair_mask(q_chunk: int, k_chunk: int, causal: bool) -> int:
    """How query chunk ``q_chunk`` sees key chunk ``k_chunk`` (equal-size
    chunks of one sequence) under a causal mask or none: FULL, CAUSAL (same
    chunk, causal) or SKIP."""
    if not causal or k_chunk < q_chunk:
        return FULL
    return CAUSAL if k_chunk == q_chunk else SKIP


def pair_visible(q_chunk: int, k_chunk: int, n: int, causal: bool, window_left: int = -1,
                 window_right: int = -1) -> bool:
    """Whether any key of chunk ``k_chunk`` is visible from any query of chunk
    ``q_chunk`` (chunks of ``n`` positions): the distance j - i of global
    positions spans (k_chunk - q_chunk) n +- (n - 1), and the masks allow
    -window_left <= j - i <= min(0 if causal, window_right)."""
    dmin = (k_chunk - q_chunk) * n - (n - 1)
    dmax = (k_chunk - q_chunk) * n + (n - 1)
    hi = None if window_right < 0 else window_right
    if causal:
        hi = 0 if hi is None else min(hi, 0)
    lo = None if window_left < 0 else -window_left
    return (hi is None or dmin <= hi) and (lo is None or dmax >= lo)


def schedule(rank: int, world: int, layout: str, causal: bool, window_left: int = -1,
             window_right: int = -1, n: int = 1) -> List[List[Tuple[int, int, int]]]:
    """Per ring step s (this rank then holds the key/value block of rank
    (rank - s) mod world) the (local query chunk, block key chunk, global
    query chunk - global key chunk) triples to compute: the pairs with any
    visible element for chunks of ``n`` positions."""
    mine = chunk_ids(rank, world, layout)
    steps = []
    for s in range(world):
        theirs = chunk_ids((rank - s) % world, world, layout)
        steps.append([(c, kc, gq - gk)
                      for c, gq in enumerate(mine) for kc, gk in enumerate(theirs)
                      if pair_visible(gq, gk, n, causal, window_left, window_right)])
    return steps


def shard(x: torch.Tensor, rank: int, world: int, layout: str = "zigzag",
          dim: int = 1) -> torch.Tensor:
    """This rank's chunks of a whole-sequence tensor (sequence along
    ``dim``), stacked chunk-major and contiguous."""
    nc = num_chunks(world, layout)
    if x.shape[dim] % nc:
        raise ValueError(f"sequence length {x.shape[dim]} is not a multiple of {nc} chunks")
    parts = x.chunk(nc, dim=dim)
    return torch.stack([parts[g] for g in chunk_ids(rank, world, layout)]).contiguous()


def unshard(shards: Sequence[torch.Tensor], layout: str = "zigzag", dim: int = 1) -> torch.Tensor:
    """Inverse of ``shard``: the whole-sequence tensor from every rank's
    chunk-major tensor (list indexed by rank)."""
    world = len(shards)
    by_chunk = {}
    for r, t in enumerate(shards):
        for c, g in enumerate(chunk_ids(r, world, layout)):
            by_chunk[g] = t[c]
    return torch.cat([by_chunk[g] for g in range(num_chunks(world, layout))], dim=dim)


class _Ring:
    """This rank's place in the ring: rank, world size and the global ranks
    of its neighbours.  Without an initialised process group (and no group
    given) the ring is this process alone."""

    def __init__(self, group):
        if group is None and not dist.is_initialized():
            self.rank, self.world, self.next, self.prev = 0, 1, 0, 0
            return
        g = group if group is not None else dist.group.WORLD
        self.rank, self.world = dist.get_rank(g), dist.get_world_size(g)
        self.next = dist.get_global_rank(g, (self.rank + 1) % self.world)
        self.prev = dist.get_global_rank(g, (self.rank - 1) % self.world)
        self.group = g

    def exchange(self, send: torch.Tensor, recv: torch.Tensor):
        """Start sending ``send`` to the next rank and receiving the previous
        rank's into ``recv``; returns the works to wait on."""
        ops = [dist.P2POp(dist.isend, send, self.next, self.group),
               dist.P2POp(dist.irecv, recv, self.prev, self.group)]
        return dist.batch_isend_irecv(ops)


def _wait(works) -> None:
    for w in works:
        w.wait()


def _check_layout(q, k, v, ring, layout):
    C = len(chunk_ids(ring.rank, ring.world, layout))
    if q.dim() != 5 or k.dim() != 5 or q.shape[0] != C or k.shape[0] != C:
        raise ValueError(f"expected chunk-major q (C, B, n, H, d) and k, v (C, B, n, Hkv, d) with "
                         f"C = {C} for layout {layout!r}")
    if k.shape[2] != q.shape[2] or v.shape != k.shape:
        raise ValueError("q, k and v chunks must have the same length n; v the shape of k")
    return C


def ring_attn_fwd(q, k, v, softmax_scale: Optional[float] = None, causal: bool = False,
                  layout: str = "zigzag", group=None, window_left: int = -1,
                  window_right: int = -1, alibi_slopes=None):
    """Attention of this rank's query chunks over the whole sequence.

    q (C, B, n, H, d), k and v (C, B, n, Hkv, d): this rank's chunks, 16-bit
    contiguous CUDA tensors.  Returns (o (C, B, n, H, d), lse (C, B, H, n)
    float32), equal to the matching chunks of single-device attention over
    the whole sequence, with its causal mask, sliding window (positions
    relative to the whole sequence) and per-head positional slopes."""
    ring = _Ring(group)
    C = _check_layout(q, k, v, ring, layout)
    _, B, n, H, _ = q.shape
    steps = schedule(ring.rank, ring.world, layout, causal, window_left, window_right, n)
    nparts = [sum(1 for st in steps for (c2, _, _) in st if c2 == c) for c in range(C)]
    o_parts = [torch.empty((m,) + tuple(q.shape[1:]), dtype=q.dtype, device=q.device) for m in nparts]
    lse_parts = [torch.empty((m, B, H, n), dtype=torch.float32, device=q.device) for m in nparts]
    slot = [0] * C
    kv = torch.stack((k, v))  # (2, C, B, n, Hkv, d): one message per step
    for s in range(ring.world):
        nxt, works = None, []
        if s + 1 < ring.world:
            nxt = torch.empty_like(kv)
            works = ring.exchange(kv, nxt)
        for c, kc, dg in steps[s]:
            _lib.attn_fwd(q[c], kv[0, kc], kv[1, kc], softmax_scale, causal, window_left,
                          window_right, out=o_parts[c][slot[c]], lse=lse_parts[c][slot[c]],
                          alibi_slopes=alibi_slopes, pos_offset=dg * n)
            slot[c] += 1
        _wait(works)
        if nxt is not None:
            kv = nxt
    o = torch.empty_like(q)
    lse = torch.empty((C, B, H, n), dtype=torch.float32, device=q.device)
    for c in range(C):
        _lib.attn_merge(o_parts[c], lse_parts[c], out=o[c], lse=lse[c])
    return o, lse


def ring_attn_bwd(q, k, v, o, lse, do, softmax_scale: Optional[float] = None,
                  causal: bool = False, layout: str = "zigzag", group=None,
                  window_left: int = -1, window_right: int = -1, alibi_slopes=None):
    """Gradients (dq, dk, dv) of sum(o * do) for ``ring_attn_fwd`` with the
    same arguments; ``o`` and ``lse`` are its results, ``do`` (C, B, n, H, d).
    Each rank gets the gradients of its own chunks."""
    ring = _Ring(group)
    C = _check_layout(q, k, v, ring, layout)
    n = q.shape[2]
    steps = schedule(ring.rank, ring.world, layout, causal, window_left, window_right, n)
    # per query chunk: Dvec, LSE in base 2 and the float32 dQ accumulator
    ws, pq = [], []
    for c in range(C):
        p = _lib.params_for(q[c], k[0], softmax_scale, False)
        w = torch.empty(max(_lib.attn_bwd_workspace_size(p), 1), dtype=torch.uint8, device=q.device)
        _lib.attn_bwd_prepare(p, o[c], lse[c], do[c], w)
        ws.append(w)
        pq.append(p)
    kv = torch.stack((k, v))
    # float32 dK / dV sums of the block held now; they travel round the ring
    # one step behind their block.  The kernels add into them directly.
    dkv = torch.zeros(kv.shape, dtype=torch.float32, device=kv.device)
    dkv_in, dkv_works = None, []
    for s in range(ring.world):
        nxt, works = None, []
        if s + 1 < ring.world:
            nxt = torch.empty_like(kv)
            works = ring.exchange(kv, nxt)
        if s > 0:
            # the sums of the ranks the block visited before: added onto here
            _wait(dkv_works)
            dkv = dkv_in
        for c, kc, dg in steps[s]:
            p = _lib.params_for(q[c], kv[0, kc], softmax_scale, causal, window_left, window_right,
                                alibi_slopes, pos_offset=dg * n)
            _lib.attn_bwd_accumulate_f32(p, q[c], kv[0, kc], kv[1, kc], do[c], dkv[0, kc],
                                         dkv[1, kc], ws[c])
        if ring.world > 1:
            dkv_in = torch.empty_like(dkv)
            dkv_works = ring.exchange(dkv, dkv_in)
        else:
            dkv_in = dkv
        _wait(works)
        if nxt is not None:
            kv = nxt
    dq = torch.empty_like(q)
    for c in range(C):
        _lib.attn_bwd_finalize(pq[c], dq[c], ws[c])
    _wait(dkv_works)  # the last hop brings this rank's own block home
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    _lib.attn_f32_to_16(dkv_in[0], dk)
    _lib.attn_f32_to_16(dkv_in[1], dv)
    return dq, dk, dv


class _RingAttn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, softmax_scale, causal, layout, group, window_left, window_right,
                alibi_slopes):
        o, lse = ring_attn_fwd(q, k, v, softmax_scale, causal, layout, group, window_left,
                               window_right, alibi_slopes)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.args = (softmax_scale, causal, layout, group, window_left, window_right,
                    alibi_slopes)
        ctx.mark_non_differentiable(lse)
        return o, lse

    @staticmethod
    def backward(ctx, do, _dlse):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = ring_attn_bwd(q, k, v, o, lse, do.contiguous(), *ctx.args)
        return dq, dk, dv, None, None, None, None, None, None, None


def ring_flash_attn_func(q, k, v, softmax_scale: Optional[float] = None, causal: bool = False,
                         layout: str = "zigzag", group=None, return_lse: bool = False,
                         window_size=(-1, -1), alibi_slopes=None):
    """Differentiable ``ring_attn_fwd``: chunk-major local q, k, v in, the
    local output chunks (and, with ``return_lse``, their LSE) out;
    ``window_size`` = (left, right) in positions of the whole sequence."""
    wl, wr = (int(x) for x in window_size)
    o, lse = _RingAttn.apply(q, k, v, softmax_scale, bool(causal), layout, group, wl, wr,
                             alibi_slopes)
    return (o, lse) if return_lse else o
