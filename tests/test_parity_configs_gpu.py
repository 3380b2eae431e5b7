"""Parity on the five stated workloads at their full sizes, in the launch
configuration the benchmark times, with the raw errors recorded.

Exact attention (the tiled method reaches the untiled definition's result:
"FlashAttention transformer optimization", technical deep dive; "What is
FlashAttention", definition) is checked against the float64 oracle:

  * every row of the forward on the causal N=8192 workload and every row of
    the forward and backward on the GQA sliding-window workload;
  * on the other full-size passes, sampled rows: every row at a query- or
    key-tile boundary of the kernels (128-row forward tiles, 64-row backward
    query tiles, 128-row key tiles), the first and last 64 rows, and random
    rows up to >= 1024 query rows and >= 256 key rows per (batch, head).

Per pass the record holds the raw max|O - O_ref|, the rounding floor
max|round(O_ref) - O_ref| of the output dtype, how many elements exceed the
flat 1e-2 (each must lie within 1e-2 plus half an ulp of O_ref: see
tests/parity.py), max|LSE - LSE_ref| and the relative Frobenius error of
dQ, dK, dV over the checked rows.  The sampled backward passes are also
checked on every row through identities of the exact gradients (sum_j dK_j
= 0 and sum_j dV_j = sum_i dO_i per kv head).  With ATTN_PARITY_REPORT_DIR
set, each test writes its record there as JSON.
"""
import json
import os
import time

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import WORKLOADS, make_inputs, sample_rows
from parity import GRAD_REL_TOL, LSE_TOL, O_TOL, half_ulp, rel_fro
from test_bwd_gpu import _identities

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def _record(name, rec):
    rec = dict(rec, workload=name, oracle_threads=oracle.num_threads())
    print(json.dumps(rec))
    out = os.environ.get("ATTN_PARITY_REPORT_DIR")
    if out:
        os.makedirs(out, exist_ok=True)
        with open(os.path.join(out, f"{name}_{rec['pass']}.json"), "w") as f:
            json.dump(rec, f, indent=1)


def o_stats(o_gpu: torch.Tensor, o_ref: np.ndarray) -> dict:
    """Raw errors of an output against the oracle and whether every element
    is within the bound (1e-2 plus half an ulp at |O_ref|)."""
    og = o_gpu.to(torch.float64).numpy()
    err = np.abs(og - o_ref)
    floor = np.abs(torch.from_numpy(o_ref).to(o_gpu.dtype).double().numpy() - o_ref)
    over = err > O_TOL
    bound = O_TOL + half_ulp(o_ref, o_gpu.dtype)
    return {
        "o_max_abs_err": float(err.max()),
        "o_rounding_floor": float(floor.max()),
        "o_elements": int(err.size),
        "o_over_1e-2": int(over.sum()),
        "o_max_excess_over_floor_bound": float((err - bound).max()),
        "o_finite": bool(np.isfinite(og).all()),
        "o_within_bound": bool((err <= bound).all()),
    }


def lse_stats(lse_gpu: torch.Tensor, lse_ref: np.ndarray) -> dict:
    lg = lse_gpu.to(torch.float64).numpy()
    fin = np.isfinite(lse_ref)
    same_inf = bool(np.array_equal(np.isfinite(lg), fin) and np.all(lg[~fin] == lse_ref[~fin]))
    return {"lse_max_abs_err": float(np.abs(lg[fin] - lse_ref[fin]).max()) if fin.any() else 0.0,
            "lse_inf_pattern_equal": same_inf}


def assert_fwd(rec):
    assert rec["o_finite"] and rec["o_within_bound"], rec
    assert rec["lse_inf_pattern_equal"] and rec["lse_max_abs_err"] <= LSE_TOL, rec


def _rows(n, must, count, seed):
    """``must`` plus seeded random rows until there are ``count`` distinct."""
    rows = sample_rows(n, 0, seed, must=must)
    extra = 0
    while len(rows) < min(count, n):
        extra += count - len(rows)
        rows = sample_rows(n, extra, seed, must=must)
    return rows


def fwd_rows(n):
    """Rows of a sampled forward check: 128-row tile edges, both ends, and
    random rows up to >= 2048."""
    must = [r for t in range(0, n, 128) for r in (t, t + 127)] + list(range(64)) + \
        list(range(n - 64, n))
    return _rows(n, must, 2048, 4242)


def bwd_rows(n, tile, count, seed):
    must = [r for t in range(0, n, tile) for r in (t, t + tile - 1)] + list(range(64)) + \
        list(range(n - 64, n))
    return _rows(n, must, count, seed)


def run(attn, w, with_bwd):
    q, k, v, do = make_inputs(w, with_dout=with_bwd)
    args = (w.scale, w.causal, w.window_left, w.window_right)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = attn.attn_fwd(qc, kc, vc, *args)
    grads = None
    if with_bwd:
        grads = attn.attn_bwd(qc, kc, vc, o, lse, do.cuda(), *args)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    cpu = lambda t: t.cpu()  # noqa: E731
    return (q, k, v, do), cpu(o), cpu(lse), (tuple(map(cpu, grads)) if grads else None), args


def check_fwd(name, q, k, v, o, lse, args, rows=None):
    t0 = time.time()
    if rows is None:
        o_ref, lse_ref = oracle.attention_fwd(q, k, v, *args)
        o_chk, l_chk, nrows = o, lse, q.shape[1]
    else:
        o_ref, lse_ref = oracle.attention_fwd_rows(q, k, v, rows, *args)
        o_chk, l_chk, nrows = o[:, rows], lse[:, :, rows], len(rows)
    rec = {"pass": "fwd", "rows_checked_per_head": int(nrows), "rows_per_head": int(q.shape[1])}
    rec.update(o_stats(o_chk, o_ref))
    rec.update(lse_stats(l_chk, lse_ref))
    rec["oracle_s"] = round(time.time() - t0, 1)
    _record(name, rec)
    assert_fwd(rec)


def check_bwd(name, q, k, v, do, grads, args, qrows=None, krows=None):
    t0 = time.time()
    dq, dk, dv = grads
    if qrows is None:
        refs = oracle.attention_bwd(q, k, v, do, *args)
        got = (dq, dk, dv)
        nq, nk = q.shape[1], k.shape[1]
    else:
        refs = oracle.attention_bwd_rows(q, k, v, do, qrows, krows, *args)
        got = (dq[:, qrows], dk[:, krows], dv[:, krows])
        nq, nk = len(qrows), len(krows)
    rec = {"pass": "bwd", "query_rows_checked_per_head": int(nq),
           "key_rows_checked_per_head": int(nk), "rows_per_head": int(q.shape[1])}
    for n, g, r in zip(("dq", "dk", "dv"), got, refs):
        rec[f"{n}_rel_fro"] = rel_fro(g, r)
    rec["oracle_s"] = round(time.time() - t0, 1)
    _record(name, rec)
    for n in ("dq", "dk", "dv"):
        assert rec[f"{n}_rel_fro"] <= GRAD_REL_TOL, rec


def test_tiny_every_row(attn):
    name = "tiny_b1_h2_n128_d64"
    w = WORKLOADS[name]
    (q, k, v, do), o, lse, grads, args = run(attn, w, True)
    check_fwd(name, q, k, v, o, lse, args)
    check_bwd(name, q, k, v, do, grads, args)


def test_causal_n8192_fwd_every_row_bwd_sampled(attn):
    name = "causal_b2_h32_n8192_d128"
    w = WORKLOADS[name]
    (q, k, v, do), o, lse, grads, args = run(attn, w, True)
    _identities(w, do, grads[1], grads[2])
    check_fwd(name, q, k, v, o, lse, args)
    check_bwd(name, q, k, v, do, grads, args, bwd_rows(w.seqlen_q, 64, 1024, 11),
              bwd_rows(w.seqlen_k, 128, 256, 12))


def test_full_n16384_sampled(attn):
    name = "full_b1_h16_n16384_d128"
    w = WORKLOADS[name]
    (q, k, v, do), o, lse, grads, args = run(attn, w, True)
    _identities(w, do, grads[1], grads[2])
    check_fwd(name, q, k, v, o, lse, args, fwd_rows(w.seqlen_q))
    check_bwd(name, q, k, v, do, grads, args, bwd_rows(w.seqlen_q, 64, 1024, 21),
              bwd_rows(w.seqlen_k, 128, 256, 22))


def test_gqa_window_every_row(attn):
    name = "gqa_window_b4_h32_kv8_n4096_d128"
    w = WORKLOADS[name]
    (q, k, v, do), o, lse, grads, args = run(attn, w, True)
    check_fwd(name, q, k, v, o, lse, args)
    check_bwd(name, q, k, v, do, grads, args)


def test_long_fp16_d256_fwd_sampled(attn):
    name = "long_fp16_b1_h8_n65536_d256"
    w = WORKLOADS[name]
    (q, k, v, _), o, lse, _, args = run(attn, w, False)
    check_fwd(name, q, k, v, o, lse, args, fwd_rows(w.seqlen_q))


def test_long_fp16_d256_bwd_sampled(attn):
    """The backward at the long-sequence head-dim-256 shape (N = 65536, fp16,
    causal, the same input distribution) with one head: the oracle needs
    every query row's statistics for the key gradients, so its cost grows
    with N^2 d per head.  Query rows at every 64- and 128-row tile edge (the
    two kernel tilings of the queries), key rows at every 128-key tile edge."""
    w = WORKLOADS["long_fp16_b1_h8_n65536_d256"].replace(
        name="long_fp16_b1_h1_n65536_d256", nheads=1, nheads_kv=1, passes="fwd+bwd")
    (q, k, v, do), o, lse, grads, args = run(attn, w, True)
    _identities(w, do, grads[1], grads[2])
    check_bwd(w.name, q, k, v, do, grads, args, bwd_rows(w.seqlen_q, 64, 1024, 31),
              bwd_rows(w.seqlen_k, 128, 256, 32))
