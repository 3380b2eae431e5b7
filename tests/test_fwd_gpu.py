"""Forward parity: the sm_100a kernels against the float64 oracle on the same
seeded inputs, element by element (full outputs at small sizes; sampled rows
at the full workload sizes)."""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import WORKLOADS, Workload, make_inputs, sample_rows
from parity import check_lse, check_o, check_o_derived

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def run_fwd(attn, w: Workload):
    q, k, v, _ = make_inputs(w, with_dout=False)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), w.scale, w.causal, w.window_left,
                           w.window_right)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    return (q, k, v), o.cpu(), lse.cpu()


def full_check(attn, w: Workload):
    (q, k, v), o, lse = run_fwd(attn, w)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.scale, w.causal, w.window_left, w.window_right)
    check_o(o, o_ref, w.name)
    check_lse(lse, lse_ref, w.name)


def W(name, B, H, Hkv, Nq, Nk, d, causal=False, wl=-1, wr=-1, dtype="bf16", seed=100, sigma=1.0):
    return Workload(name, B, H, Hkv, Nq, Nk, d, causal, wl, wr, dtype, sigma, seed)


SMALL = [
    W("d64_n128", 1, 2, 2, 128, 128, 64),
    W("d128_n128", 1, 2, 2, 128, 128, 128),
    W("d256_n128", 1, 2, 2, 128, 128, 256),
    W("d128_ragged_300", 2, 4, 4, 300, 300, 128, seed=101),
    W("d128_causal_513", 1, 3, 3, 513, 513, 128, causal=True, seed=102),
    W("d64_causal_ragged", 2, 2, 1, 200, 200, 64, causal=True, seed=103),
    W("d256_causal_ragged", 1, 2, 2, 333, 333, 256, causal=True, seed=104),
    W("d128_fp16", 1, 4, 2, 256, 256, 128, dtype="fp16", seed=105),
    W("d256_fp16_causal", 1, 2, 2, 384, 384, 256, causal=True, dtype="fp16", seed=106, sigma=0.5),
    W("gqa4_window", 2, 8, 2, 700, 700, 128, causal=True, wl=129, wr=0, seed=107),
    W("gqa8_window_edge", 1, 8, 1, 640, 640, 128, causal=True, wl=127, seed=108),
    W("window_128_noncausal", 1, 2, 2, 500, 500, 128, wl=128, wr=128, seed=109),
    W("window_right_only", 1, 2, 2, 260, 260, 64, wr=3, seed=110),
    W("nq_lt_nk_causal", 2, 2, 2, 100, 390, 128, causal=True, seed=111),
    W("nq_gt_nk_causal_empty_rows", 1, 2, 2, 300, 130, 128, causal=True, seed=112),
    W("nq_gt_nk_noncausal", 1, 2, 1, 257, 65, 64, seed=113),
    W("single_row", 1, 1, 1, 1, 1, 128, seed=114),
    W("single_query_long_keys", 1, 2, 2, 1, 1000, 128, causal=True, seed=115),
]

# Inputs ~N(0, 3^2): scores 9x wider than the stated regime, so the running
# max moves by more than the rescale threshold; checked against the bound
# derived from 16-bit P instead of the flat 1e-2.
WIDE = [
    W("wide_scores", 1, 2, 2, 256, 256, 128, seed=116, sigma=3.0),
    W("wide_scores_causal", 1, 2, 2, 384, 384, 128, causal=True, seed=117, sigma=3.0),
    W("wide_scores_fp16", 1, 2, 2, 256, 256, 64, dtype="fp16", seed=118, sigma=3.0),
]


@pytest.mark.parametrize("w", WIDE, ids=lambda w: w.name)
def test_fwd_wide_scores(attn, w):
    (q, k, v), o, lse = run_fwd(attn, w)
    args = (w.scale, w.causal, w.window_left, w.window_right)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, *args)
    pabs, _ = oracle.attention_fwd(q, k, v.abs(), *args)
    check_o_derived(o, o_ref, pabs, w.name)
    check_lse(lse, lse_ref, w.name)


# Many short work units (at least four per SM, at most 12 key tiles per
# query tile on average, no slopes or dropout): these run the persistent
# forward, each CTA taking a unit after another.
PERSIST = [
    W("persist_causal_ragged", 6, 32, 32, 1000, 1000, 128, causal=True, seed=130),
    W("persist_window_gqa", 4, 40, 8, 2048, 2048, 128, causal=True, wl=512, seed=131),
    W("persist_full_short", 16, 16, 16, 640, 640, 128, seed=132),
    W("persist_d64_fp16", 8, 48, 12, 700, 700, 64, causal=True, dtype="fp16", seed=133),
    W("persist_nq_lt_nk", 20, 32, 16, 300, 900, 128, causal=True, seed=134),
    W("persist_window_both", 6, 32, 32, 1500, 1500, 128, wl=200, wr=100, seed=135),
]


@pytest.mark.parametrize("w", PERSIST, ids=lambda w: w.name)
def test_fwd_persistent_full(attn, w):
    full_check(attn, w)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fwd_small_full(attn, w):
    full_check(attn, w)


def test_fwd_tiny_workload(attn):
    full_check(attn, WORKLOADS["tiny_b1_h2_n128_d64"])


@pytest.mark.parametrize("name", ["causal_b2_h32_n8192_d128", "full_b1_h16_n16384_d128",
                                  "gqa_window_b4_h32_kv8_n4096_d128",
                                  "long_fp16_b1_h8_n65536_d256"])
def test_fwd_full_size_sampled_rows(attn, name):
    w = WORKLOADS[name]
    (q, k, v), o, lse = run_fwd(attn, w)
    must = [1, 2, 127, 128, 129, w.seqlen_q // 2]
    if w.window_left >= 0:
        must += [w.window_left - 1, w.window_left, w.window_left + 1, w.window_left + 128]
    rows = sample_rows(w.seqlen_q, 24, w.seed, must=must)
    o_ref, lse_ref = oracle.attention_fwd_rows(q, k, v, rows, w.scale, w.causal, w.window_left,
                                               w.window_right)
    check_o(o[:, rows], o_ref, name)
    check_lse(lse[:, :, rows], lse_ref, name)
    # every row, any size: finite output, and |O| bounded by max |V| (a convex combination)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert o.abs().max() <= v.abs().max() * 1.001 + 1e-3


def test_fwd_no_keys(attn):
    w = W("no_keys", 2, 2, 2, 50, 0, 128)
    q = torch.randn(2, 50, 2, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.empty(2, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd(q, k, k.clone(), w.scale)
    torch.cuda.synchronize()
    assert (o == 0).all() and torch.isneginf(lse).all()


def test_fwd_no_queries(attn):
    q = torch.empty(1, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(1, 10, 2, 64, dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd(q, k, k.clone())
    assert o.shape == (1, 0, 2, 64) and lse.shape == (1, 2, 0)


def test_fwd_rejects_bad_arguments(attn):
    q = torch.randn(1, 16, 2, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError) as e:
        attn.attn_fwd(q, q.clone(), q.clone())
    assert e.value.status == 2
    buf = torch.empty(16 * 2 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    qm = buf[1:1 + 16 * 2 * 128].view(1, 16, 2, 128)  # 2-byte offset: not 16-byte aligned
    k = torch.randn(1, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError) as e:
        attn.attn_fwd(qm, k, k.clone())
    assert e.value.status == 4
    with pytest.raises(TypeError):
        attn.attn_fwd(k.float(), k.float(), k.float())


def test_fwd_repeatable(attn):
    w = W("repeat", 1, 4, 4, 300, 300, 128, causal=True, seed=120)
    (q, k, v), o1, l1 = run_fwd(attn, w)
    _, o2, l2 = run_fwd(attn, w)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
