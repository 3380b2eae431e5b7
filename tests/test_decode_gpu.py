"""The decode path (attn_fwd_decode: a few query rows against a long key /
value sequence, CUDA cores, keys split over blocks and merged) on the GPU
against the float64 oracle: GQA groups with one and several query tokens,
MHA, causal (bottom-right) and sliding-window masks, head dims 64 and 128,
fp16, short key sequences that leave splits empty, no keys; and the
limits it refuses."""
import pytest
import torch

import oracle
from attn_inputs import Workload, make_inputs
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import io_aware_exact_33_b200 as m
    return m


def W(name, B, H, Hkv, Nq, Nk, d, causal=True, wl=-1, wr=-1, dtype="bf16", seed=970):
    return Workload(name, B, H, Hkv, Nq, Nk, d, causal, wl, wr, dtype, 1.0, seed)


CASES = [
    W("gqa8_one_token", 2, 32, 4, 1, 5000, 128, seed=971),
    W("gqa4_four_tokens", 1, 16, 4, 4, 3000, 128, seed=972),
    W("mha_d64_fp16", 2, 8, 8, 3, 2049, 64, dtype="fp16", seed=973),
    W("window", 1, 8, 2, 2, 4000, 128, wl=1024, seed=974),
    W("full_mask", 1, 4, 2, 2, 777, 128, causal=False, seed=975),
    W("short", 3, 4, 1, 1, 70, 128, seed=976),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_decode_parity(attn, w):
    q, k, v, _ = make_inputs(w, with_dout=False)
    o, lse = attn.attn_fwd_decode(q.cuda(), k.cuda(), v.cuda(), w.scale, w.causal,
                                  w.window_left, w.window_right)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.scale, w.causal, w.window_left,
                                          w.window_right)
    check_o(o.cpu(), o_ref, w.name)
    check_lse(lse.cpu(), lse_ref, w.name)


def test_decode_no_keys_and_limits(attn):
    q = torch.randn(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda")
    k0 = torch.zeros(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    o, lse = attn.attn_fwd_decode(q, k0, k0)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isinf(lse))
    k = torch.randn(1, 64, 1, 128, dtype=torch.bfloat16, device="cuda")
    q17 = torch.randn(1, 17, 1, 128, dtype=torch.bfloat16, device="cuda")  # 17 rows > 16
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_decode(q17, k, k)
    q256 = torch.randn(1, 1, 1, 256, dtype=torch.bfloat16, device="cuda")
    k256 = torch.randn(1, 64, 1, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_decode(q256, k256, k256)
