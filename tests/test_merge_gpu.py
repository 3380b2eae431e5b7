"""attn_merge: partial forward results over disjoint key ranges, merged on
the GPU, against the oracle over all keys and against the oracle's merge of
the same partials (non-causal with GQA and an empty range, causal split-KV
decoding, fp16 with d = 64 and 256, rows no part sees)."""
import numpy as np
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


CASES = [
    # name, B, H, Hkv, Nq, Nk, d, dtype, causal, cuts
    ("noncausal_gqa", 2, 4, 2, 200, 1000, 128, "bf16", False, (0, 300, 300, 777, 1000)),
    ("causal_decode", 2, 8, 2, 4, 3000, 128, "bf16", True, (0, 1000, 2000, 3000)),
    ("d64_fp16", 1, 2, 2, 130, 513, 64, "fp16", False, (0, 128, 129, 513)),
    ("d256_fp16", 1, 2, 1, 64, 700, 256, "fp16", False, (0, 350, 700)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_merge_split_kv(attn, case):
    name, B, H, Hkv, Nq, Nk, d, dtype, causal, cuts = case
    w = Workload(name, B, H, Hkv, Nq, Nk, d, causal, -1, -1, dtype, 1.0, 600 + len(name))
    q, k, v, _ = make_inputs(w, with_dout=False)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    parts_o, parts_l = [], []
    for a, z in zip(cuts, cuts[1:]):
        o_p, l_p = attn.attn_fwd(qc, kc[:, a:z].contiguous(), vc[:, a:z].contiguous(), w.scale,
                                 causal and z == Nk)
        parts_o.append(o_p)
        parts_l.append(l_p)
    po, pl = torch.stack(parts_o), torch.stack(parts_l)
    o, lse = attn.attn_merge(po, pl)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    # against the definition over all keys
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, w.scale, causal)
    check_o(o.cpu(), o_ref, name)
    check_lse(lse.cpu(), lse_ref, name)
    # against the oracle's merge of the same (16-bit) partials
    om_ref, lm_ref = oracle.attention_merge(po.cpu(), pl.cpu())
    check_o(o.cpu(), om_ref, name + " (same partials)")
    check_lse(lse.cpu(), lm_ref, name + " (same partials)")


def test_merge_rows_no_part_sees(attn):
    po = torch.zeros(3, 1, 5, 2, 128, dtype=torch.bfloat16, device="cuda")
    pl = torch.full((3, 1, 2, 5), -float("inf"), device="cuda")
    pl[1, 0, 1, 2] = 0.5  # one row seen by one part
    po[1, 0, 2, 1] = 1.0
    o, lse = attn.attn_merge(po, pl)
    torch.cuda.synchronize()
    lse_c = lse.cpu()
    assert torch.isinf(lse_c).sum() == 9 and abs(lse_c[0, 1, 2].item() - 0.5) < 1e-6
    assert torch.all(o.cpu()[0, 2, 1] == 1.0)
    mask = torch.ones(5, 2, dtype=torch.bool)
    mask[2, 1] = False
    assert torch.all(o.cpu()[0][mask] == 0)
