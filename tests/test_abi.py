"""The C ABI without a GPU: the library loads, exports every declared entry
point, and its pure host functions (argument checks, workspace sizes, status
strings) behave as include/attn.h states."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def attn():
    from io_aware_exact_33_b200 import build
    build.build()
    import io_aware_exact_33_b200 as m
    return m


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    syms = declared_symbols()
    assert "attn_fwd" in syms and "attn_bwd" in syms
    assert len(syms) >= 8


def test_library_exports_every_declared_symbol(attn):
    lib = ctypes.CDLL(attn.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), f"libattn.so does not export {name}"
    assert set(attn.EXPORTED) <= set(declared_symbols())


def test_version_and_status_strings(attn):
    assert re.match(r"^\d+\.\d+\.\d+$", attn.attn_version())
    for code in range(0, 9):
        s = attn.attn_status_string(code)
        assert s and s != "unknown status"
    assert attn.attn_status_string(99) == "unknown status"


def P(attn, **kw):
    base = dict(batch=2, seqlen_q=100, seqlen_k=90, nheads=8, nheads_kv=2, headdim=128,
                dtype=attn.ATTN_BF16, softmax_scale=None, causal=False, window_left=-1,
                window_right=-1)
    base.update(kw)
    return attn.make_params(**base)


def test_check_params_accepts_valid(attn):
    for d in (64, 128, 256):
        assert attn.attn_check_params(P(attn, headdim=d), 0) == 0
    for d in (64, 128):
        assert attn.attn_check_params(P(attn, headdim=d), 1) == 0
    assert attn.attn_check_params(P(attn, dtype=attn.ATTN_FP16, causal=True, window_left=5,
                                    window_right=0), 0) == 0
    assert attn.attn_check_params(P(attn, seqlen_q=0, seqlen_k=0, batch=0), 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(nheads=6, nheads_kv=4), 1),
    (dict(nheads_kv=0), 1),
    (dict(batch=-1), 1),
    (dict(seqlen_q=-5), 1),
    (dict(softmax_scale=0.0), 1),
    (dict(softmax_scale=-1.0), 1),
    (dict(softmax_scale=float("inf")), 1),
    (dict(window_left=-2), 1),
    (dict(window_right=-3), 1),
    (dict(headdim=96), 2),
    (dict(headdim=32), 2),
    (dict(dtype=7), 3),
])
def test_check_params_rejects(attn, kw, code):
    assert attn.attn_check_params(P(attn, **kw), 0) == code


def test_bwd_headdim_256_checks(attn):
    """The backward takes head dim 256 without dropout only."""
    assert attn.attn_check_params(P(attn, headdim=256), 1) == 0
    assert attn.attn_check_params(P(attn, headdim=256, dropout_p=0.1), 1) == 2
    assert attn.attn_check_params(P(attn, headdim=96), 1) == 2


def test_causal_flag_must_be_boolean(attn):
    p = P(attn)
    p.causal = 2
    assert attn.attn_check_params(p, 0) == 1


def test_workspace_sizes(attn):
    p = P(attn, batch=2, seqlen_q=100, nheads=8, headdim=128)
    assert attn.attn_fwd_workspace_size(p) == 0
    ws = attn.attn_bwd_workspace_size(p)
    nq_pad = 128
    rows = 2 * 8 * nq_pad * 4
    acc = 2 * 100 * 8 * 128 * 4
    assert ws >= 2 * rows + acc
    assert ws % 256 == 0
    assert attn.attn_bwd_workspace_size(P(attn, headdim=96)) == 0


def test_alibi_pointer_alignment(attn):
    p = P(attn)
    p.alibi_slopes = 2  # not 4-byte aligned; never dereferenced on the host
    assert attn.attn_check_params(p, 0) == 4  # ATTN_ERR_MISALIGNED
    p.alibi_slopes = 256
    assert attn.attn_check_params(p, 0) == 0


def test_dropout_checks(attn):
    """dropout_p must be in [0, 255.5 / 256) (its threshold round(256 p) at
    most 255); the headdim-256 forward has no dropout variant, but a rate
    that rounds to threshold 0 is no dropout and passes."""
    assert attn.attn_check_params(P(attn, dropout_p=0.1, dropout_seed=7), 0) == 0
    assert attn.attn_check_params(P(attn, dropout_p=0.1), 1) == 0
    for bad in (-0.1, 1.0, 0.999, float("nan"), float("inf")):
        assert attn.attn_check_params(P(attn, dropout_p=bad), 0) == 1, bad
    assert attn.attn_check_params(P(attn, headdim=256, dropout_p=0.1), 0) == 2
    assert attn.attn_check_params(P(attn, headdim=256, dropout_p=0.001), 0) == 0
    v = attn.make_varlen_params(2, 10, 10, 5, 5, 4, 2, 64, dropout_p=1.5)
    assert attn.attn_check_varlen_params(v, 0) == 1


def test_merge_host_checks(attn):
    """attn_merge rejects bad sizes before touching the GPU; an empty merge
    is a no-op."""
    def call(**kw):
        base = dict(splits=2, batch=1, seqlen_q=4, nheads=2, headdim=128, dtype=0)
        base.update(kw)
        p = attn.AttnMergeParams(*[base[n] for n, _ in attn.AttnMergeParams._fields_])
        return attn._lib.attn_merge(ctypes.byref(p), None, None, None, None, None)
    assert call(splits=0) == 1
    assert call(nheads=0) == 1
    assert call(headdim=96) == 2
    assert call(dtype=5) == 3
    assert call(batch=0) == 0
    assert call() == 1  # null pointers with work to do


def test_header_is_plain_c(attn, tmp_path):
    """include/attn.h compiles as strict C99 and a C program links against
    libattn.so and calls its host-only entry points (no GPU needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_attn.c"
    src.write_text(r"""
#include <stddef.h>
#include <stdio.h>
#include "attn.h"
int main(void) {
  attn_params p = {0};
  p.batch = 2; p.seqlen_q = 100; p.seqlen_k = 100; p.nheads = 8; p.nheads_kv = 2;
  p.headdim = 128; p.dtype = ATTN_BF16; p.softmax_scale = 0.088f;
  attn_varlen_params v = {0};
  v.batch = 3; v.total_q = 50; v.total_k = 60; v.max_seqlen_q = 20; v.max_seqlen_k = 30;
  v.nheads = 8; v.nheads_kv = 2; v.headdim = 64; v.dtype = ATTN_FP16; v.softmax_scale = 0.125f;
  printf("%d %d %d %zu %zu %s\n", (int)attn_check_params(&p, 0), (int)attn_check_params(&p, 1),
         (int)attn_check_varlen_params(&v, 1), attn_bwd_workspace_size(&p),
         attn_bwd_varlen_workspace_size(&v), attn_version());
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(attn_params),
         offsetof(attn_params, dropout_p), offsetof(attn_params, dropout_offset),
         offsetof(attn_params, dropout_seed), sizeof(attn_varlen_params),
         offsetof(attn_varlen_params, dropout_p), offsetof(attn_varlen_params, dropout_offset),
         offsetof(attn_varlen_params, dropout_seed), offsetof(attn_params, pos_offset));
  return 0;
}
""")
    libdir = os.path.dirname(attn.LIB_PATH)
    exe = tmp_path / "use_attn"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lattn",
                    f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[:3] == ["0", "0", "0"]
    # the Python mirrors of the parameter structs have the C layout
    layout = [int(x) for x in out[6:15]]
    A, V = attn.AttnParams, attn.AttnVarlenParams
    assert layout == [ctypes.sizeof(A), A.dropout_p.offset, A.dropout_offset.offset,
                      A.dropout_seed.offset, ctypes.sizeof(V), V.dropout_p.offset,
                      V.dropout_offset.offset, V.dropout_seed.offset, A.pos_offset.offset]
    p = P(attn, batch=2, seqlen_q=100, seqlen_k=100, nheads=8, nheads_kv=2, headdim=128)
    assert int(out[3]) == attn.attn_bwd_workspace_size(p)
    assert int(out[4]) > 0 and out[5] == attn.attn_version()


def _decode_splits(pairs, tiles, slots):
    """The decode split rule: the split count (without empty splits) that
    minimises waves x (tiles per block + 2), fewest splits on ties."""
    best, best_s = None, 1
    for s in range(1, min(tiles, 4096) + 1):
        tps = -(-tiles // s)
        s_eff = -(-tiles // tps)
        cost = -(-(pairs * s_eff) // slots) * (tps + 2)
        if best is None or cost < best:
            best, best_s = cost, s_eff
    return best_s


def test_decode_host_checks(attn):
    """attn_fwd_decode's workspace follows its split rule (64-key tiles of
    the visible key range cut so that the blocks fill whole waves of the 148
    SMs, two blocks per SM for up to 8 query rows per kv head) and it
    refuses, before touching any pointer, more than 16 query rows per kv
    head, head dim 256 and positional slopes."""
    fn = attn._lib.attn_fwd_decode_workspace_size
    fn.argtypes = [ctypes.POINTER(attn.AttnParams)]
    fn.restype = ctypes.c_size_t
    for B, Nq, Nk, H, Hkv, wl, slots in ((2, 1, 5000, 32, 4, -1, 296),
                                         (8, 1, 32768, 32, 8, -1, 296),
                                         (1, 2, 4000, 8, 2, 1024, 296),
                                         (1, 3, 900, 16, 4, -1, 148)):
        p = P(attn, batch=B, seqlen_q=Nq, seqlen_k=Nk, nheads=H, nheads_kv=Hkv, causal=True,
              window_left=wl)
        lo = max(0, Nk - Nq - wl) if wl >= 0 else 0
        tiles = -(-(Nk - lo) // 64)
        splits = _decode_splits(B * Hkv, tiles, slots)
        rows = splits * B * Nq * H
        assert fn(ctypes.byref(p)) == -(-rows * 128 * 2 // 256) * 256 + -(-rows * 4 // 256) * 256
    call = attn._lib.attn_fwd_decode
    vp = ctypes.c_void_p
    call.argtypes = [ctypes.POINTER(attn.AttnParams), vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    call.restype = ctypes.c_int
    too_many = P(attn, seqlen_q=5, nheads=8, nheads_kv=2)  # 4 heads x 5 tokens = 20 rows
    assert call(ctypes.byref(too_many), None, None, None, None, None, None, 0, None) == 1
    assert call(ctypes.byref(P(attn, headdim=256)), None, None, None, None, None, None, 0,
                None) == 2
    slopes = P(attn, seqlen_q=1)
    slopes.alibi_slopes = 256
    assert call(ctypes.byref(slopes), None, None, None, None, None, None, 0, None) == 1


def test_backward_wrappers_refuse_host_tensors(attn):
    """attn_bwd and attn_bwd_noalloc check their tensors before any pointer
    reaches the library: host tensors are refused with ValueError."""
    import torch
    q = torch.zeros(1, 16, 2, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 16, 2, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 16)
    for fn in (attn.attn_bwd, attn.attn_bwd_noalloc):
        with pytest.raises(ValueError, match="CUDA"):
            fn(q, k, k, q, lse, q, 0.125)


def test_pos_offset_checks(attn):
    """pos_offset is accepted by the dense calls; the reserved word must be 0;
    the decode path refuses a nonzero offset before touching any pointer."""
    p = P(attn, pos_offset=-300)
    assert attn.attn_check_params(p, 0) == 0 and attn.attn_check_params(p, 1) == 0
    p.reserved0 = 1
    assert attn.attn_check_params(p, 0) == 1
    call = attn._lib.attn_fwd_decode
    vp = ctypes.c_void_p
    call.argtypes = [ctypes.POINTER(attn.AttnParams), vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    call.restype = ctypes.c_int
    q = P(attn, seqlen_q=1, pos_offset=5)
    assert call(ctypes.byref(q), None, None, None, None, None, None, 0, None) == 1
