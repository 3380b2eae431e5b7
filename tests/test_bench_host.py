"""bench.py host logic on the CPU: FLOP accounting, the exact visible-pair
count, clock-sample parsing, and the multi-rank path (world size 2, gloo):
barrier and the maximum over ranks that the timing uses."""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from attn_inputs import WORKLOADS
from oracle_pins import mask_matrix


def test_step_flops_formula():
    w = WORKLOADS["causal_b2_h32_n8192_d128"]
    fwd, bwd = bench.step_flops(w)
    assert fwd == 4 * 2 * 32 * 8192 * 8192 * 128 / 2
    assert bwd == 2.5 * fwd
    w2 = WORKLOADS["full_b1_h16_n16384_d128"]
    assert bench.step_flops(w2)[0] == 4 * 16 * 16384 ** 2 * 128


@pytest.mark.parametrize("nq,nk,causal,wl,wr", [
    (7, 7, True, -1, -1), (9, 5, True, 2, -1), (5, 9, False, 1, 3), (8, 8, False, -1, 0),
    (6, 6, False, 0, 0), (10, 4, True, -1, -1),
])
def test_visible_pairs_matches_brute_force(nq, nk, causal, wl, wr):
    vis = mask_matrix(nq, nk, causal=causal, window_left=wl, window_right=wr)
    assert bench.visible_pairs(nq, nk, causal, wl, wr) == int(vis.sum())
    rows = [0, nq - 1]
    assert bench.visible_pairs(nq, nk, causal, wl, wr, rows=rows) == int(vis[rows].sum())


def test_window_workload_pair_count():
    w = WORKLOADS["gqa_window_b4_h32_kv8_n4096_d128"]
    # min(i, 1024) + 1 keys per query
    assert bench.visible_pairs(w.seqlen_q, w.seqlen_k, w.causal, w.window_left, w.window_right) == \
        sum(min(i, 1024) + 1 for i in range(4096)) == 3673600


def test_clock_summary_parsing():
    """Only samples that arrived while the timed region ran count; a region
    shorter than the sampling period takes the sample nearest its middle."""
    c = bench.ClockSampler(0)
    c.t0, c.t1 = 10.0, 10.1
    c.samples = [
        (9.9, "1100, 1965, 300.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"),
        (10.02, "1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"),
        (10.05, "1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active"),
        (10.09, "1320, 1965, 1001.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active"),
        (10.5, "900, 1965, 100.0, 0x0000000000000000, Active, Not Active, Not Active, Not Active"),
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    c.t0, c.t1 = 10.2, 10.21
    s = c.summary()
    assert s["samples"] == 1 and s["sm_mhz"] == 1320


def test_peaks_loaded_or_fallback():
    peaks, kind = bench.load_peaks()
    assert kind in ("measured", "fallback")
    assert peaks["bf16_tflops"] > 1000 and peaks["hbm_gbs"] > 1000


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    r, lr, ws = bench.world_info()
    dist = bench.init_dist("gloo", ws)
    bench.barrier(dist)
    # each rank "measured" a different time; the job time is the slowest rank's
    got = bench.max_over_ranks(10.0 + 5.0 * r, dist)
    bench.barrier(dist)
    q.put((r, lr, ws, got))
    dist.destroy_process_group()


def test_two_ranks_gloo_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[2] == 2 for r in res)
    assert all(r[3] == 15.0 for r in res)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_varlen_flops_match_closed_form():
    """The packed workload's FLOPs: every causal sequence of L tokens has
    L (L + 1) / 2 visible pairs (4 d FLOPs each forward, 2.5x backward)."""
    import bench
    from attn_inputs import VARLEN_WORKLOADS
    w = VARLEN_WORKLOADS["varlen_causal_16seq_h32_d128"]
    pairs = sum(n * (n + 1) // 2 for n in w.lens)
    f, b = bench.varlen_flops(w)
    assert f == 4.0 * w.nheads * w.headdim * pairs and b == 2.5 * f
    assert len(w.lens) == 16 and all(256 <= n <= 1792 for n in w.lens)
    cfg = bench.varlen_config(w)
    assert cfg["tokens"] == sum(w.lens) and cfg["workload"] == w.name


def test_reference_arm_declines_packed_workload(capsys):
    import bench
    assert bench.main(["--impl", "reference", "--workload", "varlen_causal_16seq_h32_d128",
                       "--steps", "1", "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and "unavailable" in line


def test_exact_pair_flops():
    import bench
    w = WORKLOADS["causal_b2_h32_n8192_d128"]
    f, b = bench.exact_pair_flops(w)
    n = w.seqlen_q
    assert f == 4.0 * w.batch * w.nheads * (n * (n + 1) // 2) * w.headdim and b == 2.5 * f
    fc, _ = bench.step_flops(w)
    assert 1.0 < f / fc < 1.0 + 2.0 / n
    w4 = WORKLOADS["gqa_window_b4_h32_kv8_n4096_d128"]
    assert bench.exact_pair_flops(w4) == bench.step_flops(w4)  # windows already count exactly


def test_environment_is_best_effort():
    import bench

    class NoGpu:
        __version__ = "x"

        class version:
            cuda = None

        class cuda:
            @staticmethod
            def get_device_properties(dev):
                raise RuntimeError("no device")

    env = bench.environment(NoGpu, torch.device("cpu"))
    assert env["torch"] == "x" and "gpu" not in env


def test_reference_arm_line(capsys):
    """The reference arm runs the float64 oracle on the host and prints one
    JSON line with the contract's keys (rank 0 of a single process)."""
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(key, None)
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    out = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == bench.UNIT and line["value"] > 0 and line["steps"] == 1
    assert line["higher_is_better"] is True and line["dtype"] == "f64"
    assert line["config"]["workload"] == bench.WORKLOAD
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"]
    assert "queries" in cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_extra_workloads(capsys):
    """The decode and FP8 workloads exist, read more than the L2 per step,
    and the reference arm declines them (it times the headline only)."""
    from attn_inputs import EXTRA_WORKLOADS
    dec = EXTRA_WORKLOADS["decode_b8_h32_kv8_n32768_d128"]
    assert dec.seqlen_q == 1 and dec.nheads // dec.nheads_kv * dec.seqlen_q <= 16
    assert bench.input_bytes(dec) > 8 * 126e6
    fp8 = EXTRA_WORKLOADS["fp8_causal_b2_h32_n8192_d128"]
    assert (fp8.batch, fp8.nheads, fp8.seqlen_q, fp8.headdim, fp8.causal) == (2, 32, 8192, 128, True)
    for name in EXTRA_WORKLOADS:
        assert bench.main(["--impl", "reference", "--workload", name]) == 0
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert line["impl"] == "reference" and "unavailable" in line


def test_traffic_record_is_per_workload_and_sources(tmp_path, monkeypatch):
    """The committed DRAM-traffic record applies only to the workload it was
    captured on, at its own size, and only while the kernel sources hash the
    same; any other case reports null."""
    rec = {"attn_fwd_kernel": {"bytes_per_launch": 123.0, "source_hash": bench.kernel_source_hash(),
                               "workload": "causal_b2_h32_n8192_d128"}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["attn_fwd_kernel"]["source_hash"])
    assert bench.recorded_traffic("attn_fwd_kernel", "causal_b2_h32_n8192_d128") == 123.0
    assert bench.recorded_traffic("attn_fwd_kernel", "long_fp16_b1_h8_n65536_d256") is None
    assert bench.recorded_traffic("attn_fwd_kernel", None) is None  # --seqlen override
    assert bench.recorded_traffic("attn_bwd_kernel", "causal_b2_h32_n8192_d128") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("attn_fwd_kernel", "causal_b2_h32_n8192_d128") is None


def test_passes_and_seqlen_overrides_refuse_l2_sized_cases(capsys):
    """--seqlen shrinks a workload for profiling; a case whose inputs fit in
    twice the L2 is refused (it would time L2, not HBM)."""
    with pytest.raises(SystemExit):
        bench.main(["--workload", "long_fp16_b1_h8_n65536_d256", "--passes", "fwd+bwd",
                    "--seqlen", "16384"])
    assert "fits in L2" in capsys.readouterr().err
    with pytest.raises(SystemExit):
        bench.main(["--passes", "bwd-only"])
