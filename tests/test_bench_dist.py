"""The bench's multi-rank plumbing on CPU (gloo, world size 2): every rank runs
an independent replica; the whole-job value is the units of all ranks over the
slowest rank's time, and only rank 0 prints the reference arm."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        ms_rank = [4.0, 5.0][rank]          # rank 1 is the slower replica
        units_rank = [256.0, 256.0][rank]
        value, ms = bench.aggregate(units_rank, ms_rank, world, dev)
        mx = bench.reduce_max(float(rank) + 0.5, world, dev)
        sm = bench.reduce_sum(float(rank) + 1.0, world, dev)
        bench.barrier(world)
        out[rank] = (value, ms, mx, sm)
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(rank_main, args=(2, free_port(), out), nprocs=2, join=True,
                       start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for rank in (0, 1):
        value, ms, mx, sm = out[rank]
        assert ms == 5.0                      # the slowest rank's time
        assert value == pytest.approx(512.0 / 5e-3)   # all ranks' units / that time
        assert mx == 1.5 and sm == 3.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "tiny"
        steps = 1
        warmup = 0
        ref_seconds = 0.01

    bench.reference_arm(Args, world=2, rank=1)
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(capsys):
    """--impl reference: the oracle timed on the host, one JSON line with the
    contract's keys (a bounded sample of the tiny workload)."""
    import json
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "tiny"
        steps = 2
        warmup = 1
        ref_seconds = 0.01

    bench.reference_arm(Args, world=1, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["config"]["workload"] == "tiny"


def test_profile_traffic_only_while_the_sources_match(tmp_path):
    """roofline.traffic comes from a committed ncu summary only while the
    kernel's sources hash to the value recorded with it."""
    sys.path.insert(0, ROOT)
    import bench
    good = tmp_path / "good.md"
    good.write_text(f"- sources sha256: `{bench.kernel_source_hash()}`\n"
                    "- dram bytes per launch (read + write): 123456\n")
    assert bench.profile_traffic(str(good)) == 123456.0
    stale = tmp_path / "stale.md"
    stale.write_text("- sources sha256: `" + "0" * 64 + "`\n"
                     "- dram bytes per launch (read + write): 123456\n")
    assert bench.profile_traffic(str(stale)) is None
    assert bench.profile_traffic(str(tmp_path / "absent.md")) is None


def test_doc_roofline_peak_choice_and_the_stricter_gate():
    """The document pass's roofline: roof time = the slower of the bytes at
    the measured copy rate and the FLOPs at the bf16 rate (burst for a short,
    cool run; sustained for a long or power-capped one); frac = roof time /
    measured time.  The nominal figures give the stricter gate."""
    sys.path.insert(0, ROOT)
    import bench
    from shared_context_decode_b200 import workloads as wl
    W = wl.make_decode("doc16k_p256", device="cpu")
    peaks = dict(hbm=6548.0, bf16=1629.0, bf16_sustained=1390.0, source="measured")
    r = bench.doc_roofline(W, {"doc": 0.0725, "suffix": 0.0594}, peaks, None)
    b, f = 2 * 16384 * 32 * 128 * 2, 4 * 256 * 16384 * 128 * 32
    t_roof = max(b / 6548e9, f / 1629e12)
    assert r["bound"] == "tensor" and r["peak"] == 1629.0
    assert r["frac"] == pytest.approx(t_roof / 72.5e-6)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["frac_spec"] == pytest.approx(max(b / 8e12, f / 2.25e15) / 72.5e-6)
    assert r["frac_gate"] == pytest.approx(min(r["frac"], r["frac_spec"]))
    assert r["frac_sustained"] > r["frac"]
    assert r["frac_burst"] == pytest.approx(r["frac"]) and r["tensor_peak"] == "burst bf16"
    # a long or power-capped run is held to the sustained peak
    rs = bench.doc_roofline(W, {"doc": 0.0725, "suffix": 0.0594}, peaks, None, sustained=True)
    assert rs["peak"] == 1390.0 and rs["tensor_peak"] == "sustained bf16"
    assert rs["frac"] == pytest.approx(max(b / 6548e9, f / 1390e12) / 72.5e-6)
    assert rs["frac"] == pytest.approx(r["frac_sustained"])
    assert rs["frac_burst"] == pytest.approx(r["frac"])
    # a memory-bound workload (64 streams) is bound by HBM
    W2 = wl.make_decode("doc8k_p64", device="cpu")
    r2 = bench.doc_roofline(W2, {"doc": 0.030, "suffix": 0.010}, peaks, None)
    assert r2["bound"] == "hbm" and r2["unit"] == "GB/s"
    assert r2["frac"] == pytest.approx((2 * 8192 * 32 * 128 * 2 / 6548e9) / 30e-6)


def test_sweep_roof_time_by_hand():
    """The sweep's roof time on a two-stream, two-step case worked by hand:
    step 0 both streams active, step 1 only stream 1."""
    sys.path.insert(0, ROOT)
    import bench

    class W:
        N, P, H, d = 1000, 2, 4, 64
        q_len = np.array([10, 20])

    peaks = dict(hbm=1000.0, bf16=1000.0)
    kvb = 4 * 64 * 2 * 2
    # step 0: segments 11 + 21 tokens; step 1: stream 1 only, 12 tokens
    b0 = 3 * (1000 * kvb + 32 * kvb + 2 * 2 * kvb + 2 * kvb)
    f0 = 3 * 4.0 * 64 * 4 * (2 * 1000 + 32)
    b1 = 3 * (1000 * kvb + 12 * kvb + 2 * 1 * kvb + 2 * kvb)
    f1 = 3 * 4.0 * 64 * 4 * (1 * 1000 + 12)
    want = sum(max(b / 1e12, f / 1e15) for b, f in ((b0, f0), (b1, f1))) * 1e3
    got = bench.sweep_roof_ms(W, np.array([2, 1]), 2, 3, peaks)
    assert got == pytest.approx(want)
