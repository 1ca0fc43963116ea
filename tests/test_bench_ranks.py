"""The multi-rank host logic of bench.py, run as two gloo ranks on the CPU:
every rank ends with the slowest rank's time, the whole-job rate counts the
units of all ranks over that time, and the reference arm runs on rank 0
only (the other ranks exit without work)."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [12.5, 20.0][rank]
        slowest = bench.max_over_ranks(mine, dist, "cpu", world)
        rate = bench.job_rate(world, 100, 10, slowest)
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, rate in got:
        assert slowest == 20.0
        # 2 ranks x 100 units x 10 steps over 20 ms
        assert rate == pytest.approx(2 * 100 * 10 / 0.020)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, None, "cpu", 1) == 3.0
    assert bench.job_rate(1, 138, 5, 2.0) == pytest.approx(138 * 5 / 0.002)


def test_reference_arm_prints_only_on_rank_0(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps, warmup, gpus = 1, 1, 2
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.reference_arm(Args, "qwen2vl_2b")
    assert buf.getvalue() == ""


def test_peaks_read_flat_nested_partial_and_missing_files(tmp_path):
    """The roofline denominators come from the measured-peaks file whatever
    its shape (figures at the top level, one object down, or as records with
    a value); figures it lacks, and a missing or unreadable file, take the
    fallback values, and the source says which."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"hbm_gbs": 7000.5, "bf16_tflops": 1650.6, "bf16_tflops_sustained": 1354.2}))
    pk, src = bench.peaks(str(p))
    assert src == "measured" and pk == {"hbm_gbs": 7000.5, "bf16_tflops": 1650.6, "bf16_tflops_sustained": 1354.2}
    p.write_text(json.dumps({"gpu": {"hbm_gbs": {"value": 7001}, "bf16_tflops": 1600}, "clocks": [1965]}))
    pk, src = bench.peaks(str(p))
    assert pk["hbm_gbs"] == 7001.0 and pk["bf16_tflops"] == 1600.0
    assert pk["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert src.startswith("measured (hbm_gbs, bf16_tflops)") and "fallback" in src
    p.write_text("{not json")
    assert bench.peaks(str(p)) == (bench.FALLBACK_PEAKS, "fallback")
    assert bench.peaks(str(tmp_path / "absent.json")) == (bench.FALLBACK_PEAKS, "fallback")
    p.write_text(json.dumps({"hbm_gbs": 0, "bf16_tflops": True}))
    assert bench.peaks(str(p)) == (bench.FALLBACK_PEAKS, "fallback")
