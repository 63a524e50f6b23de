"""bench.py's host logic on the CPU: roofline arithmetic, peaks fallback, the
max-over-ranks reduction on two gloo ranks, and the reference arm's rank rule."""

import io
import json
import os
import socket
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_roofline_value_arithmetic():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 90.0}
    # 1e12 FLOP at 100 TFLOP/s = 10 ms, 1e9 B at 1000 GB/s = 1 ms -> 11 ms of roofline work
    assert bench.roofline_value(1e12, 1e9, 0.022, peaks) == pytest.approx(50.0)
    assert bench.roofline_value(1e12, 1e9, 0.022, peaks, n_ranks=4) == pytest.approx(200.0)


def test_tensor_peak_burst_below_one_second_sustained_above():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 90.0}
    # the driver's 20-step region (~23 ms) runs at burst clocks
    peak, why = bench.tensor_peak(peaks, 0.023)
    assert peak == 100.0 and "burst" in why and "0.023" in why
    # a region of seconds of back-to-back work runs under the power cap
    peak, why = bench.tensor_peak(peaks, 1.2)
    assert peak == 90.0 and "sustained" in why
    # the boundary itself counts as sustained
    assert bench.tensor_peak(peaks, bench.SUSTAINED_AFTER_S)[0] == 90.0


def test_peaks_fallback(tmp_path):
    p, src = bench.load_peaks(str(tmp_path / "missing.json"))
    assert src == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0, "bf16_tflops_sustained": 3.0}))
    p, src = bench.load_peaks(str(f))
    assert src == "measured" and p == {"hbm_gbs": 1.0, "bf16_tflops": 2.0,
                                       "bf16_tflops_sustained": 3.0}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.reduce_max([float(rank), 10.0 - rank, 2.5], dist)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [1.0, 10.0, 2.5]


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert buf.getvalue() == ""
