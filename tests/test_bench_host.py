"""Host logic of bench.py: byte/flop accounting, clock parsing and the multi-rank
timing reduction (world size 2 over gloo on CPU; each rank is an independent
replica, so the only collectives are the barrier and the max over ranks).
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def test_decode_bytes_accounting():
    # 4096 x 4096 signs = 2 MiB, plus a, b (fp32) and X, Y (bf16).
    assert bench.decode_call_bytes(1) == 2 * 1024 * 1024 + 4 * 4096 * 2 + 2 * 4096 * 2
    assert bench.step_bytes(2) == 2 * sum(bench.decode_call_bytes(m) for m in (1, 4, 16))
    assert bench.step_flops(1) == 2 * 21 * 4096 * 4096
    # the pool is larger than three times a 126 MB L2
    assert bench.LAYERS * bench.decode_call_bytes(0) > 3 * 126e6


def test_peaks_loaded():
    p = bench.load_peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    assert p["source"] in ("measured", "fallback")


def test_clock_summary_parsing(tmp_path):
    s = bench.ClockSampler(0)
    f = tmp_path / "c.csv"
    f.write_text("0, 1800, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Active\n"
                 "0, 1900, 1965, 600.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                 "0, 1700, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")

    class _P:  # stands in for the finished sampler process
        pass

    s.proc = _P()
    s.file = open(f)
    out = s.summary()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # Each replica times its own step; the job time is the slowest rank.
        local_ms = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(local_ms, world)
        value = world * bench.step_bytes(1) / (ms * 1e-3) / 1e9
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]  # max over ranks on both
    assert res[0][2] == res[1][2] == pytest.approx(2 * bench.step_bytes(1) / 15e-3 / 1e9)
