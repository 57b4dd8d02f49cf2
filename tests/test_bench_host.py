"""Host-side logic of bench.py (CPU only): throughput aggregation, the
max-over-ranks reduction on a 2-rank gloo group, clock-sample parsing."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_throughput_is_whole_job():
    # 2 ranks x 1 token x 100 steps in a max of 5 ms -> 40000 tokens/s
    assert bench.throughput(1, 100, 2, 5.0) == pytest.approx(40000.0)
    assert bench.throughput(512, 10, 1, 1000.0) == pytest.approx(5120.0)


def test_parse_clock_samples():
    text = ("0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "0, 1900, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    c = bench.parse_clock_samples(text)
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 3
    assert bench.parse_clock_samples("") is None


def test_peak_and_sources_sha():
    peak, kind = bench.measured_peak_hbm()
    assert peak > 1000 and kind in ("measured", "fallback")
    assert bench.kernel_sources_sha() == bench.kernel_sources_sha()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank
        m = bench.reduce_max(local_ms)
        q.put((rank, m, bench.throughput(1, 100, world, m), bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_reduce_max_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]           # both ranks see the max
    assert res[0][2] == pytest.approx(2 * 100 / 0.015)   # whole-job tokens/s
    assert res[1][3] == (1, 2, 1)


def test_reduce_max_without_group_is_identity():
    assert not dist.is_initialized()
    assert bench.reduce_max(3.5) == 3.5
