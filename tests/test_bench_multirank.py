"""The benchmark's multi-rank plumbing on CPU with two gloo ranks: each rank
gets its own batch of the same shape, timings reduce to the max over ranks,
and the whole-job value sums every rank's KV bytes over the slowest rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = bench.rank_workload("fp32_b1_n512", rank, world)
        local_ms = 10.0 + 5.0 * rank                # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"), dist)
        digest = float(w.k.double().sum())
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([digest], dtype=torch.float64))
        q.put((rank, ms, tuple(w.k.shape), [float(x) for x in sums], w.kv_bytes()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (_, ms0, shape0, sums0, kvb), (_, ms1, shape1, sums1, _) = res
    assert ms0 == ms1 == 15.0                       # both ranks see the slowest rank
    assert shape0 == shape1                         # same shape per rank (weak scaling)
    assert sums0 == sums1 and sums0[0] != sums0[1]  # different data per rank
    assert bench.whole_job_gbs(kvb, 2, ms0 / 1000) == pytest.approx(2 * kvb / 15e-6 / 1e9)


def test_single_rank_identity():
    assert bench.max_over_ranks(3.5, torch.device("cpu"), None) == 3.5
    w = bench.rank_workload("fp32_b1_n512", 0, 1)
    assert w.name == "fp32_b1_n512" and w.kv_bytes() == 1 << 20


def test_clock_summary_of_sampled_lines():
    """The clocks record: median SM clock, the highest max clock, and every
    throttle reason seen Active; malformed or unavailable samples are skipped."""
    lines = [
        "0, 1965, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 1000.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 10.0, 0x0, Not Active, Active, Not Active, Not Active",   # unavailable: skipped
        "garbage line",
    ]
    c = bench.ClockSampler.summarize(lines)
    assert c == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert bench.ClockSampler.summarize([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                                                "samples": 0}
