"""Multi-rank host logic on the CPU: two gloo ranks, as bench.py runs N GPUs.

Each rank draws its own batch (seed offset = rank), times its own steps, and
the job reports all ranks' tokens over the slowest rank's time.  No data-path
collective exists: the only collective is the max of the timings.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    import torch.distributed as dist

    from sub_quadratic_attention_b200.ranks import job_throughput, max_over_ranks, rank_seed_offset
    from sub_quadratic_attention_b200.workloads import WORKLOADS, make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["tiny_fp32"]
        inp = make_inputs(w, seed_offset=rank_seed_offset(rank))
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        m = max_over_ranks(local_ms)
        value = job_throughput(w.B * w.L, world, 4, m)
        results[rank] = (m, value, float(inp["q"].sum()), float(inp["q"][0, 0, 0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_share_only_the_timing():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()   # no fork of a multi-threaded test process
    results = mgr.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 15.0                      # max over ranks
    expected = 1 * 256 * 2 * 4 / (15.0e-3)             # all ranks' tokens / slowest time
    assert abs(r0[1] - expected) < 1e-6 * expected and r0[1] == r1[1]
    assert r0[2] != r1[2]                               # each rank mixes its own batch


def test_single_process_reduces_to_local_values():
    from sub_quadratic_attention_b200.ranks import job_throughput, max_over_ranks

    assert max_over_ranks(3.5) == 3.5
    assert job_throughput(100, 1, 10, 1000.0) == 1000.0
    with pytest.raises(ValueError):
        job_throughput(100, 1, 0, 1.0)


def test_rank_inputs_are_deterministic():
    from sub_quadratic_attention_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS["tiny_fp32"]
    a = make_inputs(w, seed_offset=1)
    b = make_inputs(w, seed_offset=1)
    c = make_inputs(w, seed_offset=0)
    assert torch.equal(a["q"], b["q"]) and not torch.equal(a["q"], c["q"])
