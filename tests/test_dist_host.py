"""The multi-GPU bench's host-side plumbing on CPU: two gloo ranks, as the
launcher starts them (one process each, rendezvous on 127.0.0.1).  No GPU:
every rank does its own "work" and the job's time is the slowest rank's."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from chunked_hierarchical_sparse_b200 import dist_util


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    w, r, lr = dist_util.env_ranks()
    dist_util.init(w, "gloo", timeout_s=60)
    seed = dist_util.rank_seed(1003, r)
    dist_util.barrier(w)
    my_ms = 10.0 * (r + 1)  # rank 1 is the slowest
    job_ms = dist_util.max_over_ranks(my_ms, w)
    value = dist_util.job_throughput(65536, w, 3, job_ms)
    dist_util.finish(w)
    out.put((r, w, lr, seed, job_ms, value))


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in res] == [0, 1]
    assert all(w == world and lr == r for r, w, lr, *_ in res)
    # independent problems: distinct seeds, rank 0 keeps the base seed
    assert res[0][3] == 1003 and res[1][3] != res[0][3]
    # every rank sees the slowest rank's time, and the same whole-job throughput
    assert all(job == pytest.approx(20.0) for *_, job, _ in res)
    assert all(v == pytest.approx(2 * 65536 * 3 / 0.020) for *_, v in res)


def test_single_rank_needs_no_process_group():
    assert dist_util.max_over_ranks(7.5, 1) == 7.5
    assert dist_util.job_throughput(100, 1, 2, 1000.0) == pytest.approx(200.0)
    with pytest.raises(ValueError):
        dist_util.job_throughput(1, 1, 1, 0.0)
