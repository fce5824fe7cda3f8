"""The benchmark's multi-rank host logic, on CPU with two gloo ranks.

One process per GPU runs the same step on its own sequences (weak scaling, no data-path
collective); the job's time is the slowest rank's and its rate counts every rank's queries.
Here two CPU processes check that each rank draws its own sequences, that the time reduction
is a maximum seen identically by both ranks, and the whole-job rate."""
import datetime
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench

W = "csa_decode_128k_b32"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        lengths = bench.rank_lengths(W, rank)
        seen = [None] * world
        dist.all_gather_object(seen, lengths)
        ms = bench.max_over_ranks(10.0 + rank, dist, "cpu")
        e2e = bench.max_over_ranks(20.0 - rank, dist, "cpu")
        rate = bench.whole_job_rate(32, world, 200, ms)
        dist.barrier()
        out.put((rank, seen, ms, e2e, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    c = bench.WORKLOADS[W]
    for rank, seen, ms, e2e, rate in res:
        assert ms == 11.0 and e2e == 20.0            # the slowest rank, on every rank
        assert rate == 32 * 2 * 200 / 0.011
        assert seen == res[0][1]                     # both ranks see the same lists
        assert seen[0] != seen[1]                    # each rank its own sequences
        for lengths in seen:
            assert len(lengths) == c["B"]
            assert all(abs(t - c["T"]) <= c["jitter"] for t in lengths)
    assert bench.rank_lengths(W, 0) == res[0][1][0]  # deterministic per rank


def test_one_process_time_is_its_own():
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.whole_job_rate(8, 1, 10, 2.0) == 8 * 10 / 0.002
