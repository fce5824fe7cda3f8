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


# ---- context-parallel decode: the exchange of candidates and selected rows ---------------
def _cp_worker(rank, world, port, out):
    import types

    import torch

    from long_context_compressed_04_b200 import cp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # two sequences of 1000 and 37 entries, one decode query each (all entries visible)
        n_ent = torch.tensor([1000, 37])
        wl = types.SimpleNamespace(n_ent=n_ent, q_seq=torch.tensor([0, 1], dtype=torch.int32),
                                   q_pos=(n_ent * 4 - 1).to(torch.int32), m=4)
        bounds = [cp.slice_bounds(int(x), world, rank) for x in n_ent]
        off = torch.tensor([0, bounds[0][1] - bounds[0][0]], dtype=torch.int64)
        sl = cp.make_slice(wl, world, rank, off)
        # this rank's store: row i holds the global entry index of its slice's row i
        rows = []
        for b, (lo, hi) in enumerate(bounds):
            for e in range(lo, hi):
                rows.append([b, e % 256, e // 256, rank])
        store = torch.tensor(rows, dtype=torch.uint8)
        # candidates: the slice's entries divisible by 7, ascending, padded to k = 8 with -1
        k = 8
        cand = torch.full((2, k), -1, dtype=torch.int32)
        for b, (lo, hi) in enumerate(bounds):
            sel = [e for e in range(lo, hi) if e % 7 == 0][:k]
            cand[b, :len(sel)] = torch.tensor(sel, dtype=torch.int32)
        parts = cp.exchange(cand)
        merged_in_order = torch.cat(parts, dim=1)
        # the top-k: the 3 lowest candidates of every sequence, ascending (a stand-in for
        # the library's merge), -1 padded
        idx = torch.full((2, k), -1, dtype=torch.int32)
        for b in range(2):
            v = merged_in_order[b][merged_in_order[b] >= 0]
            idx[b, :3] = v[:3]
        packed = cp.pack_rows(idx, sl, wl.q_seq, store, 4)
        got = cp.unpack_rows(cp.exchange(packed), idx, [cp.make_slice(wl, world, r, off) for r in range(world)],
                             wl.q_seq)
        out.put((rank, merged_in_order.tolist(), idx.tolist(), got.tolist(),
                 sl.q_pos.tolist(), sl.q_live.tolist()))
    finally:
        dist.destroy_process_group()


def test_context_parallel_exchange_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, m0, idx0, got0, qp0, live0), (_, m1, idx1, got1, qp1, live1) = res
    # both ranks gather the same candidates, slices in rank order: ascending per sequence
    assert m0 == m1
    for b in range(2):
        v = [x for x in m0[b] if x >= 0]
        assert v == sorted(v) and len(set(v)) == len(v)
    assert idx0 == idx1 == [[0, 7, 14, -1, -1, -1, -1, -1], [0, 7, 14, -1, -1, -1, -1, -1]]
    # every selected row arrives from the rank whose slice holds it, at its position
    for got in (got0, got1):
        for b in range(2):
            for j, e in enumerate(idx0[b]):
                if e < 0:
                    assert got[b][j] == [0, 0, 0, 0]
                else:
                    lo1 = [500, 18][b]
                    assert got[b][j] == [b, e % 256, e // 256, 0 if e < lo1 else 1]
    # slices as sequences of their own: rank 0 sees entries 0..499 and 0..17, rank 1 the rest
    assert qp0 == [500 * 4 - 1, 18 * 4 - 1] and qp1 == [500 * 4 - 1, 19 * 4 - 1]
    assert live0 == live1 == [True, True]
