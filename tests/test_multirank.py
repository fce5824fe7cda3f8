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
        # three sequences of 1000, 37 and 1 entries, one decode query each (all entries
        # visible); rank 0's slice of the third is empty
        n_ent = torch.tensor([1000, 37, 1])
        Q, k = 3, 8
        wl = types.SimpleNamespace(n_ent=n_ent, q_seq=torch.tensor([0, 1, 2], dtype=torch.int32),
                                   q_pos=(n_ent * 4 - 1).to(torch.int32), m=4)
        bounds = [cp.slice_bounds(int(x), world, rank) for x in n_ent]
        sl = cp.make_slice(wl, world, rank, torch.zeros(3, dtype=torch.int64))
        # this rank's candidates, as csa_cp_candidates lays them out: the slice's entries
        # divisible by 7, ascending, -1 padded; their scores (bits in the second half)
        cand = torch.full((2, Q, k), -1, dtype=torch.int32)
        for b, (lo, hi) in enumerate(bounds):
            sel = [e for e in range(lo, hi) if e % 7 == 0][:k]
            cand[0, b, :len(sel)] = torch.tensor(sel, dtype=torch.int32)
            cand[1, b] = torch.full((k,), float(rank + 1)).view(torch.int32)
        buf = types.SimpleNamespace(cand=cand, gathered=torch.zeros((world, 2, Q, k),
                                                                    dtype=torch.int32))
        cp.exchange_candidates(buf)
        # the merged selection (a stand-in for csa_topk_merge): the 3 lowest candidates
        idx = torch.full((Q, k), -1, dtype=torch.int32)
        for b in range(Q):
            v = buf.gathered[:, 0, b].flatten()
            v = v[v >= 0]
            idx[b, :min(3, v.numel())] = v[:3]
        # the packed rows, as csa_cp_pack_rows lays them out: the row if this rank's slice
        # holds the entry (here [b, e % 256, e // 256, rank + 1]), zeros otherwise
        buf.packed = torch.zeros((Q, k, 4), dtype=torch.uint8)
        for b, (lo, hi) in enumerate(bounds):
            for j in range(k):
                e = int(idx[b, j])
                if e >= 0 and lo <= e < hi:
                    buf.packed[b, j] = torch.tensor([b, e % 256, e // 256, rank + 1],
                                                    dtype=torch.uint8)
        cp.exchange_rows(buf)
        out.put((rank, buf.gathered.tolist(), idx.tolist(), buf.packed.tolist(),
                 sl.q_pos.tolist(), sl.seq_len.tolist(), sl.max_n))
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
    (_, g0, idx0, got0, qp0, sq0, mx0), (_, g1, idx1, got1, qp1, sq1, mx1) = res
    # both ranks gather the same candidates, slices in rank order: ascending per sequence,
    # each rank's scores with it
    assert g0 == g1
    for b in range(3):
        v = [x for r in range(2) for x in g0[r][0][b] if x >= 0]
        assert v == sorted(v) and len(set(v)) == len(v)
        for r in range(2):
            assert all(x == torch_float_bits(float(r + 1)) for x in g0[r][1][b])
    assert idx0 == idx1 == [[0, 7, 14, -1, -1, -1, -1, -1], [0, 7, 14, -1, -1, -1, -1, -1],
                            [0, -1, -1, -1, -1, -1, -1, -1]]
    # the integer sum is the gather: every selected row from the rank whose slice holds it
    assert got0 == got1
    lo1 = [500, 18, 0]
    for b in range(3):
        for j, e in enumerate(idx0[b]):
            if e < 0:
                assert got0[b][j] == [0, 0, 0, 0]
            else:
                assert got0[b][j] == [b, e % 256, e // 256, 1 if e < lo1[b] else 2]
    # slices as sequences of their own: rank 0 sees entries 0..499, 0..17 and none of the
    # third; rank 1 the rest; m - 1 extra tokens make position 0 valid for an empty slice
    assert qp0 == [500 * 4 - 1, 18 * 4 - 1, 0] and qp1 == [500 * 4 - 1, 19 * 4 - 1, 1 * 4 - 1]
    assert sq0 == [500 * 4 + 3, 18 * 4 + 3, 3] and sq1 == [500 * 4 + 3, 19 * 4 + 3, 4 + 3]
    assert mx0 == mx1 == 500


def torch_float_bits(x: float) -> int:
    import struct
    return struct.unpack("<i", struct.pack("<f", x))[0]
