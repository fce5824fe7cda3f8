"""GPU parity of lightning_indexer_topk against the oracle.

Integer-valued e4m3 inputs make every dot product exact, so scores and index sets must be
bit-identical (the fp32 head accumulation order is part of the definition).  With real
FP8 inputs the dot products round differently, so selections may differ only among
entries whose oracle score lies within the rounding bound of the k-th score."""
import numpy as np
import pytest
import torch

import _orc
from long_context_compressed_04_b200 import CSA_DEV_CAPACITY, pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(wl, scores=True):
    buf = pipeline.alloc(wl, DEV)
    sc = None
    if scores:
        sc = torch.full((wl.Q, max(buf.max_n, 1)), float("nan"), device=DEV)
    pipeline.indexer_topk(wl, buf, scores_out=sc)
    torch.cuda.synchronize()
    return buf, sc


def _exact(wl):
    buf, sc = _run(wl)
    assert int(buf.dev_status.item()) == 0
    idx_o, s_o = _orc.indexer(wl.to("cpu"))
    s_g = sc.cpu().numpy()
    n = (_orc.i64(wl.q_pos) + 1) // wl.m
    for q in range(wl.Q):
        assert np.array_equal(s_g[q, :n[q]].view(np.uint32), s_o[q, :n[q]].view(np.uint32)), q
    assert np.array_equal(buf.idx.cpu().numpy(), idx_o)
    return buf.idx.cpu().numpy()


def test_decode_4k_shape_bit_exact():
    # CSA decode, 1 sequence of 4096 tokens: 1024 entries, 4 indexer heads x 64, top-64
    _exact(synth.csa_decode_4k(device=DEV))


@pytest.mark.parametrize("HI,dI,k", [(64, 128, 512), (4, 64, 64), (16, 128, 100), (1, 128, 64),
                                     (20, 64, 100), (40, 128, 256), (64, 64, 512)])
def test_ragged_batch_bit_exact(HI, dI, k):
    # visible counts 1500, 4000, 300 (< k for some shapes: padded with -1), 7.  Head counts
    # other than 16, 32 and 64 run on the next MMA width with zero heads added.
    wl = synth.make_workload("t", B=4, T=[6003, 16000, 1201, 29], D=128, H=16, m=4, span=8,
                             H_I=HI, d_I=dI, k=k, seed=21, device=DEV)
    idx = _exact(wl)
    assert np.all(idx[3, 7:] == -1) and idx[3, :7].tolist() == list(range(7))


def test_long_sequences_many_work_items_bit_exact():
    # 130K + 25K + 750 entries: many 1024-entry work items per query on the tensor-core path
    wl = synth.make_workload("t", B=3, T=[520003, 100000, 3001], D=128, H=16, m=4, span=8,
                             H_I=64, d_I=128, k=1024, seed=26, device=DEV)
    _exact(wl)


def test_ties_break_toward_lower_index():
    wl = synth.make_workload("t", B=2, T=[8192, 5000], D=128, H=16, m=4, span=8, H_I=16,
                             d_I=128, k=256, seed=22, device=DEV)
    # only 5 distinct key rows -> massive ties at the k-th score
    g = torch.Generator(device=DEV).manual_seed(0)
    rows = wl.kI[torch.randint(0, 5, (wl.kI.shape[0],), device=DEV, generator=g)]
    wl.kI.copy_(rows)
    wl.w.fill_(1.0)
    _exact(wl)


def test_long_rows_cluster_of_seven_bit_exact():
    # 210K and 70K visible entries: rows past one CTA's shared memory take the per-query
    # cluster path, here 7 ranks (a cluster size that is not a power of two)
    wl = synth.make_workload("t", B=2, T=[840003, 280001], D=128, H=16, m=4, span=8, H_I=16,
                             d_I=128, k=1024, keep_raw=64, seed=28, device=DEV)
    _exact(wl)


def test_long_rows_massive_ties_bit_exact():
    # only 3 distinct key rows over 150K entries: no bin ever gets small, so every bit is
    # resolved across the cluster and the ties split between ranks by entry order
    wl = synth.make_workload("t", B=1, T=[600001], D=128, H=16, m=4, span=8, H_I=16,
                             d_I=128, k=1024, keep_raw=64, seed=29, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(1)
    rows = wl.kI[torch.randint(0, 3, (wl.kI.shape[0],), device=DEV, generator=g)]
    wl.kI.copy_(rows)
    wl.w.fill_(1.0)
    _exact(wl)


def _scores_from_scales(wl, ks):
    """Every key row and every query head the same positive vector, all weights 1: each
    entry's score is its key scale times one positive constant per query, so the scales
    set the ranking exactly."""
    row = wl.kI[0].clone()
    row[row == 0] = 0x38   # e4m3 1.0 wherever the row is 0, so q.k = |k|^2 > 0
    wl.kI[:] = row
    wl.qI[:] = row
    wl.w.fill_(1.0)
    wl.qs.fill_(1.0)
    wl.ks.copy_(torch.as_tensor(ks, dtype=torch.float32, device=DEV))


def test_sampled_bound_too_high_falls_back():
    # 40000 entries, top-512: the strided sample the selection starts from holds the 1024
    # largest scores of the row (distinct), so fewer than k keys reach the bound taken
    # from it and the general radix passes must run; the result stays the unique top-k
    wl = synth.make_workload("t", B=1, T=[160000], D=128, H=16, m=4, span=8, H_I=16,
                             d_I=128, k=512, seed=24, device=DEV)
    n = 40000
    ks = np.random.default_rng(7).uniform(1.0, 2.0, wl.kI.shape[0]).astype(np.float32)
    sample = (np.arange(1024, dtype=np.int64) * n) // 1024
    ks[sample] = 100.0 + np.arange(1024, dtype=np.float32)
    _scores_from_scales(wl, ks)
    idx = _exact(wl)
    # the top 512 are the upper half of the sample positions
    assert np.array_equal(idx[0], np.sort(sample[512:]))


def test_sampled_bound_too_many_candidates_falls_back():
    # all but one score equal: every key reaches the bound, far more than the candidate list
    # holds, so the general passes run; ties go to the lowest entries
    wl = synth.make_workload("t", B=1, T=[160000], D=128, H=16, m=4, span=8, H_I=16,
                             d_I=128, k=512, seed=25, device=DEV)
    ks = np.full(wl.kI.shape[0], 1.5, np.float32)
    ks[777] = 0.5
    _scores_from_scales(wl, ks)
    idx = _exact(wl)
    assert np.array_equal(idx[0], np.arange(512))


@pytest.mark.parametrize("hot", [2048, 8192])
def test_group_bound_with_clustered_top_scores(hot):
    # 60000 entries, top-1024: the `hot` first entries score highest, so the k largest group
    # maxima come from few groups.  hot = 2048: about 3000 entries reach the bound (the
    # group path); hot = 8192: more than its 4096-entry list, so the full row is used
    wl = synth.make_workload("t", B=1, T=[240000], D=128, H=16, m=4, span=8, H_I=16,
                             d_I=128, k=1024, seed=27, device=DEV)
    ks = np.random.default_rng(8).uniform(1.0, 2.0, wl.kI.shape[0]).astype(np.float32)
    ks[:hot] = 10.0 + np.random.default_rng(9).uniform(0.0, 1.0, hot).astype(np.float32)
    _scores_from_scales(wl, ks)
    idx = _exact(wl)
    assert np.all(idx[0] < hot)


def test_group_path_across_a_ragged_batch_bit_exact():
    # long and short rows in one batch: rows of at least 32k entries select from the group
    # maxima, the shorter ones from their full rows
    wl = synth.make_workload("t", B=5, T=[400003, 8000, 250001, 160000, 1001], D=128, H=16,
                             m=4, span=8, H_I=64, d_I=128, k=512, keep_raw=64, seed=30,
                             device=DEV)
    _exact(wl)


def _abs_bound(wl, q):
    """fp32 rounding bound of one query's scores: the dot products accumulate 128 e4m3
    products in fp32 (error <= 2^-17 of the sum of |products| each, doubled for margin)
    and the head chain adds <= 2^-18 of |s| per step."""
    cw = wl.to("cpu")
    qv = torch.from_numpy(_orc.u8(cw.qI[q])).view(torch.float8_e4m3fn).double().abs()
    kv = torch.from_numpy(_orc.u8(cw.kI)).view(torch.float8_e4m3fn).double().abs()
    b = int(cw.q_seq[q])
    e0, n = int(cw.ent_off[b]), (int(cw.q_pos[q]) + 1) // wl.m
    ws = (cw.w[q].double() * cw.qs[q].double())
    mag = (kv[e0:e0 + n] @ qv.T) @ ws * cw.ks[e0:e0 + n].double()
    return (2.0 ** -16 * mag).numpy()


def test_real_fp8_inputs_select_within_rounding():
    wl = synth.make_workload("t", B=3, T=[40000, 9000, 20001], D=128, H=16, m=4, span=8,
                             H_I=64, d_I=128, k=512, indexer="fp8", seed=23, device=DEV)
    buf, sc = _run(wl)
    idx_o, s_o = _orc.indexer(wl.to("cpu"))
    idx_g = buf.idx.cpu().numpy()
    s_g = sc.cpu().numpy()
    n = (_orc.i64(wl.q_pos) + 1) // wl.m
    for q in range(wl.Q):
        bound = _abs_bound(wl, q) + 2.0 ** -18 * 64 * np.abs(s_o[q, :n[q]])
        assert np.all(np.abs(s_g[q, :n[q]] - s_o[q, :n[q]]) <= bound)
        order = np.argsort(-s_o[q, :n[q]], kind="stable")
        kth = s_o[q, order[wl.k - 1]]
        diff = set(idx_g[q].tolist()) ^ set(idx_o[q].tolist())
        for i in diff:
            assert abs(s_o[q, i] - kth) <= 2 * (bound[i] + bound[order[wl.k - 1]]), (q, i)


def test_batch_invariance_bitwise():
    base = synth.make_workload("t", B=7, T=[3001, 60000, 777, 12345, 4096, 50, 99999], D=128,
                               H=16, m=4, span=8, H_I=64, d_I=128, k=512, indexer="fp8",
                               seed=24, device=DEV)
    parts = synth.split(base)
    target = 3
    ref_buf, ref_sc = _run(synth.merge([parts[target]]))
    for order in ([1, 3, 0], [6, 5, 4, 3, 2, 1, 0], [3] + [i for i in range(7) if i != 3]):
        wl = synth.merge([parts[i] for i in order])
        buf, sc = _run(wl)
        slot = order.index(target)
        n = int(parts[target].n_ent[0])
        assert torch.equal(buf.idx[slot], ref_buf.idx[0])
        assert torch.equal(sc[slot, :n].view(torch.int32), ref_sc[0, :n].view(torch.int32))


def test_capacity_flag_when_max_n_too_small():
    wl = synth.make_workload("t", B=1, T=[4000], D=128, H=16, m=4, span=8, H_I=4, d_I=64, k=8,
                             seed=25, device=DEV)
    buf = pipeline.alloc(wl, DEV)
    buf.max_n = 500
    pipeline.indexer_topk(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) & CSA_DEV_CAPACITY
