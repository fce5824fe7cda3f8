"""Context-parallel decode, its ranks run in turn on one GPU.

A batch's compressed entries are split into W contiguous slices; each slice's top-k is
selected by the library as on its own rank and turned into candidates, the candidates are
merged by csa_topk_merge, the selected rows are packed by the ranks that hold them and
summed, and the attention runs on those rows.  The index sets and the outputs must be bitwise equal to one GPU running the
whole step (integer-valued indexer inputs; the oracle pins the single-GPU path elsewhere).
No rank waits on another here: the slices are computed one after the other."""
import pytest
import torch

import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import cp, pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rank_store(wl, world, rank, rows):
    """The rank's key store and entry store: the rows of its slices, sequence after
    sequence, and where each sequence's slice starts in them."""
    ent_off = wl.ent_off.cpu()
    kI, ks, ents, off = [], [], [], []
    base = 0
    for b in range(wl.B):
        lo, hi = cp.slice_bounds(int(wl.n_ent[b]), world, rank)
        r0 = int(ent_off[b])
        kI.append(wl.kI[r0 + lo:r0 + hi])
        ks.append(wl.ks[r0 + lo:r0 + hi])
        ents.append(rows[r0 + lo:r0 + hi])
        off.append(base)
        base += hi - lo
    ent = torch.cat(ents).contiguous()
    if ent.shape[0] == 0:
        ent = torch.zeros((1, rows.shape[1]), dtype=torch.uint8, device=DEV)
    return (torch.cat(kI).contiguous(), torch.cat(ks).contiguous(), ent,
            torch.tensor(off, dtype=torch.int64))


def _ranks(wl, rows, world):
    ranks = []
    for r in range(world):
        kI, ks, ents, off = _rank_store(wl, world, r, rows)
        sl = cp.make_slice(wl, world, r, off)
        ranks.append((sl, kI, ks, ents, cp.alloc(wl, sl, world, DEV)))
    return ranks


def _cp_step(wl, rows, world):
    """One step with the ranks in turn; the collectives are stand-ins (stack and sum)."""
    ranks = _ranks(wl, rows, world)
    for sl, kI, ks, _e, buf in ranks:
        cp.select_local(wl, sl, kI, ks, buf)
    cands = torch.stack([buf.cand for *_x, buf in ranks])
    n0 = L.csa_launch_count()
    for sl, _k, _s, ents, buf in ranks:
        cp.exchange_candidates(buf, all_gather=lambda out, inp: out.copy_(cands))
        cp.merge(wl, buf)
        cp.pack(wl, sl, ents, buf)
    assert L.csa_launch_count() - n0 == 2 * world
    total = torch.stack([buf.packed.view(torch.int32) for *_x, buf in ranks]).sum(0,
                                                                                dtype=torch.int32)
    for *_x, buf in ranks:
        cp.exchange_rows(buf, all_reduce=lambda t: t.copy_(total))
        cp.attend(wl, buf)
    torch.cuda.synchronize()
    for *_x, buf in ranks:
        assert int(buf.dev_status.item()) == 0
        # every rank ends with the same selection and output
        assert torch.equal(buf.idx, ranks[0][4].idx)
        assert torch.equal(buf.out.view(torch.int16), ranks[0][4].out.view(torch.int16))
    return ranks[0][4].idx, ranks[0][4].out


def _one_gpu(wl, rows):
    buf = pipeline.alloc(wl, DEV)
    buf.entries.copy_(rows)
    pipeline.indexer_topk(wl, buf)
    pipeline.attend(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    return buf.idx, buf.out


@pytest.mark.parametrize("D,H,fmt,k,T,world", [
    (128, 64, 0, 512, [300001, 90000, 5000], 2),
    (128, 64, 0, 512, [300001, 90000, 5000], 3),
    (576, 128, 1, 1024, [1 << 20, 400003], 8),
    (576, 128, 1, 1024, [70000], 4),
    # a sequence of 5 entries over 8 ranks: three slices are empty
    (128, 64, 0, 512, [300001, 23], 8),
])
def test_context_parallel_step_matches_one_gpu_bitwise(D, H, fmt, k, T, world):
    wl = synth.make_workload("t", B=len(T), T=T, D=D, H=H, m=4, span=8, fmt=fmt, H_I=64,
                             d_I=128, k=k, keep_raw=256, seed=61, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(62)
    rows = synth.random_entries(wl.ent_rows, fmt, D, g, DEV)
    idx1, out1 = _one_gpu(wl, rows)
    idx2, out2 = _cp_step(wl, rows, world)
    assert torch.equal(idx1, idx2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_merge_ties_across_slices():
    # every key row the same: all scores tie, so the top-k are the k lowest entries, which
    # lie in the first slices; the merge must keep the lower-indexed ties
    wl = synth.make_workload("t", B=1, T=[200000], D=128, H=64, m=4, span=8, H_I=64, d_I=128,
                             k=512, keep_raw=256, seed=63, device=DEV)
    wl.kI.copy_(wl.kI[:1].expand_as(wl.kI))
    g = torch.Generator(device=DEV).manual_seed(64)
    rows = synth.random_entries(wl.ent_rows, 0, 128, g, DEV)
    idx1, out1 = _one_gpu(wl, rows)
    idx2, out2 = _cp_step(wl, rows, 4)
    assert idx1[0].tolist() == list(range(512))
    assert torch.equal(idx1, idx2)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_candidates_translate_and_flag_out_of_range():
    Q, k, ld = 3, 8, 50
    g = torch.Generator().manual_seed(65)
    sel = torch.randint(0, ld, (Q, k), generator=g, dtype=torch.int32)
    sel[0, 5:] = -1
    sel[2, 3] = ld          # outside the score rows: flagged, written as -1
    scores = torch.randn((Q, ld), generator=g)
    q_seq = torch.tensor([1, 0, 1], dtype=torch.int32)
    lo = torch.tensor([1000, 7], dtype=torch.int64)
    ci = torch.zeros((Q, k), dtype=torch.int32, device=DEV)
    cs = torch.zeros((Q, k), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.csa_cp_candidates(sel.to(DEV), scores.to(DEV), q_seq.to(DEV), lo.to(DEV), ci, cs, B=2,
                        dev_status=st)
    torch.cuda.synchronize()
    ci, cs = ci.cpu(), cs.cpu()
    for q in range(Q):
        for j in range(k):
            i = int(sel[q, j])
            if i < 0 or i >= ld:
                assert int(ci[q, j]) == -1 and float(cs[q, j]) == 0.0
            else:
                assert int(ci[q, j]) == i + int(lo[q_seq[q]])
                assert cs[q, j].view(torch.int32) == scores[q, i].view(torch.int32)
    assert int(st.item()) == 1   # CSA_DEV_OOB


def test_pack_rows_places_owned_rows_and_zeros():
    Q, k, rb = 2, 16, 272
    q_seq = torch.tensor([0, 1], dtype=torch.int32)
    lo = torch.tensor([100, 0], dtype=torch.int64)
    n = torch.tensor([40, 10], dtype=torch.int64)
    off = torch.tensor([10, 0], dtype=torch.int64)
    store = torch.randint(1, 256, (60, rb), dtype=torch.uint8)
    idx = torch.full((Q, k), -1, dtype=torch.int32)
    idx[0, :12] = torch.tensor([3, 99, 100, 101, 120, 139, 140, 200, 500, 600, 700, 800])
    idx[1, :4] = torch.tensor([0, 5, 9, 10])
    out = torch.full((Q, k, rb), 7, dtype=torch.uint8, device=DEV)
    li = torch.zeros((Q, k), dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.csa_cp_pack_rows(idx.to(DEV), q_seq.to(DEV), lo.to(DEV), n.to(DEV), off.to(DEV),
                       store.to(DEV), out, li, B=2, dev_status=st)
    torch.cuda.synchronize()
    out, li = out.cpu(), li.cpu()
    for q in range(Q):
        b = int(q_seq[q])
        for j in range(k):
            i = int(idx[q, j])
            assert int(li[q, j]) == (j if i >= 0 else -1)
            if i >= 0 and int(lo[b]) <= i < int(lo[b] + n[b]):
                assert torch.equal(out[q, j], store[int(off[b]) + i - int(lo[b])])
            else:
                assert int(out[q, j].abs().sum()) == 0
    assert int(st.item()) == 0
