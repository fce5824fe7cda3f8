"""Context-parallel decode, its ranks run in turn on one GPU.

A batch's compressed entries are split into W contiguous slices; each slice's top-k is
selected by the library as on its own rank, the candidates are merged by csa_topk_merge,
the selected rows are collected from the slices that hold them, and the attention runs on
those rows.  The index sets and the outputs must be bitwise equal to one GPU running the
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
    return (torch.cat(kI).contiguous(), torch.cat(ks).contiguous(), torch.cat(ents).contiguous(),
            torch.tensor(off, dtype=torch.int64))


def _cp_step(wl, rows, world):
    parts_idx, parts_sc, slices, stores = [], [], [], []
    for r in range(world):
        kI, ks, ents, off = _rank_store(wl, world, r, rows)
        sl = cp.make_slice(wl, world, r, off)
        ci, cs = cp.local_candidates(wl, sl, kI, ks)
        parts_idx.append(ci)
        parts_sc.append(cs)
        slices.append(sl)
        stores.append(ents)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    n0 = L.csa_launch_count()
    idx = cp.merge_candidates(parts_idx, parts_sc, wl.k, dev_status=st)
    assert L.csa_launch_count() - n0 == 1
    rb = cp.row_bytes_of(wl)
    packed = [cp.pack_rows(idx, sl, wl.q_seq, ents, rb) for sl, ents in zip(slices, stores)]
    sel_rows = cp.unpack_rows(packed, idx, slices, wl.q_seq)
    out = torch.zeros_like(wl.q)
    cp.attend_selected(wl, sel_rows, idx, out, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return idx, out


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
