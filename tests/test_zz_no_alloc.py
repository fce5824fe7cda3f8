"""lightning_indexer_topk_noalloc: the indexer + top-k for callers that cannot allocate
device memory (for example a plugin whose host framework owns the whole device pool, or a
loop where a cudaMalloc could stall the device).  Its scratch is a fixed device array
inside libcsa instead of a caller workspace.

Checked through the C ABI against lightning_indexer_topk on the same inputs, on two calls
in a row with different shapes (the array keeps the first call's contents when the second
runs): index sets and scores must be identical, as both run the same kernels.  This file
is collected last and also passes alone in a fresh process."""
import pytest
import torch

import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _both(wl):
    buf = pipeline.alloc(wl, DEV)
    ref_sc = torch.full((wl.Q, buf.max_n), float("nan"), device=DEV)
    pipeline.indexer_topk(wl, buf, scores_out=ref_sc)
    idx = torch.full((wl.Q, wl.k), -7, dtype=torch.int32, device=DEV)
    sc = torch.full((wl.Q, buf.max_n), float("nan"), device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.lightning_indexer_topk_noalloc(wl.qI, wl.qs, wl.w, wl.kI, wl.ks, wl.seq_len, wl.ent_off,
                                     wl.q_seq, wl.q_pos, idx, B=wl.B, H_I=wl.H_I, d_I=wl.d_I,
                                     m=wl.m, k=wl.k, max_n=buf.max_n, scores_out=sc,
                                     ld_scores=buf.max_n, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(buf.dev_status.item()) == 0
    return buf.idx, ref_sc, idx, sc


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    first = synth.make_workload("t", B=5, T=[40000, 9001, 131072, 777, 60000], D=128, H=16, m=4,
                                span=8, H_I=64, d_I=128, k=512, indexer="fp8", seed=91,
                                device=DEV)
    second = synth.make_workload("t", B=2, T=[4096, 2500], D=128, H=16, m=4, span=8, H_I=4,
                                 d_I=64, k=64, indexer="int", seed=92, device=DEV)
    for wl in (first, second):
        ref_idx, ref_sc, idx, sc = _both(wl)
        assert torch.equal(idx, ref_idx)
        n = ((wl.q_pos.to(torch.int64) + 1) // wl.m).tolist()
        for q, nq in enumerate(n):
            assert torch.equal(sc[q, :nq].view(torch.int32), ref_sc[q, :nq].view(torch.int32))


def test_noalloc_rejects_more_than_its_scratch():
    wl = synth.make_workload("t", B=1, T=[4096], D=128, H=16, m=4, span=8, H_I=4, d_I=64, k=64,
                             seed=93, device=DEV)
    idx = torch.zeros((wl.Q, wl.k), dtype=torch.int32, device=DEV)
    n0 = L.csa_launch_count()
    too_big = L.NOALLOC_SCRATCH_BYTES // 4 + 1            # visible entries of one query
    with pytest.raises(L.CSAError) as err:
        L.lightning_indexer_topk_noalloc(wl.qI, wl.qs, wl.w, wl.kI, wl.ks, wl.seq_len,
                                         wl.ent_off, wl.q_seq, wl.q_pos, idx, B=wl.B, H_I=wl.H_I,
                                         d_I=wl.d_I, m=wl.m, k=wl.k, max_n=too_big)
    assert err.value.status == 4 and "scratch" in str(err.value)
    assert L.csa_launch_count() == n0
