"""lightning_indexer_topk_noalloc: the indexer + top-k for callers that cannot allocate
device memory (for example a plugin whose host framework owns the whole device pool, or a
loop where a cudaMalloc could stall the device).  Its scratch is a fixed device array
inside libcsa instead of a caller workspace.

Checked through the C ABI against lightning_indexer_topk on the same inputs:
 - two calls in a row with different shapes and no score buffer, so the score rows live in
   the library's array and the second call finds the first call's rows there: index sets
   must be identical;
 - with a score buffer the array is not used: scores and index sets identical;
 - two calls back to back on one stream (eagerly and inside a captured CUDA graph), where
   the second call's indexer overwrites the array while the first call's top-k may still
   read it: both index sets bit-exact against the oracle (integer inputs).
This file is collected last and also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import _orc
import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(wl, idx, max_n, st=None, sc=None):
    L.lightning_indexer_topk_noalloc(wl.qI, wl.qs, wl.w, wl.kI, wl.ks, wl.seq_len, wl.ent_off,
                                     wl.q_seq, wl.q_pos, idx, B=wl.B, H_I=wl.H_I, d_I=wl.d_I,
                                     m=wl.m, k=wl.k, max_n=max_n, scores_out=sc,
                                     ld_scores=0 if sc is None else sc.shape[1], dev_status=st)


def _reference(wl, scores=False):
    buf = pipeline.alloc(wl, DEV)
    sc = torch.full((wl.Q, buf.max_n), float("nan"), device=DEV) if scores else None
    pipeline.indexer_topk(wl, buf, scores_out=sc)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    return buf.idx, sc, buf.max_n


def _workloads():
    first = synth.make_workload("t", B=5, T=[40000, 9001, 131072, 777, 60000], D=128, H=16, m=4,
                                span=8, H_I=64, d_I=128, k=512, indexer="fp8", seed=91,
                                device=DEV)
    second = synth.make_workload("t", B=2, T=[4096, 2500], D=128, H=16, m=4, span=8, H_I=4,
                                 d_I=64, k=64, indexer="int", seed=92, device=DEV)
    return first, second


def test_noalloc_scratch_matches_workspace_entry_point_on_two_calls():
    for wl in _workloads():
        ref_idx, _, max_n = _reference(wl)
        idx = torch.full((wl.Q, wl.k), -7, dtype=torch.int32, device=DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        _noalloc(wl, idx, max_n, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert torch.equal(idx, ref_idx)


def test_noalloc_with_score_buffer_matches_workspace_entry_point():
    for wl in _workloads():
        ref_idx, ref_sc, max_n = _reference(wl, scores=True)
        idx = torch.full((wl.Q, wl.k), -7, dtype=torch.int32, device=DEV)
        sc = torch.full((wl.Q, max_n), float("nan"), device=DEV)
        _noalloc(wl, idx, max_n, sc=sc)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        n = ((wl.q_pos.to(torch.int64) + 1) // wl.m).tolist()
        for q, nq in enumerate(n):
            assert torch.equal(sc[q, :nq].view(torch.int32), ref_sc[q, :nq].view(torch.int32))


@pytest.mark.parametrize("graph", [False, True])
def test_noalloc_twice_back_to_back_bit_exact(graph):
    a = synth.make_workload("t", B=4, T=[160000, 150001, 90000, 140000], D=128, H=16, m=4,
                            span=8, H_I=64, d_I=128, k=512, keep_raw=64, seed=95, device=DEV)
    b = synth.make_workload("t", B=4, T=[150000, 160001, 140000, 70001], D=128, H=16, m=4,
                            span=8, H_I=64, d_I=128, k=512, keep_raw=64, seed=96, device=DEV)
    max_n = max(pipeline.max_visible(a), pipeline.max_visible(b))
    ia = torch.full((a.Q, a.k), -7, dtype=torch.int32, device=DEV)
    ib = torch.full((b.Q, b.k), -7, dtype=torch.int32, device=DEV)
    # one call outside capture first: it resolves the array's address for this device
    _noalloc(a, ia, max_n)
    _noalloc(b, ib, max_n)
    torch.cuda.synchronize()
    ia.fill_(-7)
    ib.fill_(-7)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            _noalloc(a, ia, max_n)
            _noalloc(b, ib, max_n)
        for _ in range(3):
            g.replay()
    else:
        for _ in range(3):
            _noalloc(a, ia, max_n)
            _noalloc(b, ib, max_n)
    torch.cuda.synchronize()
    ref_a, _ = _orc.indexer(a.to("cpu"))
    ref_b, _ = _orc.indexer(b.to("cpu"))
    assert np.array_equal(ia.cpu().numpy(), ref_a)
    assert np.array_equal(ib.cpu().numpy(), ref_b)


def test_noalloc_rejects_more_than_its_scratch():
    wl = synth.make_workload("t", B=1, T=[4096], D=128, H=16, m=4, span=8, H_I=4, d_I=64, k=64,
                             seed=93, device=DEV)
    idx = torch.zeros((wl.Q, wl.k), dtype=torch.int32, device=DEV)
    n0 = L.csa_launch_count()
    too_big = L.NOALLOC_SCRATCH_BYTES // 4 + 1            # visible entries of one query
    with pytest.raises(L.CSAError) as err:
        _noalloc(wl, idx, too_big)
    assert err.value.status == 4 and "scratch" in str(err.value)
    assert L.csa_launch_count() == n0
    # k is checked before the scratch size: an invalid k is reported as such
    with pytest.raises(L.CSAError) as err:
        L.lightning_indexer_topk_noalloc(wl.qI, wl.qs, wl.w, wl.kI, wl.ks, wl.seq_len,
                                         wl.ent_off, wl.q_seq, wl.q_pos, idx, B=wl.B,
                                         H_I=wl.H_I, d_I=wl.d_I, m=wl.m, k=0, max_n=too_big)
    assert err.value.status == 2 and "k = 0" in str(err.value)
    assert L.csa_launch_count() == n0
