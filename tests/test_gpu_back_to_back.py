"""Calls in a row on one stream that share a buffer.

Every libcsa kernel is launched so that it may start while the kernel before it finishes
(programmatic dependent launch).  A kernel that stores into a buffer the previous kernel
still reads must wait for it first.  These tests issue two calls back to back on one
stream with different inputs and ONE shared workspace, eagerly and inside a captured CUDA
graph, and check each call's result against the oracle (indexer + top-k: integer inputs,
so bit for bit) or against the same call run alone (dense attention: bitwise)."""
import numpy as np
import pytest
import torch

import _orc
from long_context_compressed_04_b200 import (csa_indexer_workspace_size, dense_hca_attn,
                                             dense_hca_workspace_size, lightning_indexer_topk,
                                             pipeline, synth)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _indexer_pair():
    # same shape (so one workspace serves both), different sequences and heads; rows long
    # enough that the first top-k is still reading its score rows when the second indexer
    # starts storing
    a = synth.make_workload("t", B=4, T=[160000, 150001, 90000, 140000], D=128, H=16, m=4,
                            span=8, H_I=64, d_I=128, k=512, keep_raw=64, seed=301, device=DEV)
    b = synth.make_workload("t", B=4, T=[150000, 160001, 140000, 70001], D=128, H=16, m=4,
                            span=8, H_I=64, d_I=128, k=512, keep_raw=64, seed=302, device=DEV)
    return a, b


def _call(wl, idx, ws, max_n):
    lightning_indexer_topk(wl.qI, wl.qs, wl.w, wl.kI, wl.ks, wl.seq_len, wl.ent_off, wl.q_seq,
                           wl.q_pos, idx, ws, B=wl.B, H_I=wl.H_I, d_I=wl.d_I, m=wl.m, k=wl.k,
                           max_n=max_n)


@pytest.mark.parametrize("graph", [False, True])
def test_indexer_topk_twice_on_one_workspace_bit_exact(graph):
    a, b = _indexer_pair()
    max_n = max(pipeline.max_visible(a), pipeline.max_visible(b))
    ws = torch.zeros(csa_indexer_workspace_size(a.Q, max_n, a.k), dtype=torch.uint8,
                     device=DEV)
    ia = torch.full((a.Q, a.k), -7, dtype=torch.int32, device=DEV)
    ib = torch.full((b.Q, b.k), -7, dtype=torch.int32, device=DEV)
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):          # one warm-up outside capture
            _call(a, ia, ws, max_n)
            _call(b, ib, ws, max_n)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        ia.fill_(-7)
        ib.fill_(-7)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            _call(a, ia, ws, max_n)
            _call(b, ib, ws, max_n)
        for _ in range(3):
            g.replay()
    else:
        for _ in range(3):
            _call(a, ia, ws, max_n)
            _call(b, ib, ws, max_n)
    torch.cuda.synchronize()
    ref_a, _ = _orc.indexer(a.to("cpu"))
    ref_b, _ = _orc.indexer(b.to("cpu"))
    assert np.array_equal(ia.cpu().numpy(), ref_a)
    assert np.array_equal(ib.cpu().numpy(), ref_b)


def _dense(wl, buf, out, ws, max_n):
    dense_hca_attn(wl.q, buf.entries, wl.seq_len, wl.ent_off, wl.kv, wl.kv_off, wl.kv_pos0,
                   wl.q_seq, wl.q_pos, wl.sink, out, ws, fmt=wl.fmt, B=wl.B, H=wl.H, D=wl.D,
                   W=wl.W, m=wl.m, max_n=max_n, softmax_scale=wl.scale, rope_theta=wl.theta,
                   eps=wl.eps, dev_status=buf.dev_status)


@pytest.mark.parametrize("graph", [False, True])
def test_dense_attention_twice_on_one_workspace_bitwise(graph):
    # the chunk partials of the workspace are read by the combine kernel of the first call
    # while the second call's attention kernel stores its own
    a = synth.make_workload("t", B=4, T=[128 * 3000 + 5, 128 * 900, 128 * 2999, 700], D=128,
                            H=64, m=128, span=128, keep_raw=256, seed=311, device=DEV)
    b = synth.make_workload("t", B=4, T=[128 * 2000, 128 * 3000 + 100, 128 * 40, 128 * 2500],
                            D=128, H=64, m=128, span=128, keep_raw=256, seed=312, device=DEV)
    bufs = []
    for wl in (a, b):
        buf = pipeline.alloc(wl, DEV)
        g = torch.Generator(device=DEV).manual_seed(wl.B * 7 + wl.ent_rows)
        buf.entries.copy_(synth.random_entries(buf.entries.shape[0], 0, 128, g, DEV))
        bufs.append(buf)
    max_n = max(pipeline.max_visible(a), pipeline.max_visible(b))
    ws = torch.zeros(dense_hca_workspace_size(a.Q, 64, 128, max_n), dtype=torch.uint8,
                     device=DEV)
    alone = []
    for wl, buf in zip((a, b), bufs):
        own = torch.zeros(dense_hca_workspace_size(wl.Q, 64, 128, max_n), dtype=torch.uint8,
                          device=DEV)
        o = torch.zeros_like(buf.out)
        _dense(wl, buf, o, own, max_n)
        torch.cuda.synchronize()
        alone.append(o)
    oa, ob = torch.zeros_like(bufs[0].out), torch.zeros_like(bufs[1].out)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            _dense(a, bufs[0], oa, ws, max_n)
            _dense(b, bufs[1], ob, ws, max_n)
        for _ in range(3):
            g.replay()
    else:
        for _ in range(3):
            _dense(a, bufs[0], oa, ws, max_n)
            _dense(b, bufs[1], ob, ws, max_n)
    torch.cuda.synchronize()
    assert int(bufs[0].dev_status.item()) == 0 and int(bufs[1].dev_status.item()) == 0
    assert torch.equal(oa.view(torch.int16), alone[0].view(torch.int16))
    assert torch.equal(ob.view(torch.int16), alone[1].view(torch.int16))
