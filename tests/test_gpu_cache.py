"""The hybrid cache ("DeepSeek-V4 深度分析报告" 3.5): a state-cache ring of raw tokens and a
classical cache in blocks of 128 tokens (32 CSA entries) behind a block table, driven one
decode token at a time (append, compress the entries completed, select, attend).

Each step is compared bit for bit with the contiguous layout -- every raw token stored in a
linear array and every sequence's entries in one contiguous run -- on the same inputs: the
index sets, the attention outputs and, at the end, every compressed entry.  The contiguous
path is the one the oracle pins elsewhere, and only the addressing differs.  The physical
blocks are handed out in shuffled order, sequences cross block boundaries during the run,
and the window reads across the ring's wrap."""
import numpy as np
import pytest
import torch

import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import cache, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _contig_offsets(n):
    off = torch.zeros(len(n), dtype=torch.int64)
    off[1:] = torch.cumsum(torch.tensor(n[:-1], dtype=torch.int64), 0)
    return off


@pytest.mark.parametrize("D,H,fmt,H_I,d_I", [(576, 128, 1, 64, 128), (128, 64, 0, 64, 128),
                                             (128, 16, 0, 4, 64)])
def test_paged_ring_decode_matches_contiguous_bitwise(D, H, fmt, H_I, d_I):
    g = torch.Generator(device=DEV).manual_seed(81)
    B, S, k, W, ring = 4, 70, 64, 128, 128
    T0 = [3001, 777, 4099, 130]
    Tmax = [t + S for t in T0]
    nEmax = [t // 4 for t in Tmax]
    # all raw tokens and all indexer keys the run will use, in linear layouts
    kv_off = _contig_offsets(Tmax)
    kv_all = (torch.randn((sum(Tmax), D), generator=g, device=DEV)).to(torch.bfloat16)
    gate_all = (torch.randn((sum(Tmax), D), generator=g, device=DEV)).to(torch.bfloat16)
    bias = torch.randn((8, D), generator=g, device=DEV) * 0.1
    ent_off = _contig_offsets(nEmax)
    kI_all = synth.fp8_integer((sum(nEmax), d_I), g, DEV)
    ks_all = torch.ones(sum(nEmax), dtype=torch.float32, device=DEV)
    sink = torch.randn((H,), generator=g, device=DEV)
    rb = L.csa_entry_row_bytes(fmt, D)

    # contiguous reference: linear raw store, contiguous entries
    kv_off_d, ent_off_d = kv_off.to(DEV), ent_off.to(DEV)
    kv_pos0 = torch.zeros(B, dtype=torch.int64, device=DEV)
    ents_lin = torch.zeros((sum(nEmax), rb), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    seq_len = torch.tensor(T0, dtype=torch.int64, device=DEV)
    iseq = torch.cat([torch.full((t // 4,), b, dtype=torch.int32) for b, t in enumerate(T0)]).to(DEV)
    ient = torch.cat([torch.arange(t // 4, dtype=torch.int32) for t in T0]).to(DEV)
    L.csa_compress(kv_all, gate_all, bias, seq_len, kv_off_d, kv_pos0, ent_off_d, iseq, ient,
                   ents_lin, B=B, D=D, fmt=fmt, dev_status=st)

    # the hybrid cache, its blocks handed out in shuffled order
    n_blocks = sum((n + 31) // 32 for n in nEmax) + 8
    hc = cache.HybridCache(B, D, fmt, d_I, n_blocks=n_blocks, max_blocks=max(nEmax) // 32 + 2,
                           ring=ring, device=DEV)
    perm = torch.randperm(n_blocks, generator=torch.Generator().manual_seed(5)).tolist()
    hc.alloc.free = perm
    for b, T in enumerate(T0):
        r0, e0, n = int(kv_off[b]), int(ent_off[b]), T // 4
        lo = max(T - ring, 0)
        hc.load_prefix(b, kv_all[r0 + lo:r0 + T], gate_all[r0 + lo:r0 + T], T,
                       ents_lin[e0:e0 + n], kI_all[e0:e0 + n], ks_all[e0:e0 + n])

    q_seq = torch.arange(B, dtype=torch.int32, device=DEV)
    crossed = 0
    for s in range(S):
        p = [t + s for t in T0]                     # the new token's position
        rows = torch.tensor([int(kv_off[b]) + p[b] for b in range(B)], device=DEV)
        erow = torch.tensor([int(ent_off[b]) + max((p[b] + 1) // 4 - 1, 0) for b in range(B)],
                            device=DEV)
        q = (torch.randn((B, H, D), generator=g, device=DEV)).to(torch.bfloat16)
        qI = synth.fp8_integer((B, H_I, d_I), g, DEV)
        qs = torch.ones((B, H_I), dtype=torch.float32, device=DEV)
        w = torch.rand((B, H_I), generator=g, device=DEV)
        q_pos = torch.tensor(p, dtype=torch.int32, device=DEV)
        # reference step
        seq_len = torch.tensor([x + 1 for x in p], dtype=torch.int64, device=DEV)
        done = [b for b in range(B) if (p[b] + 1) % 4 == 0]
        if done:
            L.csa_compress(kv_all, gate_all, bias, seq_len, kv_off_d, kv_pos0, ent_off_d,
                           torch.tensor(done, dtype=torch.int32, device=DEV),
                           torch.tensor([(p[b] + 1) // 4 - 1 for b in done], dtype=torch.int32,
                                        device=DEV),
                           ents_lin, B=B, D=D, fmt=fmt, dev_status=st)
        max_n = max(x + 1 for x in p) // 4
        idx_ref = torch.full((B, k), -1, dtype=torch.int32, device=DEV)
        ws = torch.empty(L.csa_indexer_workspace_size(B, max_n, k), dtype=torch.uint8, device=DEV)
        L.lightning_indexer_topk(qI, qs, w, kI_all, ks_all, seq_len, ent_off_d, q_seq, q_pos,
                                 idx_ref, ws, B=B, H_I=H_I, d_I=d_I, m=4, k=k, max_n=max_n,
                                 dev_status=st)
        out_ref = torch.zeros((B, H, D), dtype=torch.bfloat16, device=DEV)
        L.sparse_mqa_attn(q, ents_lin, seq_len, ent_off_d, kv_all, kv_off_d, kv_pos0, q_seq,
                          q_pos, idx_ref, sink, out_ref, fmt=fmt, B=B, H=H, D=D, W=W, m=4, k=k,
                          softmax_scale=1.0 / np.sqrt(D), dev_status=st)
        # the hybrid cache's step
        nb0 = len(hc.alloc.free)
        items = hc.append(kv_all[rows], gate_all[rows], kI_all[erow], ks_all[erow])
        crossed += nb0 - len(hc.alloc.free)
        hc.compress(items, bias)
        idx = torch.full((B, k), -1, dtype=torch.int32, device=DEV)
        hc.select(qI, qs, w, q_seq, q_pos, idx, H_I=H_I, k=k)
        out = torch.zeros((B, H, D), dtype=torch.bfloat16, device=DEV)
        hc.attend(q, q_seq, q_pos, idx, sink, out, H=H, W=W, k=k, softmax_scale=1.0 / np.sqrt(D))
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(hc.dev_status.item()) == 0, s
        assert torch.equal(idx, idx_ref), s
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16)), s
    assert crossed >= 2                                    # new blocks were taken mid-run
    assert torch.equal(hc.seq_len.cpu(), torch.tensor(Tmax))
    # every entry, in its block, equals the contiguous one
    bt = hc.bt_host
    for b in range(B):
        n = Tmax[b] // 4
        i = torch.arange(n)
        prow = (bt[b, i // 32].to(torch.int64) * 32 + i % 32).to(DEV)
        assert torch.equal(hc.entries[prow], ents_lin[int(ent_off[b]):int(ent_off[b]) + n]), b


def test_block_table_rejected_by_dense_attention_and_other_ratios():
    hc = cache.HybridCache(1, 128, 0, 128, n_blocks=2, max_blocks=2, device=DEV)
    lay = hc.layout
    q = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros_like(q)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    z32 = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(L.CSAError, match="block table"):
        L.dense_hca_attn(q, hc.entries, hc.seq_len, None, hc.kv, hc.kv_off, None, z32, z32,
                         torch.zeros(64, device=DEV), out, ws, fmt=0, B=1, H=64, D=128, W=128,
                         m=128, max_n=1, softmax_scale=0.1, layout=lay)
    with pytest.raises(L.CSAError, match="m = 4"):
        L.hca_compress(hc.kv, hc.gate, torch.zeros((128, 128), device=DEV), hc.seq_len,
                       hc.kv_off, None, None, z32, z32, hc.entries, B=1, D=128, layout=lay)
