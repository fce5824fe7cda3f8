"""GPU parity of sparse_mqa_attn / dense_hca_attn against the oracle.

Both sides get the same stored entries and the same index sets, made by the oracle (the
stage-isolated comparison), so only the attention arithmetic is compared.  Tolerance for
bf16 / fp8 storage with fp32 accumulation: max abs error <= 2e-2, relative L2 <= 5e-3."""
import numpy as np
import pytest
import torch

import _orc
import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import CSA_DEV_OOB, pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _with_oracle_entries(wl):
    """Oracle-compressed entries for every complete block; installed as the GPU's buffer."""
    rows, _ = _orc.compress(wl.to("cpu"))
    buf = pipeline.alloc(wl, DEV)
    buf.entries.copy_(torch.from_numpy(rows))
    return buf, rows


def _random_idx(wl, seed, pad=0):
    g = np.random.default_rng(seed)
    n = (_orc.i64(wl.q_pos) + 1) // wl.m
    idx = np.full((wl.Q, wl.k), -1, np.int32)
    for q in range(wl.Q):
        take = min(wl.k - pad, int(n[q]))
        idx[q, :take] = np.sort(g.choice(int(n[q]), take, replace=False))
    return idx


@pytest.mark.parametrize("H,D,fmt,k,T", [
    (16, 128, 0, 64, [4096]),                      # CSA decode 4K shape
    (16, 128, 0, 512, [7001, 3000, 2100]),         # 16 heads, clusters of several CTAs
    (64, 128, 0, 512, [7001, 3000, 2100]),         # CSA decode, ragged, k = 512
    (64, 128, 0, 1024, [9001, 4000, 300]),         # k = 1024: one CTA per query combines
    (64, 128, 0, 2048, [20003, 9000]),             # all 64 heads (the prefill kernel shape)
    (128, 576, 1, 256, [3000, 1500]),              # 576-dim fp8 + bf16 RoPE entries
    (128, 576, 1, 1024, [9000, 3333, 200]),        # 1M-config shape: k = 1024, short rows padded
    (64, 576, 0, 128, [1203]),                     # 576-dim bf16 entries
])
def test_sparse_attention(H, D, fmt, k, T):
    wl = synth.make_workload("t", B=len(T), T=T, D=D, H=H, m=4, span=8, fmt=fmt, H_I=4, d_I=64,
                             k=k, seed=31, device=DEV)
    buf, rows = _with_oracle_entries(wl)
    idx = _random_idx(wl, 1, pad=3)
    buf.idx.copy_(torch.from_numpy(idx))
    pipeline.attend(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    ref = _orc.attention(wl.to("cpu"), rows, idx)
    _orc.assert_out_close(buf.out, ref)


@pytest.mark.parametrize("H,T", [(64, [128 * 40 + 77, 128 * 7]), (64, [300]),
                                 (64, [128 * 2500 + 77, 130]), (16, [128 * 300 + 5, 1000])])
def test_dense_hca_attention(H, T):
    # 16 heads run on the 64-head tile with zero heads added
    wl = synth.make_workload("t", B=len(T), T=T, D=128, H=H, m=128, span=128, seed=32,
                             device=DEV)
    buf, rows = _with_oracle_entries(wl)
    pipeline.attend(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    _orc.assert_out_close(buf.out, _orc.attention(wl.to("cpu"), rows, None))


@pytest.mark.parametrize("H,D,fmt", [(16, 128, 0), (64, 128, 0), (128, 576, 1)])
def test_short_window_and_no_window(H, D, fmt):
    for W, T in [(128, [37]), (0, [400]), (5, [400]), (128, [3]), (70, [900])]:
        wl = synth.make_workload("t", B=len(T), T=T, D=D, H=H, m=4, span=8, W=W, H_I=4,
                                 d_I=64, k=32, fmt=fmt, seed=33, device=DEV)
        buf, rows = _with_oracle_entries(wl)
        idx = _random_idx(wl, 2)
        buf.idx.copy_(torch.from_numpy(idx))
        pipeline.attend(wl, buf)
        torch.cuda.synchronize()
        _orc.assert_out_close(buf.out, _orc.attention(wl.to("cpu"), rows, idx))


@pytest.mark.parametrize("H,D,fmt", [(16, 128, 0), (64, 128, 0), (128, 576, 1)])
def test_sink_limits(H, D, fmt):
    wl = synth.make_workload("t", B=1, T=[2000], D=D, H=H, m=4, span=8, H_I=4, d_I=64, k=64,
                             fmt=fmt, seed=34, device=DEV)
    buf, rows = _with_oracle_entries(wl)
    idx = _random_idx(wl, 3)
    buf.idx.copy_(torch.from_numpy(idx))
    for sink in (-1e30, 60.0):
        wl.sink.fill_(sink)
        pipeline.attend(wl, buf)
        torch.cuda.synchronize()
        _orc.assert_out_close(buf.out, _orc.attention(wl.to("cpu"), rows, idx))
    assert buf.out.abs().max().item() < 1e-20   # sink = 60 >> logits: output ~ e^-50


@pytest.mark.parametrize("H,D,fmt", [(16, 128, 0), (64, 128, 0), (128, 576, 1)])
def test_out_of_range_index_is_flagged_and_skipped(H, D, fmt):
    wl = synth.make_workload("t", B=1, T=[2000], D=D, H=H, m=4, span=8, H_I=4, d_I=64, k=64,
                             fmt=fmt, seed=35, device=DEV)
    buf, rows = _with_oracle_entries(wl)
    idx = _random_idx(wl, 4, pad=1)
    bad = idx.copy()
    bad[0, -1] = 500                                # visible entries are 0..499
    buf.idx.copy_(torch.from_numpy(bad))
    pipeline.attend(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) & CSA_DEV_OOB
    _orc.assert_out_close(buf.out, _orc.attention(wl.to("cpu"), rows, idx))


def test_batch_invariance_bitwise():
    base = synth.make_workload("t", B=6, T=[3001, 9000, 777, 12345, 4096, 50], D=128, H=64,
                               m=4, span=8, H_I=4, d_I=64, k=512, seed=36, device=DEV)
    parts = synth.split(base)
    outs = {}
    for order in ([3], [1, 3, 0], [5, 4, 3, 2, 1, 0]):
        wl = synth.merge([parts[i] for i in order])
        buf, _ = _with_oracle_entries(wl)
        buf.idx.copy_(torch.from_numpy(_random_idx(wl, 0)))
        # the target's own index row must not depend on the batch: rebuild it per sequence
        tgt = order.index(3)
        buf.idx[tgt].copy_(torch.from_numpy(_random_idx(synth.merge([parts[3]]), 7)[0]))
        pipeline.attend(wl, buf)
        torch.cuda.synchronize()
        outs[tuple(order)] = buf.out[tgt].clone()
    vals = list(outs.values())
    for v in vals[1:]:
        assert torch.equal(v.view(torch.int16), vals[0].view(torch.int16))


def test_batch_invariance_bitwise_576_fp8_sweep():
    # the 1M configuration's sweep on the attention stage: the same queries inside batches of
    # 1, 7, 32 and 64 with random neighbour sequences; entries stored directly (656-byte rows)
    g = torch.Generator().manual_seed(5)
    lens = [int(x) for x in torch.randint(4096, 200000, (64,), generator=g)]
    base = synth.make_workload("t", B=64, T=lens, D=576, H=128, m=4, span=8, fmt=1, H_I=4,
                               d_I=64, k=1024, keep_raw=128, seed=37, device=DEV)
    parts = synth.split(base)
    targets = [0, 1]
    gd = torch.Generator(device=DEV).manual_seed(9)
    ents = synth.random_entries(base.ent_rows, 1, 576, gd, DEV)
    idx_all = torch.from_numpy(_random_idx(base, 11))
    outs = {}
    for batch in ([0], [1], [0, 1] + list(range(2, 7)), list(range(32)), list(range(63, -1, -1))):
        wl = synth.merge([parts[i] for i in batch])
        buf = pipeline.alloc(wl, DEV)
        for slot, i in enumerate(batch):
            e0, n = int(base.ent_off[i]), int(base.n_ent[i])
            f0 = int(wl.ent_off[slot])
            buf.entries[f0:f0 + n].copy_(ents[e0:e0 + n])
            buf.idx[slot].copy_(idx_all[i])
        pipeline.attend(wl, buf)
        torch.cuda.synchronize()
        assert int(buf.dev_status.item()) == 0
        for tgt in targets:
            if tgt in batch:
                outs.setdefault(tgt, []).append(buf.out[batch.index(tgt)].clone())
    for tgt in targets:
        ref = outs[tgt][0]
        assert len(outs[tgt]) >= 3
        for v in outs[tgt][1:]:
            assert torch.equal(v.view(torch.int16), ref.view(torch.int16))


def _scale_rows_pow2(rows, fmt, D, p):
    """Entry e multiplied by 2^p[e] (exact: bf16 values, fp8 block scales and the bf16 RoPE
    part all scale by a power of two without rounding)."""
    out = rows.copy()
    f = np.exp2(p.astype(np.float64)).astype(np.float32)[:, None]
    def bf16_scale(u16):
        x = (u16.astype(np.uint32) << 16).view(np.float32) * f
        return (x.view(np.uint32) >> 16).astype(np.uint16)
    if fmt == 0:
        out.view(np.uint16)[:] = bf16_scale(out.view(np.uint16))
    else:
        out[:, 512:528].view(np.float32)[:] = out[:, 512:528].view(np.float32) * f
        out[:, 528:656].view(np.uint16)[:] = bf16_scale(out[:, 528:656].view(np.uint16))
    return out


@pytest.mark.parametrize("mode,H,D,fmt", [("sparse", 64, 128, 0), ("dense", 64, 128, 0),
                                          ("sparse", 128, 576, 1)])
def test_rising_scores_move_the_reference_maximum(mode, H, D, fmt):
    # Entry e is scaled by 2^min(e // 128, 3): in entry order the scores of later key tiles
    # exceed the running reference maximum by far more than 2^8 in the exponent, so the
    # kernels must rescale their partial outputs; in reverse order the maximum comes first
    # and later tiles never move it.  Attention is invariant under the order of its keys,
    # and both runs see the same rounded q and keys (so the same logits), so the outputs
    # may differ only by the rounding of P and of the bf16 output: a few ulps of the output's
    # largest binade (2^-6 of its magnitude).  (The
    # oracle keeps q unrounded, which at these logit magnitudes leaves near-tied heads
    # ill-conditioned; the unscaled cases above pin both orders' arithmetic to it.)
    if mode == "dense":
        wl = synth.make_workload("t", B=1, T=[128 * 2500 + 77], D=D, H=H, m=128, span=128,
                                 seed=36, device=DEV)
    else:
        wl = synth.make_workload("t", B=2, T=[20000, 9000], D=D, H=H, m=4, span=8, H_I=4,
                                 d_I=64, k=512, fmt=fmt, seed=36, device=DEV)
    rows, _ = _orc.compress(wl.to("cpu"))
    ent_off = _orc.i64(wl.ent_off)
    bounds = [(int(ent_off[b]), int(ent_off[b + 1]) if b + 1 < wl.B else rows.shape[0])
              for b in range(wl.B)]
    p = np.zeros(rows.shape[0], np.int64)
    for lo, hi in bounds:
        p[lo:hi] = np.minimum(np.arange(hi - lo) // 128, 3)
    rows = _scale_rows_pow2(rows, fmt, D, p)
    outs = []
    for order in ("rising", "falling"):
        buf = pipeline.alloc(wl, DEV)
        if mode == "dense":
            r = rows.copy()
            if order == "falling":
                for lo, hi in bounds:
                    r[lo:hi] = rows[lo:hi][::-1]
            buf.entries.copy_(torch.from_numpy(r))
        else:
            buf.entries.copy_(torch.from_numpy(rows))
            idx = _random_idx(wl, 5, pad=3)
            if order == "falling":
                for q in range(wl.Q):
                    v = idx[q][idx[q] >= 0][::-1]
                    idx[q, :len(v)] = v
            buf.idx.copy_(torch.from_numpy(idx))
        pipeline.attend(wl, buf)
        torch.cuda.synchronize()
        assert int(buf.dev_status.item()) == 0
        outs.append(buf.out.float().cpu().numpy())
    a, b = outs
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    mag = np.abs(b).max()
    assert mag > 4.0                     # the scaled entries dominate the output
    assert np.abs(a - b).max() <= mag * 2.0 ** -6
    assert np.linalg.norm(a - b) <= 5e-3 * np.linalg.norm(b)


def test_dense_dual_kernels_bitwise_equal():
    # HCA dense attention runs in one of two variants chosen by the batch: small batches
    # spread each query's chunks over CTAs and combine them in a second kernel; batches of
    # at least as many queries as SMs give each query one CTA that combines its own chunks.
    # The chunks and the combine arithmetic are the same, so a query's output must be
    # bitwise the same in both; the variant is seen in the number of launches (2 vs 1).
    g = torch.Generator().manual_seed(17)
    lens = [int(x) for x in torch.randint(128 * 8, 128 * 1500, (160,), generator=g)]
    base = synth.make_workload("t", B=160, T=lens, D=128, H=64, m=128, span=128,
                               keep_raw=256, seed=38, device=DEV)
    parts = synth.split(base)
    gd = torch.Generator(device=DEV).manual_seed(19)
    rows = [synth.random_entries(int(p.n_ent[0]), 0, 128, gd, DEV) for p in parts]

    def run(order):
        wl = synth.merge([parts[i] for i in order])
        buf = pipeline.alloc(wl, DEV)
        for slot, i in enumerate(order):
            e0 = int(wl.ent_off[slot])
            buf.entries[e0:e0 + rows[i].shape[0]].copy_(rows[i])
        n0 = L.csa_launch_count()
        pipeline.attend(wl, buf)
        torch.cuda.synchronize()
        assert int(buf.dev_status.item()) == 0
        return buf.out, L.csa_launch_count() - n0

    big, n_big = run(list(range(160)))
    assert n_big == 1
    for tgt in (0, 77, 159):
        small, n_small = run([tgt])
        assert n_small == 2
        assert torch.equal(small[0].view(torch.int16), big[tgt].view(torch.int16))
