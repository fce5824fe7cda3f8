"""Batch invariance of the whole decode pass ("DeepSeek为保护V4的特性不遗余力": a token's
output is bitwise identical in any batch; "DeepSeek-V4 深度分析报告" 3.3).

The same target sequences are decoded inside batches of different sizes, next to random
neighbour sequences and in different slots, through the whole hot path of one decode step:
compression of each sequence's newest entry, lightning indexer + top-k, attention.  The
compressed cache before the step is a set of stored-format rows drawn once per sequence
(the raw store keeps only the tail, as a decode state does).  Each target's index set,
indexer scores and attention output must be bitwise equal in every batch."""
import numpy as np
import pytest
import torch

from long_context_compressed_04_b200 import pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pool(T, *, D, H, fmt, m, span, H_I=0, d_I=0, k=0, seed):
    """All sequences of a sweep, split into single-sequence workloads, and their cache rows."""
    base = synth.make_workload("inv", B=len(T), T=T, D=D, H=H, m=m, span=span, fmt=fmt,
                               H_I=H_I, d_I=d_I, k=k, indexer="fp8", keep_raw=256, seed=seed,
                               device=DEV)
    parts = synth.split(base)
    g = torch.Generator(device=DEV).manual_seed(seed + 1)
    rows = [synth.random_entries(int(p.n_ent[0]), fmt, D, g, DEV) for p in parts]
    return parts, rows


def _step(parts, rows, order, targets):
    """One decode step over the sequences `order` (indices into parts); per target present:
    (index set, scores, output)."""
    wl = synth.merge([parts[i] for i in order])
    buf = pipeline.alloc(wl, DEV)
    for slot, i in enumerate(order):
        e0 = int(wl.ent_off[slot])
        buf.entries[e0:e0 + rows[i].shape[0]].copy_(rows[i])
    seq, ent = pipeline.newest_entry_items(wl, DEV)
    pipeline.compress(wl, buf, seq, ent)
    sc = None
    if wl.H_I:
        sc = torch.zeros((wl.Q, buf.max_n), dtype=torch.float32, device=DEV)
        pipeline.indexer_topk(wl, buf, scores_out=sc)
    pipeline.attend(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    res = {}
    for slot, i in enumerate(order):
        if i in targets:
            n = int(wl.n_ent[slot])
            res[i] = (None if buf.idx is None else buf.idx[slot].clone(),
                      None if sc is None else sc[slot, :n].clone(), buf.out[slot].clone())
    return res


def _sweep(parts, rows, targets, batches):
    got = {t: [] for t in targets}
    for order in batches:
        for t, r in _step(parts, rows, order, targets).items():
            got[t].append(r)
    for t in targets:
        assert len(got[t]) >= 3, t
        idx0, sc0, out0 = got[t][0]
        for idx, sc, out in got[t][1:]:
            if idx0 is not None:
                assert torch.equal(idx, idx0), t
                assert torch.equal(sc.view(torch.int32), sc0.view(torch.int32)), t
            assert torch.equal(out.view(torch.int16), out0.view(torch.int16)), t


def _batches(targets, neighbours, sizes, seed):
    """Batches of the given sizes: every target alone (size 1); otherwise the targets (as
    many as fit) with neighbours, in shuffled slots."""
    rng = np.random.default_rng(seed)
    out = []
    for size in sizes:
        if size == 1:
            out += [[t] for t in targets]
            continue
        for start in range(0, len(targets), max(size - 1, 1)):
            ts = targets[start:start + size - 1] if size <= len(targets) else targets
            fill = list(rng.choice(neighbours, size - len(ts), replace=False))
            order = [int(x) for x in ts] + [int(x) for x in fill]
            rng.shuffle(order)
            out.append(order)
            if size > len(targets):
                break
    return out


def test_csa_decode_1m_fp8_sweep_1_7_32_64():
    # the 1M configuration: 8 target queries at 1,048,576 tokens (576-dim FP8 entries, 128
    # heads, top-1024, 64 x 128 FP8 indexer) inside batches of 1, 7, 32 and 64 with
    # neighbours of 4K - 1M tokens
    g = torch.Generator().manual_seed(11)
    neigh = [int(x) for x in torch.randint(4096, (1 << 20) + 1, (56,), generator=g)]
    T = [1 << 20] * 8 + neigh
    parts, rows = _pool(T, D=576, H=128, fmt=1, m=4, span=8, H_I=64, d_I=128, k=1024, seed=51)
    targets = list(range(8))
    _sweep(parts, rows, targets, _batches(targets, list(range(8, 64)), [1, 7, 32, 64], 3))


def test_csa_decode_128k_sweep_1_7_64():
    # the 128K configuration: 4 targets of 131072 +- 1024 tokens (64 heads x 128, top-512)
    # inside batches of 1, 7 and 64 with neighbours of 4K - 256K tokens
    g = torch.Generator().manual_seed(12)
    neigh = [int(x) for x in torch.randint(4096, 262145, (60,), generator=g)]
    T = synth.jittered_lengths(4, 131072, 1024, 5) + neigh
    parts, rows = _pool(T, D=128, H=64, fmt=0, m=4, span=8, H_I=64, d_I=128, k=512, seed=52)
    targets = list(range(4))
    _sweep(parts, rows, targets, _batches(targets, list(range(4, 64)), [1, 7, 64], 4))


def test_hca_decode_sweep_1_7_64_across_chunk_grids():
    # HCA dense attention: 4 targets of 1,048,576 tokens (8192 entries) inside batches of 1,
    # 7 and 64 whose neighbours range from 4K to 2M tokens, so the longest sequence of the
    # batch -- and with it the launch's grid of fixed-size chunks -- changes from batch to
    # batch while each target's own chunks stay the same
    g = torch.Generator().manual_seed(13)
    neigh = [int(x) for x in torch.randint(4096, (2 << 20) + 1, (60,), generator=g)]
    T = [1 << 20] * 4 + neigh
    parts, rows = _pool(T, D=128, H=64, fmt=0, m=128, span=128, seed=53)
    targets = list(range(4))
    batches = _batches(targets, list(range(4, 64)), [1, 7, 64], 5)
    # at least one batch whose longest sequence is a neighbour longer than the targets
    assert any(max(T[i] for i in b) > (1 << 20) for b in batches)
    _sweep(parts, rows, targets, batches)
