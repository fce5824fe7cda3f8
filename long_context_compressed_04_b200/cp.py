"""Context-parallel decode: one step for sequences whose compressed entries (and indexer
keys) are split across ranks, as the stuffyNLP post's context parallelism splits a long
sequence over GPUs.

Rank r holds a contiguous slice [lo_r, hi_r) of every sequence's entries; the query inputs
and the raw tail (the window) are on every rank.  One decode step:
 1. each rank selects the top-k of its slice (``lightning_indexer_topk`` with scores) and
    ``csa_cp_candidates`` turns it into candidates: entry indices of the whole sequence and
    their scores, one [2, Q, k] int32 buffer (indices, then the scores' bits);
 2. the buffers are gathered on every rank, slices in rank order (one all_gather into a
    [W, 2, Q, k] tensor);
 3. ``csa_topk_merge`` selects the sequence's top-k from them -- the same index set, bit for
    bit, as one GPU selecting over the whole sequence;
 4. ``csa_cp_pack_rows`` writes the selected rows of the rank's slice into a [Q, k, row]
    buffer at their output positions (zeros elsewhere); every position has one rank with a
    non-zero row, so an integer sum over the ranks (one all_reduce) gathers every row;
 5. the attention runs over those rows, renumbered 0..k-1: the same keys in the same order
    as on one GPU, so the same output bits.
Rows cross ranks only through the collectives (no kernel reads another GPU's memory).  A
step issues library kernels and the two collectives only: no host synchronisation, so it
can be captured in a CUDA graph.

This module only slices, allocates and exchanges; every score, selection, translation, row
copy and attention is a libcsa call.  One query per sequence (decode).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional

import torch

from . import (csa_cp_candidates, csa_cp_pack_rows, csa_entry_row_bytes,
               csa_indexer_workspace_size, csa_topk_merge, lightning_indexer_topk,
               sparse_mqa_attn)
from .synth import Workload


def slice_bounds(n_ent: int, world: int, rank: int):
    """Contiguous slice [lo, hi) of n_ent entries owned by `rank` of `world`."""
    return n_ent * rank // world, n_ent * (rank + 1) // world


@dataclasses.dataclass
class Slice:
    """A rank's slice of a batch of sequences, laid out for the library calls."""
    lo: torch.Tensor        # [B] int64: first entry of the slice, per sequence
    n: torch.Tensor         # [B] int64: entries of the slice (hi - lo)
    seq_len: torch.Tensor   # [B] int64: the slice as a sequence of its own (see make_slice)
    ent_off: torch.Tensor   # [B] int64: the slice's first row in the rank's key / entry store
    q_pos: torch.Tensor     # [Q] int32: a position whose visible entries are the query's
    max_n: int              # the most entries a query sees in this slice (>= 1)


def make_slice(wl: Workload, world: int, rank: int, ent_off_local: torch.Tensor) -> Slice:
    """The rank's slice of `wl` (entries numbered per sequence as in `wl`), with the slice's
    rows starting at ent_off_local[b] in the rank's own stores.

    The slice of sequence b is a sequence of its own with n entries and m - 1 more tokens
    that complete no entry (seq_len = n * m + m - 1), so that position 0 -- which sees no
    entry -- is valid even for an empty slice.  A query that sees nv of the slice's entries
    sits at position nv * m - 1 (0 for nv = 0)."""
    assert wl.m >= 2
    dev = wl.q_pos.device
    n_ent = wl.n_ent.cpu()
    lo = torch.tensor([slice_bounds(int(x), world, rank)[0] for x in n_ent], dtype=torch.int64)
    hi = torch.tensor([slice_bounds(int(x), world, rank)[1] for x in n_ent], dtype=torch.int64)
    n = hi - lo
    qs = wl.q_seq.cpu().to(torch.int64)
    vis = (wl.q_pos.cpu().to(torch.int64) + 1) // wl.m
    nv = torch.minimum(torch.clamp(vis - lo[qs], min=0), n[qs])
    q_pos = torch.where(nv > 0, nv * wl.m - 1, torch.zeros_like(nv)).to(torch.int32)
    return Slice(lo=lo.to(dev), n=n.to(dev), seq_len=(n * wl.m + wl.m - 1).to(dev),
                 ent_off=ent_off_local.to(torch.int64).to(dev), q_pos=q_pos.to(dev),
                 max_n=max(int(nv.max()) if nv.numel() else 0, 1))


@dataclasses.dataclass
class Buffers:
    """One rank's device buffers for a decode step."""
    scores: torch.Tensor     # [Q, max_n] fp32: the slice's indexer scores
    sel: torch.Tensor        # [Q, k] int32: the slice's top-k (slice-local)
    workspace: torch.Tensor  # the selection's workspace
    cand: torch.Tensor       # [2, Q, k] int32: candidates (indices; scores' bits)
    gathered: torch.Tensor   # [W, 2, Q, k] int32: every rank's candidates, rank order
    idx: torch.Tensor        # [Q, k] int32: the merged top-k (entry indices of the sequence)
    packed: torch.Tensor     # [Q, k, row] uint8: selected rows (this rank's, then all)
    local_idx: torch.Tensor  # [Q, k] int32: the selection renumbered to packed's positions
    attn_off: torch.Tensor   # [B] int64: the first packed row of each sequence's query
    out: torch.Tensor        # [Q, H, D] bf16
    dev_status: torch.Tensor


def alloc(wl: Workload, sl: Slice, world: int, device) -> Buffers:
    Q, k = wl.Q, wl.k
    assert int(wl.Q) == int(wl.B) and sorted(wl.q_seq.tolist()) == list(range(wl.B)), \
        "one query per sequence"
    rb = csa_entry_row_bytes(wl.fmt, wl.D)
    ws = csa_indexer_workspace_size(Q, sl.max_n, k)
    attn_off = torch.empty(wl.B, dtype=torch.int64)
    attn_off[wl.q_seq.cpu().long()] = torch.arange(Q, dtype=torch.int64) * k
    i32 = dict(dtype=torch.int32, device=device)
    return Buffers(scores=torch.zeros((Q, sl.max_n), dtype=torch.float32, device=device),
                   sel=torch.full((Q, k), -1, **i32),
                   workspace=torch.zeros(max(ws, 256), dtype=torch.uint8, device=device),
                   cand=torch.zeros((2, Q, k), **i32),
                   gathered=torch.zeros((world, 2, Q, k), **i32),
                   idx=torch.full((Q, k), -1, **i32),
                   packed=torch.zeros((Q, k, rb), dtype=torch.uint8, device=device),
                   local_idx=torch.full((Q, k), -1, **i32),
                   attn_off=attn_off.to(device),
                   out=torch.zeros((Q, wl.H, wl.D), dtype=torch.bfloat16, device=device),
                   dev_status=torch.zeros(1, **i32))


def select_local(wl: Workload, sl: Slice, kI: torch.Tensor, ks: torch.Tensor, buf: Buffers,
                 stream=None):
    """Step 1: the top-k of the rank's slice, as candidates in buf.cand.  kI / ks: the rank's
    key store (the slice of sequence b at rows sl.ent_off[b] ..)."""
    lightning_indexer_topk(wl.qI, wl.qs, wl.w, kI, ks, sl.seq_len, sl.ent_off, wl.q_seq,
                           sl.q_pos, buf.sel, buf.workspace, B=wl.B, H_I=wl.H_I, d_I=wl.d_I,
                           m=wl.m, k=wl.k, max_n=sl.max_n, scores_out=buf.scores,
                           ld_scores=sl.max_n, dev_status=buf.dev_status, stream=stream)
    csa_cp_candidates(buf.sel, buf.scores, wl.q_seq, sl.lo, buf.cand[0],
                      buf.cand[1].view(torch.float32), B=wl.B, dev_status=buf.dev_status,
                      stream=stream)


def exchange_candidates(buf: Buffers, group=None, all_gather: Optional[Callable] = None):
    """Step 2: every rank's candidates into buf.gathered, rank order (all_gather_into_tensor,
    or a stand-in taking (out, in))."""
    if all_gather is not None:
        return all_gather(buf.gathered, buf.cand)
    import torch.distributed as dist
    # the concatenated form ([W * 2, Q, k]), which every backend takes
    dist.all_gather_into_tensor(buf.gathered.view(-1, *buf.cand.shape[1:]), buf.cand,
                                group=group)


def merge(wl: Workload, buf: Buffers, stream=None):
    """Step 3: the sequence's top-k from the gathered candidates, into buf.idx."""
    csa_topk_merge(buf.gathered[:, 1].view(torch.float32), buf.gathered[:, 0], buf.idx,
                   dev_status=buf.dev_status, stream=stream)


def pack(wl: Workload, sl: Slice, entries: torch.Tensor, buf: Buffers, stream=None):
    """Step 4, local part: the selected rows of this rank's slice into buf.packed.  entries:
    the rank's store, the slice of sequence b at rows sl.ent_off[b] .."""
    csa_cp_pack_rows(buf.idx, wl.q_seq, sl.lo, sl.n, sl.ent_off, entries, buf.packed,
                     buf.local_idx, B=wl.B, dev_status=buf.dev_status, stream=stream)


def exchange_rows(buf: Buffers, group=None, all_reduce: Optional[Callable] = None):
    """Step 4, exchange: the integer sum of every rank's packed rows (each position has one
    non-zero contributor, so the sum is the gather), in place."""
    t = buf.packed.view(torch.int32)
    if all_reduce is not None:
        return all_reduce(t)
    import torch.distributed as dist
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def attend(wl: Workload, buf: Buffers, stream=None):
    """Step 5: the attention over the gathered rows (query q's at rows q * k ..); the window
    from the raw tail as usual."""
    Q, k = buf.idx.shape
    sparse_mqa_attn(wl.q, buf.packed.view(Q * k, -1), wl.seq_len, buf.attn_off, wl.kv,
                    wl.kv_off, wl.kv_pos0, wl.q_seq, wl.q_pos, buf.local_idx, wl.sink, buf.out,
                    fmt=wl.fmt, B=wl.B, H=wl.H, D=wl.D, W=wl.W, m=wl.m, k=k,
                    softmax_scale=wl.scale, rope_theta=wl.theta, eps=wl.eps,
                    dev_status=buf.dev_status, stream=stream)


def step(wl: Workload, sl: Slice, kI, ks, entries, buf: Buffers, group=None, stream=None):
    """One context-parallel decode step on this rank (every rank calls it)."""
    select_local(wl, sl, kI, ks, buf, stream)
    exchange_candidates(buf, group)
    merge(wl, buf, stream)
    pack(wl, sl, entries, buf, stream)
    exchange_rows(buf, group)
    attend(wl, buf, stream)


def exchange_bytes(wl: Workload, world: int):
    """Bytes one rank contributes to each exchange of a step: the candidate buffer (the
    all_gather sends it to every other rank) and the packed rows (the all_reduce)."""
    return 2 * wl.Q * wl.k * 4, wl.Q * wl.k * csa_entry_row_bytes(wl.fmt, wl.D)
