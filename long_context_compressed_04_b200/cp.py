"""Context-parallel decode: one step for sequences whose compressed entries (and indexer
keys) are split across ranks, as the stuffyNLP post's context parallelism splits a long
sequence over GPUs.

Rank r holds a contiguous slice [lo_r, hi_r) of every sequence's entries; the query inputs
and the raw tail (the window) are on every rank.  One decode step:
 1. each rank selects the top-k of its slice (``lightning_indexer_topk`` with scores);
 2. the slices' index sets (translated to entry indices of the whole sequence) and scores
    are gathered on every rank, slices in rank order (one ``all_gather``);
 3. ``csa_topk_merge`` selects the sequence's top-k from them -- the same index set, bit for
    bit, as one GPU selecting over the whole sequence;
 4. each rank writes the selected rows of its slice into a [k, row] buffer at their output
    positions, and the buffers are gathered (one ``all_gather``), so every rank holds the
    selected rows in index order;
 5. the attention runs over those rows, renumbered 0..k-1: the same keys in the same order
    as on one GPU, so the same output bits.
Rows cross ranks only through the collective (no kernel reads another GPU's memory).

This module only slices, marshals and exchanges; every score, selection and attention is a
libcsa call.  One query per sequence (decode).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional

import torch

from . import csa_entry_row_bytes, csa_topk_merge, lightning_indexer_topk, sparse_mqa_attn
from .synth import Workload


def slice_bounds(n_ent: int, world: int, rank: int):
    """Contiguous slice [lo, hi) of n_ent entries owned by `rank` of `world`."""
    return n_ent * rank // world, n_ent * (rank + 1) // world


@dataclasses.dataclass
class Slice:
    """A rank's slice of a batch of sequences, laid out for the library calls."""
    lo: torch.Tensor        # [B] int64: first entry of the slice, per sequence
    n: torch.Tensor         # [B] int64: entries of the slice (hi - lo)
    seq_len: torch.Tensor   # [B] int64: n * m, the slice as a sequence of its own
    ent_off: torch.Tensor   # [B] int64: the slice's first row in the rank's key store
    q_pos: torch.Tensor     # [Q] int32: n_vis * m - 1 for the slice's visible entries
    q_live: torch.Tensor    # [Q] bool: the query sees at least one entry of the slice


def make_slice(wl: Workload, world: int, rank: int, ent_off_local: torch.Tensor) -> Slice:
    """The rank's slice of `wl` (entries numbered per sequence as in `wl`), with the slice's
    rows starting at ent_off_local[b] in the rank's own key store."""
    dev = wl.q_pos.device
    n_ent = wl.n_ent.cpu()
    lo = torch.tensor([slice_bounds(int(x), world, rank)[0] for x in n_ent], dtype=torch.int64)
    hi = torch.tensor([slice_bounds(int(x), world, rank)[1] for x in n_ent], dtype=torch.int64)
    n = hi - lo
    qs = wl.q_seq.cpu().to(torch.int64)
    vis = (wl.q_pos.cpu().to(torch.int64) + 1) // wl.m
    nv = torch.clamp(vis - lo[qs], min=0)
    nv = torch.minimum(nv, n[qs])
    live = nv > 0
    q_pos = torch.where(live, nv * wl.m - 1, torch.zeros_like(nv)).to(torch.int32)
    return Slice(lo=lo.to(dev), n=n.to(dev), seq_len=(n * wl.m).to(dev),
                 ent_off=ent_off_local.to(dev), q_pos=q_pos.to(dev), q_live=live.to(dev))


def local_candidates(wl: Workload, sl: Slice, kI: torch.Tensor, ks: torch.Tensor,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """Step 1: the top-k of the rank's slice.  kI / ks: the rank's key store (the slice of
    sequence b at rows sl.ent_off[b] ..).  Returns (idx [Q, k] int32 entry indices of the
    whole sequence, -1 = none; scores [Q, k] fp32 of those entries)."""
    dev = wl.q.device
    Q, k = wl.Q, wl.k
    max_n = max(int(sl.n.max()), 1)
    scores = torch.zeros((Q, max_n), dtype=torch.float32, device=dev)
    idx = torch.full((Q, k), -1, dtype=torch.int32, device=dev)
    if workspace is None:
        from . import csa_indexer_workspace_size
        workspace = torch.empty(csa_indexer_workspace_size(Q, max_n, k), dtype=torch.uint8,
                                device=dev)
    live = sl.q_live
    if bool(live.any()):
        # queries that see no entry of this slice have no candidate here (they keep -1)
        sel = torch.nonzero(live).flatten()
        sub_idx = torch.full((sel.numel(), k), -1, dtype=torch.int32, device=dev)
        sub_sc = torch.zeros((sel.numel(), max_n), dtype=torch.float32, device=dev)
        lightning_indexer_topk(wl.qI[sel], wl.qs[sel], wl.w[sel], kI, ks, sl.seq_len, sl.ent_off,
                               wl.q_seq[sel], sl.q_pos[sel], sub_idx, workspace, B=wl.B,
                               H_I=wl.H_I, d_I=wl.d_I, m=wl.m, k=k, max_n=max_n,
                               scores_out=sub_sc, ld_scores=max_n, stream=stream)
        idx[sel] = sub_idx
        scores[sel] = sub_sc
    valid = idx >= 0
    cand_sc = torch.where(valid, torch.gather(scores, 1, idx.clamp_min(0).long()),
                          torch.zeros((), device=dev))
    lo = sl.lo[wl.q_seq.long()].to(torch.int32)[:, None]
    cand_idx = torch.where(valid, idx + lo, idx)
    return cand_idx, cand_sc


def exchange(t: torch.Tensor, group=None, all_gather: Optional[Callable] = None) -> List[torch.Tensor]:
    """Every rank's `t`, in rank order (torch.distributed.all_gather, or a stand-in)."""
    if all_gather is not None:
        return all_gather(t)
    import torch.distributed as dist
    out = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, t.contiguous(), group=group)
    return out


def merge_candidates(parts_idx: List[torch.Tensor], parts_sc: List[torch.Tensor], k: int,
                     dev_status=None, stream=None) -> torch.Tensor:
    """Steps 2-3: the sequence's top-k from the ranks' candidates (rank order)."""
    cand_idx = torch.cat(parts_idx, dim=1).contiguous()
    cand_sc = torch.cat(parts_sc, dim=1).contiguous()
    out = torch.full((cand_idx.shape[0], k), -1, dtype=torch.int32, device=cand_idx.device)
    csa_topk_merge(cand_sc, cand_idx, out, dev_status=dev_status, stream=stream)
    return out


def pack_rows(idx: torch.Tensor, sl: Slice, q_seq: torch.Tensor, entries: torch.Tensor,
              row_bytes: int) -> torch.Tensor:
    """Step 4, local part: [Q, k, row] with the rows of the selected entries that lie in this
    rank's slice at their output positions (zeros elsewhere).  entries: the rank's store,
    the slice of sequence b at rows sl.ent_off[b] .."""
    Q, k = idx.shape
    lo = sl.lo[q_seq.long()][:, None]
    n = sl.n[q_seq.long()][:, None]
    local = idx.to(torch.int64) - lo
    mine = (idx >= 0) & (local >= 0) & (local < n)
    rows = sl.ent_off[q_seq.long()][:, None] + local
    out = torch.zeros((Q, k, row_bytes), dtype=torch.uint8, device=idx.device)
    if bool(mine.any()):
        out[mine] = entries[rows[mine]]
    return out


def unpack_rows(parts: List[torch.Tensor], idx: torch.Tensor, sls: List[Slice],
                q_seq: torch.Tensor) -> torch.Tensor:
    """Step 4, after the exchange: each selected row from the rank whose slice holds it."""
    out = torch.zeros_like(parts[0])
    for part, sl in zip(parts, sls):
        lo = sl.lo[q_seq.long()][:, None]
        n = sl.n[q_seq.long()][:, None]
        local = idx.to(torch.int64) - lo
        mine = (idx >= 0) & (local >= 0) & (local < n)
        out[mine] = part[mine]
    return out


def attend_selected(wl: Workload, rows: torch.Tensor, idx: torch.Tensor, out: torch.Tensor,
                    dev_status=None, stream=None):
    """Step 5: the attention over the selected rows, renumbered 0..k-1 per query (query q's
    rows at q * k ..); the window from the raw tail as usual."""
    Q, k = idx.shape
    assert int(wl.Q) == int(wl.B), "one query per sequence"
    dev = idx.device
    qs = wl.q_seq.long()
    ent_off = torch.empty(wl.B, dtype=torch.int64, device=dev)
    ent_off[qs] = torch.arange(Q, dtype=torch.int64, device=dev) * k
    j = torch.arange(k, dtype=torch.int32, device=dev)[None, :].expand(Q, k)
    local_idx = torch.where(idx >= 0, j, torch.full_like(j, -1)).contiguous()
    flat = rows.reshape(Q * k, rows.shape[-1]).contiguous()
    sparse_mqa_attn(wl.q, flat, wl.seq_len, ent_off, wl.kv, wl.kv_off, wl.kv_pos0, wl.q_seq,
                    wl.q_pos, local_idx, wl.sink, out, fmt=wl.fmt, B=wl.B, H=wl.H, D=wl.D,
                    W=wl.W, m=wl.m, k=k, softmax_scale=wl.scale, rope_theta=wl.theta,
                    eps=wl.eps, dev_status=dev_status, stream=stream)


def row_bytes_of(wl: Workload) -> int:
    return csa_entry_row_bytes(wl.fmt, wl.D)
