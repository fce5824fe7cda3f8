"""Plumbing for one hot-path pass over a workload: buffer allocation with torch and the
sequence of libcsa calls (compress -> lightning indexer + top-k -> attention).

Nothing here computes: every step is a call into libcsa through the binding.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import (CSA_KV_BF16, csa_compress, csa_entry_row_bytes, csa_indexer_workspace_size,
               dense_hca_attn, dense_hca_workspace_size, hca_compress, lightning_indexer_topk,
               lightning_indexer_topk_mxfp4, sparse_mqa_attn)
from .synth import Workload


def all_entry_items(wl: Workload, device):
    """(item_seq, item_ent) listing every complete entry of every sequence."""
    n = wl.n_ent.cpu()
    seq = torch.repeat_interleave(torch.arange(wl.B, dtype=torch.int32), n)
    ent = torch.cat([torch.arange(int(x), dtype=torch.int32) for x in n]) if wl.B else seq
    return seq.to(device), ent.to(device)


def newest_entry_items(wl: Workload, device):
    """(item_seq, item_ent): the last complete entry of every sequence (one decode step's
    compression work)."""
    n = wl.n_ent.cpu()
    seq = torch.arange(wl.B, dtype=torch.int32)
    ent = (n - 1).clamp_min(0).to(torch.int32)
    keep = n > 0
    return seq[keep].to(device), ent[keep].to(device)


def max_visible(wl: Workload) -> int:
    return int(((wl.q_pos.cpu().to(torch.int64) + 1) // wl.m).max()) if wl.Q else 0


@dataclasses.dataclass
class Buffers:
    entries: torch.Tensor
    idx: Optional[torch.Tensor]
    out: torch.Tensor
    workspace: torch.Tensor
    dev_status: torch.Tensor
    max_n: int


def alloc(wl: Workload, device) -> Buffers:
    rb = csa_entry_row_bytes(wl.fmt, wl.D)
    entries = torch.zeros((max(wl.ent_rows, 1), rb), dtype=torch.uint8, device=device)
    max_n = max_visible(wl)
    if wl.H_I:
        ws = csa_indexer_workspace_size(wl.Q, max_n, wl.k)
        idx = torch.full((wl.Q, wl.k), -1, dtype=torch.int32, device=device)
    else:
        ws = dense_hca_workspace_size(wl.Q, wl.H, wl.D, max_n)
        idx = None
    workspace = torch.zeros(max(ws, 256), dtype=torch.uint8, device=device)
    out = torch.zeros((wl.Q, wl.H, wl.D), dtype=torch.bfloat16, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    return Buffers(entries, idx, out, workspace, st, max_n)


def compress(wl: Workload, buf: Buffers, item_seq, item_ent, stream=None):
    fn = csa_compress if wl.m == 4 else hca_compress
    fn(wl.kv, wl.gate, wl.bias, wl.seq_len, wl.kv_off, wl.kv_pos0, wl.ent_off, item_seq, item_ent,
       buf.entries, B=wl.B, D=wl.D, fmt=wl.fmt, rope_theta=wl.theta, eps=wl.eps,
       dev_status=buf.dev_status, stream=stream)


def indexer_topk(wl: Workload, buf: Buffers, scores_out=None, stream=None):
    lightning_indexer_topk(wl.qI, wl.qs, wl.w, wl.kI, wl.ks, wl.seq_len, wl.ent_off, wl.q_seq, wl.q_pos,
                           buf.idx, buf.workspace, B=wl.B, H_I=wl.H_I, d_I=wl.d_I, m=wl.m,
                           k=wl.k, max_n=buf.max_n, scores_out=scores_out,
                           ld_scores=0 if scores_out is None else scores_out.shape[1],
                           dev_status=buf.dev_status, stream=stream)


def indexer_topk_mxfp4(wl: Workload, fp4, buf: Buffers, select_bf16: bool = False,
                       scores_out=None, stream=None):
    """The MXFP4 indexer + top-k into buf.idx; fp4 = (qI, qI_sf, kI, kI_sf)."""
    qI, qsf, kI, ksf = fp4
    lightning_indexer_topk_mxfp4(qI, qsf, wl.w, kI, ksf, wl.seq_len, wl.ent_off, wl.q_seq,
                                 wl.q_pos, buf.idx, buf.workspace, B=wl.B, H_I=wl.H_I,
                                 d_I=wl.d_I, m=wl.m, k=wl.k, max_n=buf.max_n,
                                 select_bf16=select_bf16, scores_out=scores_out,
                                 ld_scores=0 if scores_out is None else scores_out.shape[1],
                                 dev_status=buf.dev_status, stream=stream)


def attend(wl: Workload, buf: Buffers, stream=None):
    if wl.H_I:
        sparse_mqa_attn(wl.q, buf.entries, wl.seq_len, wl.ent_off, wl.kv, wl.kv_off, wl.kv_pos0, wl.q_seq,
                        wl.q_pos, buf.idx, wl.sink, buf.out, fmt=wl.fmt, B=wl.B, H=wl.H, D=wl.D,
                        W=wl.W, m=wl.m, k=wl.k, softmax_scale=wl.scale, rope_theta=wl.theta,
                        eps=wl.eps, dev_status=buf.dev_status, stream=stream)
    else:
        dense_hca_attn(wl.q, buf.entries, wl.seq_len, wl.ent_off, wl.kv, wl.kv_off, wl.kv_pos0, wl.q_seq,
                       wl.q_pos, wl.sink, buf.out, buf.workspace, fmt=wl.fmt, B=wl.B, H=wl.H,
                       D=wl.D, W=wl.W, m=wl.m, max_n=buf.max_n, softmax_scale=wl.scale,
                       rope_theta=wl.theta, eps=wl.eps, dev_status=buf.dev_status,
                       stream=stream)


def step(wl: Workload, buf: Buffers, item_seq, item_ent, stream=None):
    """One pass of the hot path: compress the listed entries, select (CSA; the MXFP4
    indexer when the workload carries MXFP4 inputs), attend."""
    compress(wl, buf, item_seq, item_ent, stream)
    if wl.H_I and wl.kI4 is not None:
        indexer_topk_mxfp4(wl, (wl.qI4, wl.qsf4, wl.kI4, wl.ksf4), buf,
                           select_bf16=wl.select_bf16, stream=stream)
    elif wl.H_I:
        indexer_topk(wl, buf, stream=stream)
    attend(wl, buf, stream)
