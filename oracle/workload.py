"""Workload-level wrappers of the oracle: take the host copies of a synthetic workload's
tensors and run the oracle's steps on them.  TEST INFRASTRUCTURE ONLY (tests/, the smoke
check and the benchmark's CPU-baseline and reference legs)."""
from __future__ import annotations

import numpy as np
import torch

from . import attention as _attention
from . import compress as _compress
from . import indexer_topk as _indexer_topk
from . import indexer_topk_mxfp4 as _indexer_topk_mxfp4


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().to(torch.float32).numpy()


def i64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().to(torch.int64).numpy()


def i32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().to(torch.int32).numpy()


def compress(wl, item_seq=None, item_ent=None, entries=None):
    """Oracle compression of the listed entries (default: all).  Returns (rows, fp64)."""
    if item_seq is None:
        n = i64(wl.n_ent)
        item_seq = np.repeat(np.arange(wl.B, dtype=np.int32), n)
        item_ent = np.concatenate([np.arange(x, dtype=np.int32) for x in n])
    return _compress(u16(wl.kv), u16(wl.gate), f32(wl.bias), i64(wl.kv_off),
                           i64(wl.kv_pos0), i64(wl.ent_off), np.asarray(item_seq, np.int32),
                           np.asarray(item_ent, np.int32), m=wl.m, span=wl.span, D=wl.D,
                           fmt=wl.fmt, theta=wl.theta, eps=wl.eps,
                           n_entry_rows=max(wl.ent_rows, 1), entries=entries)


def indexer(wl, want_scores=True):
    max_n = int(((i64(wl.q_pos) + 1) // wl.m).max())
    return _indexer_topk(u8(wl.qI), f32(wl.qs), f32(wl.w), u8(wl.kI), f32(wl.ks),
                               i64(wl.ent_off), i32(wl.q_seq), i32(wl.q_pos), H_I=wl.H_I,
                               d_I=wl.d_I, m=wl.m, k=wl.k, want_scores=want_scores,
                               ld_scores=max(max_n, 1))


def indexer_mxfp4(wl, fp4, select_bf16=False, want_scores=True):
    """The MXFP4 indexer on `wl`'s queries; fp4 = (qI, qI_sf, kI, kI_sf) as the synthetic
    generator lays them out."""
    qI, qsf, kI, ksf = fp4
    max_n = int(((i64(wl.q_pos) + 1) // wl.m).max())
    return _indexer_topk_mxfp4(u8(qI), u8(qsf), f32(wl.w), u8(kI), u8(ksf),
                               i64(wl.ent_off), i32(wl.q_seq), i32(wl.q_pos),
                               H_I=wl.H_I, d_I=wl.d_I, m=wl.m, k=wl.k,
                               select_bf16=select_bf16, want_scores=want_scores,
                               ld_scores=max(max_n, 1))


def attention(wl, entries_rows: np.ndarray, idx):
    return _attention(u16(wl.q), entries_rows, wl.fmt, i64(wl.ent_off), u16(wl.kv),
                            i64(wl.kv_off), i64(wl.kv_pos0), i32(wl.q_seq), i32(wl.q_pos),
                            None if idx is None else np.asarray(idx, np.int32), f32(wl.sink),
                            H=wl.H, D=wl.D, W=wl.W, m=wl.m, scale=wl.scale, theta=wl.theta,
                            eps=wl.eps)
