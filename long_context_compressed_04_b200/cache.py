"""The hybrid KV cache of one CSA layer for decode ("DeepSeek-V4 深度分析报告" 3.5, KV cache
management).

- State cache: a fixed-size ring of ``ring`` raw-token rows per sequence (the sliding
  window's KV and the tokens the next entry pools); token p of sequence b sits in row
  b * ring + p mod ring.
- Classical cache: compressed entries (and their indexer keys) in blocks of 128 tokens, i.e.
  32 CSA entries; a block table maps each sequence's blocks to physical blocks, which a
  free list hands out as entries complete.

A decode step appends one token per sequence (``csa_cache_append``: ring row, and the
indexer key of an entry the token completes), compresses the entries completed this step
from the ring into their blocks (``csa_compress``), selects (``lightning_indexer_topk``) and
attends (``sparse_mqa_attn``), every call with the same cache layout.  This module keeps the
host-side bookkeeping (block allocation, the item lists of completed entries); every copy,
compression, score, selection and attention runs in libcsa.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from . import (CSA_KV_BF16, cache_layout, csa_cache_append, csa_compress, csa_entry_row_bytes,
               csa_indexer_workspace_size, lightning_indexer_topk, sparse_mqa_attn)

BLOCK_TOKENS = 128      # lcm(m, m') of the pages
M = 4                   # CSA compression ratio
BLOCK_ENTRIES = BLOCK_TOKENS // M


class BlockAllocator:
    """Free list of classical-cache blocks."""

    def __init__(self, n_blocks: int):
        self.free: List[int] = list(range(n_blocks - 1, -1, -1))

    def alloc(self) -> int:
        if not self.free:
            raise RuntimeError("classical cache full")
        return self.free.pop()

    def release(self, blocks):
        self.free.extend(int(x) for x in blocks)


class HybridCache:
    """Device buffers and bookkeeping of one CSA layer's cache for B decode sequences."""

    def __init__(self, B: int, D: int, fmt: int, d_I: int, n_blocks: int, max_blocks: int,
                 ring: int = 128, device="cuda"):
        self.B, self.D, self.fmt, self.d_I, self.ring = B, D, fmt, d_I, ring
        dev = torch.device(device)
        self.device = dev
        rb = csa_entry_row_bytes(fmt, D)
        rows = n_blocks * BLOCK_ENTRIES
        self.kv = torch.zeros((B * ring, D), dtype=torch.bfloat16, device=dev)
        self.gate = torch.zeros((B * ring, D), dtype=torch.bfloat16, device=dev)
        self.kv_off = torch.arange(B, dtype=torch.int64, device=dev) * ring
        self.entries = torch.zeros((rows, rb), dtype=torch.uint8, device=dev)
        self.kI = torch.zeros((rows, d_I), dtype=torch.uint8, device=dev)
        self.ks = torch.zeros(rows, dtype=torch.float32, device=dev)
        self.block_table = torch.full((B, max_blocks), -1, dtype=torch.int32, device=dev)
        self.bt_host = torch.full((B, max_blocks), -1, dtype=torch.int32)
        self.seq_len = torch.zeros(B, dtype=torch.int64, device=dev)
        self.len_host = [0] * B
        self.alloc = BlockAllocator(n_blocks)
        self.layout = cache_layout(self.block_table, kv_ring=ring)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=dev)

    # ---- bookkeeping ---------------------------------------------------------------
    def _ensure_blocks(self, b: int, n_entries: int):
        need = (n_entries + BLOCK_ENTRIES - 1) // BLOCK_ENTRIES
        changed = False
        for j in range(need):
            if int(self.bt_host[b, j]) < 0:
                self.bt_host[b, j] = self.alloc.alloc()
                changed = True
        return changed

    def _push_table(self):
        self.block_table.copy_(self.bt_host, non_blocking=False)

    def release(self, b: int):
        """Frees sequence b's blocks (the sequence ends)."""
        blocks = [int(x) for x in self.bt_host[b] if int(x) >= 0]
        self.alloc.release(blocks)
        self.bt_host[b] = -1
        self.len_host[b] = 0
        self._push_table()
        self.seq_len[b] = 0

    # ---- loading a prefix (set-up) -----------------------------------------------
    def load_prefix(self, b: int, kv_tail, gate_tail, T: int, entries, kI, ks):
        """Sequence b with T tokens: the last min(T, ring) raw rows (kv_tail, gate_tail, in
        position order), its T // 4 entry rows, indexer keys and scales (in entry order)."""
        n = T // M
        self._ensure_blocks(b, n)
        self._push_table()
        t0 = T - kv_tail.shape[0]
        slots = (torch.arange(t0, T) % self.ring) + b * self.ring
        self.kv[slots.to(self.device)] = kv_tail
        self.gate[slots.to(self.device)] = gate_tail
        i = torch.arange(n)
        rows = (self.bt_host[b, i // BLOCK_ENTRIES].to(torch.int64) * BLOCK_ENTRIES
                + i % BLOCK_ENTRIES).to(self.device)
        self.entries[rows] = entries
        self.kI[rows] = kI
        self.ks[rows] = ks
        self.seq_len[b] = T
        self.len_host[b] = T

    # ---- one decode step -----------------------------------------------------------
    def append(self, kv_new, gate_new, kI_new, ks_new, stream=None):
        """One token per sequence (bf16 [B, D] raw KV and gate; e4m3 [B, d_I] indexer key and
        fp32 [B] scale, used by the sequences whose token completes an entry).  Returns the
        (item_seq, item_ent) lists of the entries completed, for compress()."""
        changed = False
        for b in range(self.B):
            changed |= self._ensure_blocks(b, (self.len_host[b] + 1) // M)
        if changed:
            self._push_table()
        csa_cache_append(kv_new, gate_new, self.seq_len, self.kv_off, None, self.kv, self.gate,
                         B=self.B, D=self.D, m=M, kI_new=kI_new, kI_scale_new=ks_new,
                         kI=self.kI, kI_scale=self.ks, layout=self.layout,
                         dev_status=self.dev_status, stream=stream)
        seqs, ents = [], []
        for b in range(self.B):
            self.len_host[b] += 1
            if self.len_host[b] % M == 0:
                seqs.append(b)
                ents.append(self.len_host[b] // M - 1)
        return (torch.tensor(seqs, dtype=torch.int32, device=self.device),
                torch.tensor(ents, dtype=torch.int32, device=self.device))

    def compress(self, items, bias, rope_theta=10000.0, eps=1e-6, stream=None):
        seq, ent = items
        if seq.numel() == 0:
            return
        csa_compress(self.kv, self.gate, bias, self.seq_len, self.kv_off, None, None, seq, ent,
                     self.entries, B=self.B, D=self.D, fmt=self.fmt, rope_theta=rope_theta,
                     eps=eps, layout=self.layout, dev_status=self.dev_status, stream=stream)

    def select(self, qI, qs, w, q_seq, q_pos, idx_out, *, H_I: int, k: int,
               workspace: Optional[torch.Tensor] = None, stream=None):
        max_n = max(self.len_host) // M
        if workspace is None:
            workspace = torch.empty(max(csa_indexer_workspace_size(q_seq.numel(), max(max_n, 1), k), 256),
                                    dtype=torch.uint8, device=self.device)
        lightning_indexer_topk(qI, qs, w, self.kI, self.ks, self.seq_len, None, q_seq, q_pos,
                               idx_out, workspace, B=self.B, H_I=H_I, d_I=self.d_I, m=M, k=k,
                               max_n=max(max_n, 1), layout=self.layout,
                               dev_status=self.dev_status, stream=stream)

    def attend(self, q, q_seq, q_pos, idx, sink, out, *, H: int, W: int, k: int,
               softmax_scale: float, rope_theta=10000.0, eps=1e-6, stream=None):
        sparse_mqa_attn(q, self.entries, self.seq_len, None, self.kv, self.kv_off, None, q_seq,
                        q_pos, idx, sink, out, fmt=self.fmt, B=self.B, H=H, D=self.D, W=W, m=M,
                        k=k, softmax_scale=softmax_scale, rope_theta=rope_theta, eps=eps,
                        layout=self.layout, dev_status=self.dev_status, stream=stream)


__all__ = ["BlockAllocator", "HybridCache", "BLOCK_TOKENS", "BLOCK_ENTRIES", "CSA_KV_BF16"]
