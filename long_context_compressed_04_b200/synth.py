"""Seeded synthetic workloads for the CSA / HCA hot path.

This module only draws random inputs and lays them out in the library's buffer formats.
It holds none of the method's arithmetic (no pooling, normalisation, RoPE, scoring,
selection or attention); both the CUDA library's tests/benchmarks and the CPU oracle
consume the tensors it returns.

Distributions follow the workloads the method is specified on: raw per-token KV and gate
logits ~N(0,1) stored as bf16, positional bias ~N(0, 0.1) fp32, attention-sink logits
~N(0,1) per head, queries ~N(0,1) bf16, indexer heads in FP8 E4M3 -- either
integer-valued in [-3, 3] with unit scales (exact-arithmetic runs) or N(0,1) quantised
with one scale per 1x128 row -- and per-head indexer weights ~U(0,1).  MXFP4 indexer
inputs (packed e2m1 + UE8M0 block scales) are drawn either as uniform codes with scales
near 1 or as N(0,1) values quantised per 32-element block.

Random numbers come from ``torch.Generator`` seeded per workload, on the device the
tensors are made on; a given (workload, seed, device) always yields the same tensors.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

E4M3 = torch.float8_e4m3fn


@dataclasses.dataclass
class Workload:
    """Inputs of one hot-path pass.  Integer offsets are int64, positions int32."""
    name: str
    B: int                      # sequences
    T: torch.Tensor             # [B] int64 context lengths (host tensor)
    D: int                      # head dim (RoPE on the last 64)
    H: int                      # query heads
    m: int                      # compression ratio used for visibility (4 CSA, 128 HCA)
    span: int                   # tokens pooled per entry (2m CSA, m' HCA)
    W: int                      # sliding window
    fmt: int                    # entry storage format: 0 bf16, 1 = 576-dim fp8 + bf16 rope
    # raw per-token data: position p of sequence b sits in row kv_off[b] + p - kv_pos0[b]
    kv: torch.Tensor            # [rows, D] bf16
    gate: torch.Tensor          # [rows, D] bf16
    kv_off: torch.Tensor        # [B] int64
    kv_pos0: torch.Tensor       # [B] int64
    bias: torch.Tensor          # [span, D] fp32
    # compressed entries: entry i of sequence b is row ent_off[b] + i
    ent_off: torch.Tensor       # [B] int64
    n_ent: torch.Tensor         # [B] int64 = floor(T_b / m)
    # queries
    q_seq: torch.Tensor         # [Q] int32
    q_pos: torch.Tensor         # [Q] int32
    q: torch.Tensor             # [Q, H, D] bf16
    sink: torch.Tensor          # [H] fp32
    # lightning indexer (CSA only; None for HCA)
    H_I: int = 0
    d_I: int = 0
    k: int = 0
    kI: Optional[torch.Tensor] = None   # [ent_rows, d_I] uint8 (e4m3 codes)
    ks: Optional[torch.Tensor] = None   # [ent_rows] fp32
    qI: Optional[torch.Tensor] = None   # [Q, H_I, d_I] uint8
    qs: Optional[torch.Tensor] = None   # [Q, H_I] fp32
    w: Optional[torch.Tensor] = None    # [Q, H_I] fp32
    # MXFP4 indexer inputs (instead of kI / ks / qI / qs when set; see mxfp4_indexer)
    kI4: Optional[torch.Tensor] = None   # [ent_rows, d_I / 2] uint8 (packed e2m1)
    ksf4: Optional[torch.Tensor] = None  # [ent_rows, d_I / 32] uint8 (UE8M0)
    qI4: Optional[torch.Tensor] = None   # [Q, H_I, d_I / 2] uint8
    qsf4: Optional[torch.Tensor] = None  # [Q, H_I, d_I / 32] uint8
    select_bf16: bool = False            # MXFP4 path: select on BF16-rounded scores
    theta: float = 10000.0
    eps: float = 1e-6

    @property
    def seq_len(self) -> torch.Tensor:
        """[B] int64 context lengths on the workload's device."""
        if getattr(self, "_seq_len", None) is None or self._seq_len.device != self.kv.device:
            self._seq_len = self.T.to(self.kv.device)
        return self._seq_len

    @property
    def Q(self) -> int:
        return int(self.q_seq.numel())

    @property
    def ent_rows(self) -> int:
        return int(self.n_ent.sum())

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def to(self, device) -> "Workload":
        f = {}
        for fld in dataclasses.fields(self):
            v = getattr(self, fld.name)
            if isinstance(v, torch.Tensor) and fld.name != "T":
                v = v.to(device)
            f[fld.name] = v
        return Workload(**f)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _bf16_normal(shape, g, device, std=1.0):
    return (torch.randn(shape, generator=g, device=device) * std).to(torch.bfloat16)


def fp8_integer(shape, g, device, lo=-3, hi=3):
    """E4M3 codes of integers drawn uniformly from [lo, hi] (exact in e4m3)."""
    x = torch.randint(lo, hi + 1, shape, generator=g, device=device).to(torch.float32)
    return x.to(E4M3).view(torch.uint8)


def fp8_rows_from_normal(rows, cols, g, device):
    """N(0,1) rows quantised to E4M3 with one fp32 scale per row (amax / 448)."""
    x = torch.randn((rows, cols), generator=g, device=device)
    amax = x.abs().amax(dim=1).clamp_min(1e-12)
    scale = (amax / 448.0).to(torch.float32)
    codes = (x / scale[:, None]).clamp(-448.0, 448.0).to(E4M3).view(torch.uint8)
    return codes, scale


def random_entries(n, fmt, D, g, device):
    """Random stored entry rows (used where entries are generated directly, e.g. for
    neighbour sequences).  fmt 0: bf16 N(0,1).  fmt 1 (D=576): e4m3 codes of N(0,1)
    quantised per 128 channels, the 4 fp32 scales, then 64 bf16 N(0,1) values."""
    if fmt == 0:
        return _bf16_normal((n, D), g, device).view(torch.uint8).reshape(n, 2 * D)
    assert fmt == 1 and D == 576
    x = torch.randn((n, 4, 128), generator=g, device=device)
    amax = x.abs().amax(dim=2).clamp_min(1e-12)
    scale = (amax / 448.0).to(torch.float32)
    codes = (x / scale[:, :, None]).clamp(-448.0, 448.0).to(E4M3).view(torch.uint8)
    rope = _bf16_normal((n, 64), g, device)
    row = torch.empty((n, 656), dtype=torch.uint8, device=device)
    row[:, :512] = codes.reshape(n, 512)
    row[:, 512:528] = scale.view(torch.uint8).reshape(n, 16)
    row[:, 528:] = rope.view(torch.uint8).reshape(n, 128)
    return row


def _offsets(lengths: torch.Tensor) -> torch.Tensor:
    off = torch.zeros(lengths.numel(), dtype=torch.int64)
    if lengths.numel() > 1:
        off[1:] = torch.cumsum(lengths[:-1], 0)
    return off


def make_workload(name: str, *, B: int, T, D: int, H: int, m: int, span: int, W: int = 128,
                  fmt: int = 0, H_I: int = 0, d_I: int = 0, k: int = 0,
                  indexer: str = "int", keep_raw: Optional[int] = None,
                  queries: str = "decode", n_new: int = 0, seed: int = 0,
                  device="cpu") -> Workload:
    """Draw one workload.

    T: int or list of context lengths.  queries="decode": one query per sequence at
    position T_b - 1.  queries="prefill": the last ``n_new`` positions of every sequence.
    keep_raw: store only the last ``keep_raw`` raw tokens of each sequence (None = all).
    indexer: "int" (integers in [-3,3], unit scales) or "fp8" (N(0,1), 1x128 scales).
    """
    g = _gen(seed, device)
    T = torch.as_tensor(T if not isinstance(T, int) else [T] * B, dtype=torch.int64)
    assert T.numel() == B
    keep = T.clone() if keep_raw is None else torch.minimum(T, torch.tensor(keep_raw))
    kv_pos0 = T - keep
    kv_off = _offsets(keep)
    rows = int(keep.sum())
    kv = _bf16_normal((rows, D), g, device)
    gate = _bf16_normal((rows, D), g, device)
    bias = torch.randn((span, D), generator=g, device=device) * 0.1
    n_ent = T // m
    ent_off = _offsets(n_ent)
    if queries == "decode":
        q_seq = torch.arange(B, dtype=torch.int32)
        q_pos = (T - 1).to(torch.int32)
    else:
        q_seq = torch.arange(B, dtype=torch.int32).repeat_interleave(n_new)
        q_pos = torch.cat([torch.arange(int(t) - n_new, int(t), dtype=torch.int32) for t in T])
    Q = q_seq.numel()
    q = _bf16_normal((Q, H, D), g, device)
    sink = torch.randn((H,), generator=g, device=device)
    wl = Workload(name=name, B=B, T=T, D=D, H=H, m=m, span=span, W=W, fmt=fmt, kv=kv,
                  gate=gate, kv_off=kv_off.to(device), kv_pos0=kv_pos0.to(device), bias=bias,
                  ent_off=ent_off.to(device), n_ent=n_ent.to(device),
                  q_seq=q_seq.to(device), q_pos=q_pos.to(device), q=q, sink=sink)
    if H_I:
        er = int(n_ent.sum())
        if indexer == "int":
            kI = fp8_integer((er, d_I), g, device)
            ks = torch.ones(er, dtype=torch.float32, device=device)
            qI = fp8_integer((Q, H_I, d_I), g, device)
            qs = torch.ones((Q, H_I), dtype=torch.float32, device=device)
        else:
            kI, ks = fp8_rows_from_normal(er, d_I, g, device)
            qI, qs = fp8_rows_from_normal(Q * H_I, d_I, g, device)
            qI = qI.reshape(Q, H_I, d_I)
            qs = qs.reshape(Q, H_I)
        w = torch.rand((Q, H_I), generator=g, device=device)
        wl.H_I, wl.d_I, wl.k = H_I, d_I, k
        wl.kI, wl.ks, wl.qI, wl.qs, wl.w = kI, ks, qI, qs, w
    return wl


def jittered_lengths(B: int, T: int, jitter: int, seed: int) -> list:
    g = torch.Generator().manual_seed(int(seed) + 7919)
    return (T + torch.randint(-jitter, jitter + 1, (B,), generator=g)).tolist()


# ---- the named workloads -------------------------------------------------------------
def csa_decode_4k(device="cpu", seed=0, indexer="int") -> Workload:
    """CSA single layer, decode, batch 1, 4096 tokens -> 1024 entries; indexer 4 heads x 64,
    top-64; 16 query heads, head dim 128; window 128."""
    return make_workload("csa_decode_4k_b1", B=1, T=4096, D=128, H=16, m=4, span=8, W=128,
                         H_I=4, d_I=64, k=64, indexer=indexer, seed=seed, device=device)


def csa_decode_128k(device="cpu", seed=0, indexer="int", B=32, keep_raw=None) -> Workload:
    """CSA decode, 32 sequences of 131072 +- 1024 tokens; 64 heads, head dim 128; indexer
    64 heads x 128 FP8; top-512; window 128."""
    return make_workload("csa_decode_128k_b32", B=B, T=jittered_lengths(B, 131072, 1024, seed),
                         D=128, H=64, m=4, span=8, W=128, H_I=64, d_I=128, k=512,
                         indexer=indexer, keep_raw=keep_raw, seed=seed, device=device)


def hca_decode_1m(device="cpu", seed=0, B=16, keep_raw=None) -> Workload:
    """HCA decode, 16 sequences of 1,048,576 tokens -> 8192 entries each; dense attention
    plus window 128; 64 heads, head dim 128."""
    return make_workload("hca_decode_1m_b16", B=B, T=1 << 20, D=128, H=64, m=128, span=128,
                         W=128, keep_raw=keep_raw, seed=seed, device=device)


def csa_prefill_64k(device="cpu", seed=0, indexer="int") -> Workload:
    """CSA prefill chunk: 8192 new query tokens after 65536 prior tokens (18432 entries);
    indexer 64 x 128 FP8, top-1024; 64 heads, head dim 128; window 128."""
    return make_workload("csa_prefill_8k_on_64k", B=1, T=65536 + 8192, D=128, H=64, m=4,
                         span=8, W=128, H_I=64, d_I=128, k=1024, indexer=indexer,
                         queries="prefill", n_new=8192, seed=seed, device=device)


def csa_decode_1m_fp8(device="cpu", seed=0, indexer="int", B=8, keep_raw=None) -> Workload:
    """CSA decode at 1,048,576 tokens, batch 8, top-1024, 128 query heads, entries of head
    dim 576 stored as 512 FP8 (1x128 scales) + 64 BF16 RoPE dims; indexer 64 x 128 FP8."""
    return make_workload("csa_decode_1m_b8_fp8", B=B, T=1 << 20, D=576, H=128, m=4, span=8,
                         W=128, fmt=1, H_I=64, d_I=128, k=1024, indexer=indexer,
                         keep_raw=keep_raw, seed=seed, device=device)


# ---- MXFP4 indexer inputs -----------------------------------------------------------
# Packed e2m1 codes (element 2j in the low nibble) and one UE8M0 scale byte per 32
# elements, the layout lightning_indexer_topk_mxfp4 reads.

# e2m1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7); the midpoints between them
_E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _pack_nibbles(codes: torch.Tensor) -> torch.Tensor:
    c = codes.to(torch.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).contiguous()


def mxfp4_integer(rows, cols, g, device, exp_lo=126, exp_hi=128):
    """Uniformly drawn e2m1 codes and block exponents in [exp_lo, exp_hi] (scales 2^-1 ..
    2^1 by default): every block dot product and their sums are exact in fp32.
    Returns (packed uint8 [rows, cols / 2], scales uint8 [rows, cols / 32])."""
    codes = torch.randint(0, 16, (rows, cols), generator=g, device=device)
    sf = torch.randint(exp_lo, exp_hi + 1, (rows, cols // 32), generator=g, device=device)
    return _pack_nibbles(codes), sf.to(torch.uint8).contiguous()


def mxfp4_from_normal(rows, cols, g, device):
    """N(0,1) values quantised to MXFP4 the usual way: per block of 32 the scale exponent is
    floor(log2(amax)) - 2 (the largest e2m1 exponent), each value divided by the scale goes
    to the nearest e2m1 magnitude (saturating at 6; exact midpoints, of probability zero,
    go up).  Returns (packed uint8 [rows, cols / 2], scales uint8 [rows, cols / 32])."""
    x = torch.randn((rows, cols // 32, 32), generator=g, device=device)
    amax = x.abs().amax(dim=2).clamp_min(2.0 ** -100)
    e = torch.floor(torch.log2(amax)) - 2
    y = x / torch.exp2(e)[:, :, None]
    mids = torch.tensor(_E2M1_MIDPOINTS, device=device)
    mag = torch.bucketize(y.abs().contiguous(), mids, right=True)
    codes = mag | ((y < 0).to(mag.dtype) << 3)
    sf = (e + 127).clamp(0, 254).to(torch.uint8)
    return _pack_nibbles(codes.reshape(rows, cols)), sf.contiguous()


def mxfp4_indexer(wl: Workload, kind: str = "int", seed: int = 0):
    """MXFP4 query heads and keys for `wl`'s indexer shapes ("int": mxfp4_integer, "normal":
    mxfp4_from_normal).  Returns (qI [Q, H_I, d_I / 2], qI_sf [Q, H_I, d_I / 32],
    kI [ent_rows, d_I / 2], kI_sf [ent_rows, d_I / 32]); the head weights stay wl.w."""
    dev = wl.q.device
    g = _gen(seed * 7919 + 4, dev)
    make = mxfp4_integer if kind == "int" else mxfp4_from_normal
    kI, ksf = make(max(wl.ent_rows, 1), wl.d_I, g, dev)
    qI, qsf = make(wl.Q * wl.H_I, wl.d_I, g, dev)
    return (qI.reshape(wl.Q, wl.H_I, wl.d_I // 2), qsf.reshape(wl.Q, wl.H_I, wl.d_I // 32),
            kI, ksf)


# ---- re-batching (for batch-invariance runs) -----------------------------------------
def split(wl: Workload) -> list:
    """One single-sequence workload per sequence of ``wl`` (same tensors, re-based)."""
    out = []
    T = wl.T.cpu()
    kv_off, kv_pos0 = wl.kv_off.cpu(), wl.kv_pos0.cpu()
    ent_off, n_ent = wl.ent_off.cpu(), wl.n_ent.cpu()
    q_seq = wl.q_seq.cpu()
    for b in range(wl.B):
        r0, nr = int(kv_off[b]), int(T[b] - kv_pos0[b])
        e0, ne = int(ent_off[b]), int(n_ent[b])
        qsel = torch.nonzero(q_seq == b).flatten().to(wl.q.device)
        z = torch.zeros(1, dtype=torch.int64, device=wl.kv_off.device)
        f = dict(name=wl.name, B=1, T=T[b:b + 1].clone(), D=wl.D, H=wl.H, m=wl.m, span=wl.span,
                 W=wl.W, fmt=wl.fmt, kv=wl.kv[r0:r0 + nr], gate=wl.gate[r0:r0 + nr],
                 kv_off=z.clone(), kv_pos0=wl.kv_pos0[b:b + 1].clone(), bias=wl.bias,
                 ent_off=z.clone(), n_ent=wl.n_ent[b:b + 1].clone(),
                 q_seq=torch.zeros(qsel.numel(), dtype=torch.int32, device=wl.q_seq.device),
                 q_pos=wl.q_pos[qsel], q=wl.q[qsel], sink=wl.sink, H_I=wl.H_I, d_I=wl.d_I,
                 k=wl.k, theta=wl.theta, eps=wl.eps)
        if wl.H_I:
            f.update(kI=wl.kI[e0:e0 + ne], ks=wl.ks[e0:e0 + ne], qI=wl.qI[qsel], qs=wl.qs[qsel],
                     w=wl.w[qsel])
        out.append(Workload(**f))
    return out


def merge(parts: list) -> Workload:
    """Concatenate single- or multi-sequence workloads (same shapes) into one batch."""
    p0 = parts[0]
    dev = p0.kv.device
    Ts, kv_off, kv_pos0, ent_off, n_ent, q_seq = [], [], [], [], [], []
    rows = ents = seqs = 0
    for p in parts:
        for b in range(p.B):
            Ts.append(int(p.T[b]))
            kv_off.append(rows + int(p.kv_off[b]))
            kv_pos0.append(int(p.kv_pos0[b]))
            ent_off.append(ents + int(p.ent_off[b]))
            n_ent.append(int(p.n_ent[b]))
        q_seq.append(p.q_seq.to(torch.int64) + seqs)
        rows += p.kv.shape[0]
        ents += int(p.n_ent.sum())
        seqs += p.B
    cat = lambda name: torch.cat([getattr(p, name) for p in parts])  # noqa: E731
    as_dev = lambda v: torch.tensor(v, dtype=torch.int64, device=dev)  # noqa: E731
    f = dict(name=p0.name, B=seqs, T=torch.tensor(Ts, dtype=torch.int64), D=p0.D, H=p0.H,
             m=p0.m, span=p0.span, W=p0.W, fmt=p0.fmt, kv=cat("kv"), gate=cat("gate"),
             kv_off=as_dev(kv_off), kv_pos0=as_dev(kv_pos0), bias=p0.bias,
             ent_off=as_dev(ent_off), n_ent=as_dev(n_ent),
             q_seq=torch.cat(q_seq).to(torch.int32), q_pos=cat("q_pos"), q=cat("q"),
             sink=p0.sink, H_I=p0.H_I, d_I=p0.d_I, k=p0.k, theta=p0.theta, eps=p0.eps)
    if p0.H_I:
        f.update(kI=cat("kI"), ks=cat("ks"), qI=cat("qI"), qs=cat("qs"), w=cat("w"))
    return Workload(**f)
