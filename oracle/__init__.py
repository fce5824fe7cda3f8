"""CPU oracle for hybrid compressed attention (CSA / HCA) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  It is a plain fp64 C restatement of the method
(``csa_oracle.c``) plus this numpy-facing ctypes wrapper.  It shares no code with the CUDA
library and never imports it.

Every wrapper takes numpy arrays holding raw storage bits (bf16 as ``uint16``, e4m3 as
``uint8``) or fp32 / int arrays, exactly as the CUDA library's buffers hold them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_HDR = os.path.join(_HERE, "csa_oracle.h")
_SO = os.path.join(_HERE, "libcsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile csa_oracle.c into libcsa_oracle.so (gcc, OpenMP, no fast-math)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            L.orc_bf16_value.restype = D
            L.orc_bf16_value.argtypes = [ctypes.c_uint16]
            L.orc_bf16_round.restype = ctypes.c_uint16
            L.orc_bf16_round.argtypes = [D]
            L.orc_e4m3_value.restype = D
            L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_round.restype = ctypes.c_uint8
            L.orc_e4m3_round.argtypes = [D]
            L.orc_bf16_round_array.argtypes = [P, I64, P]
            L.orc_e4m3_round_array.argtypes = [P, I64, P]
            L.orc_rope.argtypes = [P, I, D, D]
            L.orc_rmsnorm.argtypes = [P, I, D]
            L.orc_entry_row_bytes.restype = I
            L.orc_entry_row_bytes.argtypes = [I, I]
            L.orc_entry_store.argtypes = [P, I, I, P]
            L.orc_entry_load.argtypes = [P, I, I, P]
            L.orc_compress.restype = I
            L.orc_compress.argtypes = [P, P, P, P, P, P, P, P, I64, I, I, I, I, D, D, P, P]
            L.orc_indexer_topk.restype = I
            L.orc_indexer_topk.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, I64]
            L.orc_e2m1_value.restype = D
            L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
            L.orc_e8m0_value.restype = D
            L.orc_e8m0_value.argtypes = [ctypes.c_uint8]
            L.orc_indexer_topk_mxfp4.restype = I
            L.orc_indexer_topk_mxfp4.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P,
                                                 P, I64]
            L.orc_attention.restype = I
            L.orc_attention.argtypes = [P, P, I, P, P, P, P, P, P, P, I, I, P, I, I, I, I,
                                        D, D, D, P]
            L.orc_num_threads.restype = I
            _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().orc_num_threads()


# ---- number formats -------------------------------------------------------------------
def bf16_value(bits) -> np.ndarray:
    b = _c(bits, np.uint16)
    return np.array([lib().orc_bf16_value(int(x)) for x in b.ravel()]).reshape(b.shape)


def bf16_round(x) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_round_array(_p(x), x.size, _p(out))
    return out


def e4m3_value(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    table = np.array([lib().orc_e4m3_value(v) for v in range(256)])
    return table[c]


def e4m3_round(x) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_round_array(_p(x), x.size, _p(out))
    return out


def e2m1_value(codes) -> np.ndarray:
    """FP4 E2M1 values of the low 4 bits of each code."""
    c = _c(codes, np.uint8)
    table = np.array([lib().orc_e2m1_value(v) for v in range(16)])
    return table[c & 0x0F]


def e8m0_value(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    table = np.array([lib().orc_e8m0_value(v) for v in range(256)])
    return table[c]


# ---- building blocks -----------------------------------------------------------------
def rope(x, pos: float, theta: float = 10000.0) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    lib().orc_rope(_p(y), y.shape[-1], float(pos), float(theta))
    return y


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    lib().orc_rmsnorm(_p(y), y.shape[-1], float(eps))
    return y


def entry_row_bytes(fmt: int, D: int) -> int:
    return lib().orc_entry_row_bytes(fmt, D)


def entry_store(e, fmt: int, D: int) -> np.ndarray:
    e = _c(e, np.float64)
    row = np.zeros(entry_row_bytes(fmt, D), np.uint8)
    lib().orc_entry_store(_p(e), fmt, D, _p(row))
    return row


def entry_load(row, fmt: int, D: int) -> np.ndarray:
    row = _c(row, np.uint8)
    e = np.empty(D, np.float64)
    lib().orc_entry_load(_p(row), fmt, D, _p(e))
    return e


# ---- the steps of the method ---------------------------------------------------------
def compress(kv, gate, bias, kv_off, kv_pos0, ent_off, item_seq, item_ent, *, m: int,
             span: int, D: int, fmt: int = 0, theta: float = 10000.0, eps: float = 1e-6,
             n_entry_rows: int | None = None, entries: np.ndarray | None = None):
    """Compress entries (item_seq[n], item_ent[n]).  Returns (entries rows, fp64 values).

    ``entries`` (uint8 [rows, row_bytes]) is updated in place when given; otherwise a zero
    buffer of ``n_entry_rows`` rows is made.  fp64 values are [n_items, D], before storage
    rounding."""
    kv, gate = _c(kv, np.uint16), _c(gate, np.uint16)
    bias = _c(bias, np.float32)
    kv_off, kv_pos0, ent_off = (_c(a, np.int64) for a in (kv_off, kv_pos0, ent_off))
    item_seq, item_ent = _c(item_seq, np.int32), _c(item_ent, np.int32)
    rb = entry_row_bytes(fmt, D)
    if entries is None:
        if n_entry_rows is None:
            n_entry_rows = int((ent_off[item_seq] + item_ent).max()) + 1 if item_seq.size else 0
        entries = np.zeros((n_entry_rows, rb), np.uint8)
    assert entries.dtype == np.uint8 and entries.flags.c_contiguous
    e64 = np.zeros((item_seq.size, D), np.float64)
    rc = lib().orc_compress(_p(kv), _p(gate), _p(bias), _p(kv_off), _p(kv_pos0), _p(ent_off),
                            _p(item_seq), _p(item_ent), item_seq.size, m, span, D, fmt,
                            float(theta), float(eps), _p(entries), _p(e64))
    if rc != 0:
        raise ValueError(f"orc_compress failed: {rc}")
    return entries, e64


def indexer_topk(qI, qs, w, kI, ks, ent_off, q_seq, q_pos, *, H_I: int, d_I: int, m: int,
                 k: int, want_scores: bool = False, ld_scores: int | None = None):
    """Returns idx int32 [Q, k] (and fp32 scores [Q, ld_scores], NaN where not visible)."""
    qI, kI = _c(qI, np.uint8), _c(kI, np.uint8)
    qs, w, ks = _c(qs, np.float32), _c(w, np.float32), _c(ks, np.float32)
    ent_off = _c(ent_off, np.int64)
    q_seq, q_pos = _c(q_seq, np.int32), _c(q_pos, np.int32)
    Q = q_seq.size
    idx = np.empty((Q, k), np.int32)
    scores = None
    if want_scores:
        if ld_scores is None:
            ld_scores = int(((q_pos.astype(np.int64) + 1) // m).max()) if Q else 0
        scores = np.full((Q, max(ld_scores, 1)), np.nan, np.float32)
    rc = lib().orc_indexer_topk(_p(qI), _p(qs), _p(w), _p(kI), _p(ks), _p(ent_off),
                                _p(q_seq), _p(q_pos), Q, H_I, d_I, m, k, _p(idx),
                                _p(scores), int(ld_scores or 0))
    if rc != 0:
        raise ValueError(f"orc_indexer_topk failed: {rc}")
    return (idx, scores) if want_scores else idx


def indexer_topk_mxfp4(qI, qI_sf, w, kI, kI_sf, ent_off, q_seq, q_pos, *, H_I: int, d_I: int,
                       m: int, k: int, select_bf16: bool = False, want_scores: bool = False,
                       ld_scores: int | None = None):
    """MXFP4 indexer + top-k.  qI uint8 [Q, H_I, d_I/2] packed (element 2j in the low
    nibble), qI_sf uint8 [Q, H_I, d_I/32] (E8M0), kI uint8 [rows, d_I/2], kI_sf uint8
    [rows, d_I/32].  Returns idx int32 [Q, k] (and fp32 scores [Q, ld_scores], NaN where not
    visible; the BF16-rounded values when select_bf16)."""
    qI, qI_sf, kI, kI_sf = (_c(a, np.uint8) for a in (qI, qI_sf, kI, kI_sf))
    w = _c(w, np.float32)
    ent_off = _c(ent_off, np.int64)
    q_seq, q_pos = _c(q_seq, np.int32), _c(q_pos, np.int32)
    Q = q_seq.size
    idx = np.empty((Q, k), np.int32)
    scores = None
    if want_scores:
        if ld_scores is None:
            ld_scores = int(((q_pos.astype(np.int64) + 1) // m).max()) if Q else 0
        scores = np.full((Q, max(ld_scores, 1)), np.nan, np.float32)
    rc = lib().orc_indexer_topk_mxfp4(_p(qI), _p(qI_sf), _p(w), _p(kI), _p(kI_sf), _p(ent_off),
                                      _p(q_seq), _p(q_pos), Q, H_I, d_I, m, k,
                                      1 if select_bf16 else 0, _p(idx), _p(scores),
                                      int(ld_scores or 0))
    if rc != 0:
        raise ValueError(f"orc_indexer_topk_mxfp4 failed: {rc}")
    return (idx, scores) if want_scores else idx


def attention(q, entries, fmt, ent_off, kv, kv_off, kv_pos0, q_seq, q_pos, idx, sink, *,
              H: int, D: int, W: int, m: int, scale: float | None = None,
              theta: float = 10000.0, eps: float = 1e-6) -> np.ndarray:
    """Sparse (idx given, int32 [Q, k]) or dense (idx None) attention; fp64 [Q, H, D]."""
    q = _c(q, np.uint16)
    entries = _c(entries, np.uint8)
    kv = _c(kv, np.uint16)
    ent_off, kv_off, kv_pos0 = (_c(a, np.int64) for a in (ent_off, kv_off, kv_pos0))
    q_seq, q_pos = _c(q_seq, np.int32), _c(q_pos, np.int32)
    sink = _c(sink, np.float32)
    Q = q_seq.size
    k = 0
    if idx is not None:
        idx = _c(idx, np.int32)
        k = idx.shape[1] if idx.ndim == 2 else 0
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((Q, H, D), np.float64)
    rc = lib().orc_attention(_p(q), _p(entries), fmt, _p(ent_off), _p(kv), _p(kv_off),
                             _p(kv_pos0), _p(q_seq), _p(q_pos), _p(idx), k, m, _p(sink), Q,
                             H, D, W, float(scale), float(theta), float(eps), _p(out))
    if rc != 0:
        raise ValueError(f"orc_attention failed: {rc}")
    return out
