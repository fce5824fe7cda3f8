"""Hybrid compressed attention (CSA / HCA) on B200: Python binding of libcsa.

Argument marshalling only: every function here passes tensor pointers, sizes and the
current CUDA stream to the C ABI of ``libcsa.so`` (declared in ``include/csa.h``) and raises
``CSAError`` when it returns a non-zero status.  All computation happens in the CUDA
kernels.  There is no CPU fallback: importing this package fails if ``libcsa.so`` has not
been built (``python long_context_compressed_04_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_KV_BF16 = 0
CSA_KV_FP8_576 = 1
CSA_DEV_OOB = 1
CSA_DEV_TIMEOUT = 2
CSA_DEV_NAN = 4
CSA_DEV_CAPACITY = 8

STATUS_NAMES = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED",
                3: "CSA_ERR_CUDA", 4: "CSA_ERR_WORKSPACE"}


class CSAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python long_context_compressed_04_b200/build.py` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)
_P, _I32, _I64, _F32, _SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
_SIGS = {
    "csa_version": (ctypes.c_int, []),
    "csa_last_error": (ctypes.c_char_p, []),
    "csa_entry_row_bytes": (_I32, [_I32, _I32]),
    "csa_compress": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I32, _I32, _I32,
                                    _F32, _F32, _P, _P, _P, _P]),
    "hca_compress": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I32, _I32, _I32,
                                    _F32, _F32, _P, _P, _P, _P]),
    "csa_indexer_workspace_size": (_SZ, [_I32, _I32, _I32]),
    "lightning_indexer_topk": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _I32, _I32, _I32,
                                              _I32, _I32, _I32, _I32, _P, _P, _I64, _P, _SZ, _P,
                                              _P, _P]),
    "sparse_mqa_attn": (ctypes.c_int, [_P, _P, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _P,
                                       _I32, _I32, _I32, _I32, _I32, _F32, _F32, _F32, _P, _P,
                                       _P, _P]),
    "dense_hca_workspace_size": (_SZ, [_I32, _I32, _I32, _I32]),
    "dense_hca_attn": (ctypes.c_int, [_P, _P, _I32, _I64, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32,
                                      _I32, _I32, _I32, _F32, _F32, _F32, _I32, _P, _P, _SZ, _P,
                                      _P, _P]),
    "lightning_indexer_topk_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _P, _P, _P, _P,
                                                      _I32,
                                                      _I32, _I32, _I32, _I32, _I32, _I32, _P, _P,
                                                      _I64, _P, _P]),
    "csa_launch_count": (ctypes.c_longlong, []),
    "csa_profile_enable": (None, [ctypes.c_int]),
    "csa_profile_collect": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int]),
    "csa_debug_set_wait_limit": (ctypes.c_int, [ctypes.c_longlong]),
    "lightning_indexer_topk_mxfp4": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _P, _P, _P, _P,
                                                    _I32, _I32, _I32, _I32, _I32, _I32, _I32,
                                                    _I32, _P, _P, _I64, _P, _SZ, _P, _P, _P]),
    "csa_cache_append": (ctypes.c_int, [_P, _P, _P, _P, _I32, _P, _P, _P, _I64, _P, _I64, _I32,
                                        _I32, _I32, _P, _P, _P, _P, _P, _P, _P]),
    "csa_topk_merge": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P]),
    "csa_cp_candidates": (ctypes.c_int, [_P, _P, _I64, _P, _P, _I32, _I32, _I32, _P, _P, _P,
                                         _P]),
    "csa_cp_pack_rows": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _I32, _I32, _I32, _I32,
                                        _P, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


class CacheLayout(ctypes.Structure):
    """csa_cache_layout_t (see include/csa.h): the classical cache's block table and the
    state cache's ring size."""
    _fields_ = [("block_table", ctypes.c_void_p), ("bt_stride", ctypes.c_int64),
                ("kv_ring", ctypes.c_int64)]


def cache_layout(block_table=None, kv_ring: int = 0):
    """A cache layout for the calls' ``layout`` argument, or None for the contiguous one.
    block_table: int32 [B, bt_stride] device tensor (blocks of 32 CSA entries); kv_ring:
    rows of each sequence's state-cache ring (0 = linear raw store)."""
    if block_table is None and not kv_ring:
        return None
    lay = CacheLayout(None if block_table is None else block_table.data_ptr(),
                      0 if block_table is None else block_table.stride(0), int(kv_ring))
    lay._block_table = block_table      # keeps the tensor alive with the struct
    return lay


def _lay(layout):
    return None if layout is None else ctypes.byref(layout)


def _p(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int):
    if status != 0:
        raise CSAError(status, _lib.csa_last_error().decode())


class _KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("launches", ctypes.c_longlong),
                ("total_ms", ctypes.c_double)]


def csa_launch_count() -> int:
    return _lib.csa_launch_count()


def csa_profile_enable(on: bool = True):
    _lib.csa_profile_enable(1 if on else 0)


def csa_profile_collect(keep_pending: bool = False) -> dict:
    """{kernel name: (timed launches, total device ms)} since the last collect.  With
    keep_pending, the recorded event pairs stay registered (for CUDA-graph replays)."""
    arr = (_KernelTime * 32)()
    n = _lib.csa_profile_collect(ctypes.cast(arr, ctypes.c_void_p), 32, 1 if keep_pending else 0)
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n)}


def csa_debug_set_wait_limit(cycles: int = 0):
    """Test hook: limit (SM clocks) of the kernels' bounded waits; 0 restores the default.
    Synchronous; call it with no libcsa kernel in flight and outside stream capture."""
    _check(_lib.csa_debug_set_wait_limit(int(cycles)))


def csa_version() -> int:
    return _lib.csa_version()


def csa_entry_row_bytes(fmt: int, D: int) -> int:
    return _lib.csa_entry_row_bytes(fmt, D)


def csa_indexer_workspace_size(Q: int, max_n: int, k: int) -> int:
    return _lib.csa_indexer_workspace_size(Q, max_n, k)


def dense_hca_workspace_size(Q: int, H: int, D: int, max_n: int) -> int:
    return _lib.dense_hca_workspace_size(Q, H, D, max_n)


def csa_compress(kv, gate, pos_bias, seq_len, kv_off, kv_pos0, ent_off, item_seq, item_ent,
                 entries, *,
                 B: int, D: int, fmt: int = CSA_KV_BF16, rope_theta: float = 10000.0,
                 eps: float = 1e-6, layout=None, dev_status=None, stream=None):
    _check(_lib.csa_compress(_p(kv), _p(gate), _p(pos_bias), _p(seq_len), _p(kv_off), _p(kv_pos0),
                             _p(ent_off), _p(item_seq), _p(item_ent), item_seq.numel(), B, D, fmt,
                             rope_theta, eps, _p(entries), _lay(layout), _p(dev_status),
                             _s(stream)))


def hca_compress(kv, gate, pos_bias, seq_len, kv_off, kv_pos0, ent_off, item_seq, item_ent,
                 entries, *,
                 B: int, D: int, fmt: int = CSA_KV_BF16, rope_theta: float = 10000.0,
                 eps: float = 1e-6, layout=None, dev_status=None, stream=None):
    _check(_lib.hca_compress(_p(kv), _p(gate), _p(pos_bias), _p(seq_len), _p(kv_off), _p(kv_pos0),
                             _p(ent_off), _p(item_seq), _p(item_ent), item_seq.numel(), B, D, fmt,
                             rope_theta, eps, _p(entries), _lay(layout), _p(dev_status),
                             _s(stream)))


def lightning_indexer_topk(qI, qI_scale, w, kI, kI_scale, seq_len, ent_off, q_seq, q_pos, idx_out,
                           workspace, *, B: int, H_I: int, d_I: int, m: int, k: int, max_n: int,
                           scores_out=None, ld_scores: int = 0, layout=None, dev_status=None,
                           stream=None):
    _check(_lib.lightning_indexer_topk(
        _p(qI), _p(qI_scale), _p(w), _p(kI), _p(kI_scale), kI_scale.numel(), _p(seq_len),
        _p(ent_off), _p(q_seq),
        _p(q_pos),
        q_seq.numel(), B, H_I, d_I, m, k, max_n, _p(idx_out), _p(scores_out), ld_scores,
        _p(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
        _lay(layout), _p(dev_status), _s(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def lightning_indexer_topk_noalloc(qI, qI_scale, w, kI, kI_scale, seq_len, ent_off, q_seq, q_pos,
                                   idx_out, *, B: int, H_I: int, d_I: int, m: int, k: int,
                                   max_n: int, scores_out=None, ld_scores: int = 0,
                                   dev_status=None, stream=None):
    """lightning_indexer_topk without a workspace, for callers that cannot allocate device
    memory: the scratch lives in a fixed 16 MiB device array inside libcsa, shared by all
    calls on a device (calls that overlap on the GPU race on it)."""
    _check(_lib.lightning_indexer_topk_noalloc(
        _p(qI), _p(qI_scale), _p(w), _p(kI), _p(kI_scale), kI_scale.numel(), _p(seq_len),
        _p(ent_off), _p(q_seq),
        _p(q_pos), q_seq.numel(), B, H_I, d_I, m, k, max_n, _p(idx_out), _p(scores_out),
        ld_scores, _p(dev_status), _s(stream)))


def lightning_indexer_topk_mxfp4(qI, qI_sf, w, kI, kI_sf, seq_len, ent_off, q_seq, q_pos,
                                 idx_out, workspace, *, B: int, H_I: int, d_I: int, m: int,
                                 k: int, max_n: int, select_bf16: bool = False, scores_out=None,
                                 ld_scores: int = 0, layout=None, dev_status=None,
                                 stream=None):
    """MXFP4 indexer + top-k (see include/csa.h).  qI / kI: packed e2m1 bytes; qI_sf /
    kI_sf: UE8M0 bytes."""
    _check(_lib.lightning_indexer_topk_mxfp4(
        _p(qI), _p(qI_sf), _p(w), _p(kI), _p(kI_sf), kI.shape[0], _p(seq_len), _p(ent_off),
        _p(q_seq), _p(q_pos), q_seq.numel(), B, H_I, d_I, m, k, max_n, 1 if select_bf16 else 0,
        _p(idx_out), _p(scores_out), ld_scores, _p(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _lay(layout), _p(dev_status), _s(stream)))


def csa_cache_append(kv_new, gate_new, seq_len, kv_off, kv_pos0, kv, gate, *, B: int, D: int,
                     m: int, kI_new=None, kI_scale_new=None, ent_off=None, kI=None,
                     kI_scale=None, layout=None, dev_status=None, stream=None):
    """One decode token per sequence into the state cache (and, for the entries it
    completes, their indexer keys into the key store); see include/csa.h."""
    _check(_lib.csa_cache_append(
        _p(kv_new), _p(gate_new), _p(kI_new), _p(kI_scale_new),
        0 if kI is None else kI.shape[1], _p(seq_len), _p(kv_off), _p(kv_pos0), kv.shape[0],
        _p(ent_off), 0 if kI is None else kI.shape[0], B, D, m, _p(kv), _p(gate), _p(kI),
        _p(kI_scale), _lay(layout), _p(dev_status), _s(stream)))


def csa_topk_merge(cand_scores, cand_idx, idx_out, *, dev_status=None, stream=None):
    """Top-k of sequences from their slices' candidates, [W, Q, k_in] (see include/csa.h)."""
    W, Q, k_in = cand_idx.shape
    assert cand_scores.shape == cand_idx.shape
    assert cand_idx.stride() == cand_scores.stride() and cand_idx.stride()[1:] == (k_in, 1)
    _check(_lib.csa_topk_merge(_p(cand_scores), _p(cand_idx), cand_idx.stride(0), W, Q, k_in,
                               idx_out.shape[1], _p(idx_out), _p(dev_status), _s(stream)))


def csa_cp_candidates(idx, scores, q_seq, slice_lo, cand_idx, cand_scores, *, B: int,
                      dev_status=None, stream=None):
    """A slice's selection as candidates of the whole sequence (see include/csa.h)."""
    Q, k = idx.shape
    _check(_lib.csa_cp_candidates(_p(idx), _p(scores), scores.stride(0), _p(q_seq),
                                  _p(slice_lo), Q, B, k, _p(cand_idx), _p(cand_scores),
                                  _p(dev_status), _s(stream)))


def csa_cp_pack_rows(idx, q_seq, slice_lo, slice_n, ent_off, entries, out, local_idx=None, *,
                     B: int, dev_status=None, stream=None):
    """The selected rows this rank's slice holds, at their positions (see include/csa.h)."""
    Q, k = idx.shape
    _check(_lib.csa_cp_pack_rows(_p(idx), _p(q_seq), _p(slice_lo), _p(slice_n), _p(ent_off),
                                 _p(entries), entries.shape[0], entries.shape[1], Q, B, k,
                                 _p(out), _p(local_idx), _p(dev_status), _s(stream)))


def sparse_mqa_attn(q, entries, seq_len, ent_off, kv, kv_off, kv_pos0, q_seq, q_pos, idx, sink,
                    out, *,
                    fmt: int, B: int, H: int, D: int, W: int, m: int, k: int,
                    softmax_scale: float, rope_theta: float = 10000.0, eps: float = 1e-6,
                    layout=None, dev_status=None, stream=None):
    _check(_lib.sparse_mqa_attn(
        _p(q), _p(entries), fmt, entries.shape[0], _p(seq_len), _p(ent_off), _p(kv), _p(kv_off), _p(kv_pos0), _p(q_seq),
        _p(q_pos), _p(idx), k, m, _p(sink), q_seq.numel(), B, H, D, W, softmax_scale,
        rope_theta, eps, _p(out), _lay(layout), _p(dev_status), _s(stream)))


def dense_hca_attn(q, entries, seq_len, ent_off, kv, kv_off, kv_pos0, q_seq, q_pos, sink, out,
                   workspace, *, fmt: int, B: int, H: int, D: int, W: int, m: int, max_n: int,
                   softmax_scale: float, rope_theta: float = 10000.0, eps: float = 1e-6,
                   layout=None, dev_status=None, stream=None):
    _check(_lib.dense_hca_attn(
        _p(q), _p(entries), fmt, entries.shape[0], _p(seq_len), _p(ent_off), _p(kv), _p(kv_off), _p(kv_pos0), _p(q_seq),
        _p(q_pos), m, _p(sink), q_seq.numel(), B, H, D, W, softmax_scale, rope_theta, eps,
        max_n, _p(out), _p(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(),
        _lay(layout), _p(dev_status), _s(stream)))
