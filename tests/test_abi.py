"""The C ABI on the CPU: the library loads, exports every function include/csa.h declares,
and rejects bad arguments on the host before any launch (no GPU needed for these paths)."""
import ctypes
import os
import re

import pytest

import long_context_compressed_04_b200 as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\**\s+\**([A-Za-z_][A-Za-z0-9_]*)\s*\(", src, flags=re.M))
    return names


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert {"csa_compress", "hca_compress", "lightning_indexer_topk", "sparse_mqa_attn",
            "dense_hca_attn"} <= names
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared but not exported"
    assert set(L.EXPORTED) >= names


def test_host_queries():
    assert L.csa_version() >= 100
    assert L.csa_entry_row_bytes(L.CSA_KV_BF16, 128) == 256
    assert L.csa_entry_row_bytes(L.CSA_KV_FP8_576, 576) == 656
    assert L.csa_entry_row_bytes(L.CSA_KV_FP8_576, 128) == -1
    ws = L.csa_indexer_workspace_size(32, 33000, 512)
    assert ws >= 32 * 33000 * 4 and ws % 256 == 0
    assert L.dense_hca_workspace_size(16, 64, 128, 8192) > 0


def _raw():
    return L._lib


def test_null_and_unsupported_arguments_fail_on_host():
    lib = _raw()
    P = ctypes.c_void_p
    fake = P(4096)  # never dereferenced: validation fails before any launch
    # null pointers
    st = lib.csa_compress(None, None, None, None, None, None, None, None, None, 4, 1, 128, 0, 10000.0,
                          1e-6, None, None, None, None)
    assert st == 1 and b"null" in lib.csa_last_error()
    # n_items = 0 is a no-op even with null pointers
    assert lib.csa_compress(None, None, None, None, None, None, None, None, None, 0, 1, 128, 0,
                            10000.0, 1e-6, None, None, None, None) == 0
    # unsupported head dim
    st = lib.csa_compress(fake, fake, fake, fake, fake, fake, fake, fake, fake, 4, 1, 96, 0, 10000.0,
                          1e-6, fake, None, None, None)
    assert st == 2 and b"head dim" in lib.csa_last_error()
    # misaligned
    st = lib.hca_compress(P(4097), fake, fake, fake, fake, fake, fake, fake, fake, 4, 1, 128, 0,
                          10000.0, 1e-6, fake, None, None, None)
    assert st == 1 and b"aligned" in lib.csa_last_error()
    # fp8 format needs D = 576
    st = lib.sparse_mqa_attn(fake, fake, 1, 10, fake, fake, fake, fake, fake, fake, fake, fake, 8, 4, fake,
                             1, 1, 16, 128, 128, 0.08, 10000.0, 1e-6, fake, None, None, None)
    assert st == 2
    # window above 128
    st = lib.sparse_mqa_attn(fake, fake, 0, 10, fake, fake, fake, fake, fake, fake, fake, fake, 8, 4, fake,
                             1, 1, 16, 128, 129, 0.08, 10000.0, 1e-6, fake, None, None, None)
    assert st == 1 and b"window" in lib.csa_last_error()
    # unsupported heads
    st = lib.dense_hca_attn(fake, fake, 0, 10, fake, fake, fake, fake, fake, fake, fake, 128, fake, 1, 1, 48,
                            128, 128, 0.08, 10000.0, 1e-6, 10, fake, fake, 1 << 20, None, None, None)
    assert st == 2


def test_workspace_is_checked_on_host():
    lib = _raw()
    P = ctypes.c_void_p
    fake = P(4096)
    need = lib.csa_indexer_workspace_size(2, 1000, 64)
    st = lib.lightning_indexer_topk(fake, fake, fake, fake, fake, 100, fake, fake, fake, fake, 2, 2, 4, 64,
                                    4, 64, 1000, fake, None, 0, fake, need - 1, None, None, None)
    assert st == 4 and b"workspace" in lib.csa_last_error()
    st = lib.lightning_indexer_topk(fake, fake, fake, fake, fake, 100, fake, fake, fake, fake, 2, 2, 4, 64,
                                    4, 4096, 1000, fake, None, 0, fake, need, None, None, None)
    assert st == 2 and b"k =" in lib.csa_last_error()
    st = lib.lightning_indexer_topk(fake, fake, fake, fake, fake, 100, fake, fake, fake, fake, 2, 2, 80, 64,
                                    4, 64, 1000, fake, None, 0, fake, need, None, None, None)
    assert st == 2
