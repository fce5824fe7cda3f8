"""Host-side bookkeeping of the hybrid cache (no GPU): the block free list, block-table growth
as entries complete, release, and the layout struct handed to the C calls."""
import ctypes

import pytest
import torch

import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import cache


def test_block_allocator_order_exhaustion_and_release():
    a = cache.BlockAllocator(3)
    assert [a.alloc(), a.alloc()] == [0, 1]
    a.release([0])
    assert a.alloc() == 0 and a.alloc() == 2
    with pytest.raises(RuntimeError, match="full"):
        a.alloc()


def test_blocks_follow_completed_entries():
    hc = cache.HybridCache(2, 128, L.CSA_KV_BF16, 128, n_blocks=8, max_blocks=4, device="cpu")
    # 32 entries fill one block of 128 tokens; the 33rd needs a second
    assert hc._ensure_blocks(0, 32) and int((hc.bt_host[0] >= 0).sum()) == 1
    assert not hc._ensure_blocks(0, 32)
    assert hc._ensure_blocks(0, 33) and int((hc.bt_host[0] >= 0).sum()) == 2
    assert hc._ensure_blocks(1, 1)
    used = sorted(int(x) for x in hc.bt_host.flatten() if int(x) >= 0)
    assert used == [0, 1, 2] and len(hc.alloc.free) == 5
    hc.release(0)
    assert int((hc.bt_host[0] >= 0).sum()) == 0 and len(hc.alloc.free) == 7
    assert torch.equal(hc.block_table, hc.bt_host)


def test_layout_struct_fields():
    assert L.cache_layout() is None
    bt = torch.zeros((3, 5), dtype=torch.int32)
    lay = L.cache_layout(bt, kv_ring=128)
    assert lay.block_table == bt.data_ptr() and lay.bt_stride == 5 and lay.kv_ring == 128
    assert ctypes.sizeof(L.CacheLayout) == 24
    ring_only = L.cache_layout(kv_ring=64)
    assert ring_only.block_table is None and ring_only.kv_ring == 64


def test_layout_validation_on_the_host():
    # a block table needs m = 4; the check runs before any launch
    lib = L._lib
    fake = ctypes.c_void_p(4096)
    bt = torch.zeros((1, 4), dtype=torch.int32)
    lay = L.cache_layout(bt)
    st = lib.hca_compress(fake, fake, fake, fake, fake, None, None, fake, fake, 1, 1, 128, 0,
                          10000.0, 1e-6, fake, ctypes.byref(lay), None, None)
    assert st == 1 and b"m = 4" in lib.csa_last_error()
    # without a block table, ent_off is required
    st = lib.csa_compress(fake, fake, fake, fake, fake, fake, None, fake, fake, 1, 1, 128, 0,
                          10000.0, 1e-6, fake, None, None, None)
    assert st == 1 and b"ent_off" in lib.csa_last_error()
