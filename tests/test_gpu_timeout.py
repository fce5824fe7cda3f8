"""The device-side failure path of the bounded waits.

Every mbarrier wait in the tensor-core kernels gives up after a limit: it flags
CSA_DEV_TIMEOUT in dev_status, and the CTA waits for its own copies and MMAs in flight,
frees its tensor memory and returns.  The limit is lowered here to a few hundred clocks
(csa_debug_set_wait_limit), far below the time any tile load takes, so the first wait on a
load runs out.  Only kernels launched without thread-block clusters run while it is
lowered: the tensor-core indexer (with the single-CTA top-k after it, rows of at most 10K
entries) and the dense HCA attention with its combine kernel.  Each must report
CSA_DEV_TIMEOUT and return; with the default restored, the next call must match the oracle
(index sets bit for bit, attention within the output tolerance)."""
import numpy as np
import pytest
import torch

import _orc
import long_context_compressed_04_b200 as L
from long_context_compressed_04_b200 import CSA_DEV_TIMEOUT, pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SHORT_LIMIT = 300   # SM clocks


def _with_short_limit(fn):
    torch.cuda.synchronize()
    L.csa_debug_set_wait_limit(SHORT_LIMIT)
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        L.csa_debug_set_wait_limit(0)


def test_indexer_wait_timeout_is_reported_and_recovers():
    wl = synth.make_workload("t", B=2, T=[40000, 20001], D=128, H=16, m=4, span=8, H_I=64,
                             d_I=128, k=512, seed=401, device=DEV)
    buf = pipeline.alloc(wl, DEV)
    _with_short_limit(lambda: pipeline.indexer_topk(wl, buf))
    assert int(buf.dev_status.item()) & CSA_DEV_TIMEOUT
    buf.dev_status.zero_()
    buf.idx.fill_(-7)
    pipeline.indexer_topk(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    ref, _ = _orc.indexer(wl.to("cpu"))
    assert np.array_equal(buf.idx.cpu().numpy(), ref)


def test_dense_attention_wait_timeout_is_reported_and_recovers():
    wl = synth.make_workload("t", B=2, T=[128 * 100 + 5, 128 * 30], D=128, H=64, m=128,
                             span=128, seed=402, device=DEV)
    rows, _ = _orc.compress(wl.to("cpu"))
    buf = pipeline.alloc(wl, DEV)
    buf.entries.copy_(torch.from_numpy(rows))
    _with_short_limit(lambda: pipeline.attend(wl, buf))
    assert int(buf.dev_status.item()) & CSA_DEV_TIMEOUT
    buf.dev_status.zero_()
    buf.out.zero_()
    pipeline.attend(wl, buf)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    _orc.assert_out_close(buf.out, _orc.attention(wl.to("cpu"), rows, None))
