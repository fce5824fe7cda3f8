"""End-to-end parity of the whole hot path: the GPU compresses every entry, selects with
the lightning indexer and attends; the oracle does the same from the same raw inputs.
Index sets must match bit-exactly (integer-valued indexer inputs) and outputs within the
bf16/fp8-storage tolerance."""
import numpy as np
import pytest
import torch

import _orc
from long_context_compressed_04_b200 import pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _e2e(wl):
    buf = pipeline.alloc(wl, DEV)
    seq, ent = pipeline.all_entry_items(wl, DEV)
    pipeline.step(wl, buf, seq, ent)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    cw = wl.to("cpu")
    rows, _ = _orc.compress(cw)
    idx = None
    if wl.H_I:
        idx = _orc.indexer(cw, want_scores=False)
        assert np.array_equal(buf.idx.cpu().numpy(), idx)
    ref = _orc.attention(cw, rows, idx)
    return _orc.assert_out_close(buf.out, ref)


def test_csa_decode_4k_end_to_end():
    _e2e(synth.csa_decode_4k(device=DEV))


def test_csa_decode_ragged_end_to_end():
    wl = synth.make_workload("t", B=4, T=[20001, 13000, 4099, 9000], D=128, H=64, m=4, span=8,
                             H_I=64, d_I=128, k=512, seed=41, device=DEV)
    _e2e(wl)


def test_hca_decode_end_to_end():
    wl = synth.make_workload("t", B=3, T=[128 * 64 + 5, 128 * 20, 128 * 33 + 127], D=128, H=64,
                             m=128, span=128, seed=42, device=DEV)
    _e2e(wl)


def test_csa_decode_fp8_entries_end_to_end():
    wl = synth.make_workload("t", B=2, T=[6000, 2500], D=576, H=128, m=4, span=8, fmt=1,
                             H_I=64, d_I=128, k=256, seed=43, device=DEV)
    _e2e(wl)


def test_csa_prefill_chunk_end_to_end():
    # causal prefill: 96 new queries appended to 1000 prior tokens, one sequence
    wl = synth.make_workload("t", B=1, T=[1096], D=128, H=64, m=4, span=8, H_I=64, d_I=128,
                             k=128, queries="prefill", n_new=96, seed=44, device=DEV)
    _e2e(wl)
