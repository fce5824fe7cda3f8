"""GPU parity of csa_compress / hca_compress against the oracle (fp64), element by element.

The kernel computes in fp32 and stores bf16 (or e4m3 with 1x128 scales); the oracle's
fp64 value before storage rounding bounds the stored value: bf16 within one bf16 step
(2^-8 relative), e4m3 within one e4m3 step (2^-3 relative, or the subnormal step of the
block scale).  Nearly every stored bit pattern must equal the oracle's own rounding."""
import numpy as np
import pytest
import torch

import _orc
from long_context_compressed_04_b200 import CSA_DEV_OOB, pipeline, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_values(rows: torch.Tensor, fmt: int, D: int) -> np.ndarray:
    r = rows.cpu()
    if fmt == 0:
        return r.view(torch.bfloat16).to(torch.float64).numpy().reshape(-1, D)
    n = r.shape[0]
    codes = r[:, :512].contiguous().view(torch.float8_e4m3fn).to(torch.float64).reshape(n, 4, 128)
    scale = r[:, 512:528].contiguous().view(torch.float32).to(torch.float64).reshape(n, 4, 1)
    rope = r[:, 528:].contiguous().view(torch.bfloat16).to(torch.float64).reshape(n, 64)
    return torch.cat([(codes * scale).reshape(n, 512), rope], 1).numpy()


def _check(wl, entries_gpu, item_seq=None, item_ent=None):
    rows_o, e64 = _orc.compress(wl, item_seq, item_ent)
    if item_seq is None:
        sel = np.arange(wl.ent_rows)
    else:
        sel = _orc.i64(wl.ent_off)[np.asarray(item_seq)] + np.asarray(item_ent)
    g = _gpu_values(entries_gpu[torch.as_tensor(sel, device=entries_gpu.device)], wl.fmt, wl.D)
    assert np.all(np.isfinite(g))
    if wl.fmt == 0:
        assert np.all(np.abs(g - e64) <= 2.0 ** -8 * np.abs(e64) + 1e-6)
        same = (entries_gpu.cpu().numpy()[sel] == rows_o[sel]).mean()
        assert same > 0.98, same
    else:
        r = entries_gpu.cpu().numpy()[sel]
        sc = r[:, 512:528].copy().view(np.float32)
        sco = rows_o[sel][:, 512:528].copy().view(np.float32)
        assert np.allclose(sc, sco, rtol=1e-5, atol=0)
        step = np.repeat(sc, 128, axis=1) * 2.0 ** -9
        err = np.abs(g[:, :512] - e64[:, :512])
        assert np.all(err <= 2.0 ** -3 * np.abs(e64[:, :512]) + step)
        assert (r[:, :512] == rows_o[sel][:, :512]).mean() > 0.99
        assert np.all(np.abs(g[:, 512:] - e64[:, 512:]) <= 2.0 ** -8 * np.abs(e64[:, 512:]) + 1e-6)


@pytest.mark.parametrize("D,fmt", [(128, 0), (576, 0), (576, 1)])
def test_csa_compress_all_entries_ragged(D, fmt):
    wl = synth.make_workload("t", B=3, T=[517, 64, 1203], D=D, H=16, m=4, span=8, fmt=fmt,
                             seed=11, device=DEV)
    buf = pipeline.alloc(wl, DEV)
    seq, ent = pipeline.all_entry_items(wl, DEV)
    pipeline.compress(wl, buf, seq, ent)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    _check(wl.to("cpu"), buf.entries)


def test_hca_compress_ragged():
    wl = synth.make_workload("t", B=2, T=[128 * 9 + 77, 128 * 3], D=128, H=64, m=128, span=128,
                             seed=12, device=DEV)
    buf = pipeline.alloc(wl, DEV)
    seq, ent = pipeline.all_entry_items(wl, DEV)
    pipeline.compress(wl, buf, seq, ent)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    _check(wl.to("cpu"), buf.entries)


def test_compress_from_tail_store_and_unstored_tokens_are_flagged():
    # decode-style store: only the last 64 raw tokens of each sequence are kept
    wl = synth.make_workload("t", B=2, T=[1000, 777], D=128, H=16, m=4, span=8, keep_raw=64,
                             seed=13, device=DEV)
    buf = pipeline.alloc(wl, DEV)
    seq, ent = pipeline.newest_entry_items(wl, DEV)
    pipeline.compress(wl, buf, seq, ent)
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) == 0
    _check(wl.to("cpu"), buf.entries, seq.cpu().numpy(), ent.cpu().numpy())
    # entry 10 needs tokens 36..43, which are not stored: flagged, row untouched
    before = buf.entries.clone()
    pipeline.compress(wl, buf, torch.tensor([0], dtype=torch.int32, device=DEV),
                      torch.tensor([10], dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert int(buf.dev_status.item()) & CSA_DEV_OOB
    assert torch.equal(before, buf.entries)
