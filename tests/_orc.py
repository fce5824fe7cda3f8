"""Runs the CPU oracle on a synthetic workload and compares GPU results against it.
Test infrastructure only."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle.workload import (attention, compress, f32, i32, i64, indexer, indexer_mxfp4,  # noqa: F401
                             u8, u16)

# Output tolerance for bf16 / fp8 storage with fp32 accumulation: max abs and relative L2.
ATOL = 2e-2
REL_L2 = 5e-3


def assert_out_close(gpu_out: torch.Tensor, ref: np.ndarray, atol=ATOL, rel_l2=REL_L2):
    g = gpu_out.detach().cpu().to(torch.float64).numpy()
    assert g.shape == ref.shape
    assert np.all(np.isfinite(g))
    err = np.abs(g - ref)
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= atol, f"max abs err {err.max():.3e} > {atol}"
    assert rel <= rel_l2, f"rel L2 err {rel:.3e} > {rel_l2}"
    return float(err.max()), float(rel)


def entry_values(rows: np.ndarray, fmt: int, D: int) -> np.ndarray:
    return np.stack([oracle.entry_load(r, fmt, D) for r in rows]) if len(rows) else np.zeros((0, D))
