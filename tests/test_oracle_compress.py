"""Pins for the oracle's compression step (CSA 4:1 overlapped, HCA 128:1), CPU only.

Closed forms (uniform weights -> mean pooling; one dominant logit -> that token), a library
special case (scipy's softmax), the RMSNorm norm identity, locality, permutation
invariance, the first-entry reading, and the entry counts the pages print."""
import json
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def _bits(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _vals(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()


def _case(T=64, D=128, span=8, seed=0, const_gate=False):
    rng = np.random.default_rng(seed)
    kv = _bits(rng.standard_normal((T, D)))
    gate = _bits(np.zeros((T, D)) if const_gate else rng.standard_normal((T, D)))
    bias = (np.zeros((span, D)) if const_gate else rng.standard_normal((span, D)) * 0.1).astype(np.float32)
    return kv, gate, bias


def _compress(kv, gate, bias, ents, *, m, span, D, T, eps=1e-6, theta=10000.0, pos0=0):
    n = len(ents)
    _, e = oracle.compress(kv, gate, bias, [0], [pos0], [0], np.zeros(n, np.int32),
                           np.asarray(ents, np.int32), m=m, span=span, D=D, fmt=0,
                           theta=theta, eps=eps, n_entry_rows=T // m)
    return e


def _unrope(e, pos):
    return oracle.rope(e, -pos)


def test_entry_counts_follow_the_pages():
    m, span = GOLDEN["csa_m"]["value"], GOLDEN["csa_span"]["value"]
    assert span == 2 * m
    assert GOLDEN["entries_4k_csa"]["tokens"] // m == GOLDEN["entries_4k_csa"]["entries"]
    mh = GOLDEN["hca_m"]["value"]
    assert GOLDEN["entries_1m_hca"]["tokens"] // mh == GOLDEN["entries_1m_hca"]["entries"]
    # the oracle compresses every complete block of a 4096-token sequence, and nothing past it
    T, D = 4096, 128
    kv, gate, bias = _case(T=T, D=D)
    e = _compress(kv, gate, bias, [1023], m=m, span=span, D=D, T=T)
    assert np.all(np.isfinite(e))
    with pytest.raises(ValueError):      # entry 1024 would need tokens 4096..4099
        oracle.compress(kv, gate, bias, [0], [T - 4], [0], [0], [1], m=m, span=span, D=D)


@pytest.mark.parametrize("m,span", [(4, 8), (128, 128)])
def test_uniform_weights_give_mean_pooling(m, span):
    T, D = 512, 128
    kv, gate, bias = _case(T=T, D=D, span=span, const_gate=True)
    i = 3
    e = _compress(kv, gate, bias, [i], m=m, span=span, D=D, T=T, eps=0.0)[0]
    toks = _vals(kv)[(i + 1) * m - span:(i + 1) * m]
    mean = toks.mean(axis=0)
    want = mean / np.sqrt(np.mean(mean ** 2))
    p = (i + 1) * m - 1
    assert np.allclose(e[: D - 64], want[: D - 64], rtol=0, atol=1e-12)
    assert np.allclose(_unrope(e, p), want, atol=1e-12)


def test_dominant_logit_selects_that_token():
    T, D, m, span = 64, 128, 4, 8
    kv, gate, bias = _case(T=T, D=D)
    g = _vals(gate).copy()
    i, j = 5, 2                           # token (i-1)*4 + 2 of entry 5
    g[(i - 1) * m + j] += 60.0
    e = _compress(kv, _bits(g), bias, [i], m=m, span=span, D=D, T=T, eps=0.0)[0]
    tok = _vals(kv)[(i - 1) * m + j]
    want = tok / np.sqrt(np.mean(tok ** 2))
    assert np.allclose(_unrope(e, (i + 1) * m - 1), want, atol=1e-9)


def test_pooling_matches_library_softmax():
    T, D, m, span = 64, 128, 4, 8
    kv, gate, bias = _case(T=T, D=D, seed=3)
    for i in [1, 7, 15]:
        e = _compress(kv, gate, bias, [i], m=m, span=span, D=D, T=T, eps=0.0)[0]
        sl = slice((i + 1) * m - span, (i + 1) * m)
        wts = scipy.special.softmax(_vals(gate)[sl] + bias.astype(np.float64), axis=0)
        pooled = (wts * _vals(kv)[sl]).sum(axis=0)
        want = pooled / np.sqrt(np.mean(pooled ** 2))
        assert np.allclose(_unrope(e, (i + 1) * m - 1), want, atol=1e-12)


def test_first_csa_entry_drops_missing_previous_block():
    # Entry 0 has no previous block: it must equal a 4-token pooling of tokens 0..3 with the
    # bias rows that belong to the current block (rows 4..7).
    T, D = 64, 128
    kv, gate, bias = _case(T=T, D=D, seed=4)
    e_csa = _compress(kv, gate, bias, [0], m=4, span=8, D=D, T=T)[0]
    e_blk = _compress(kv, gate, np.ascontiguousarray(bias[4:]), [0], m=4, span=4, D=D, T=T)[0]
    assert np.array_equal(e_csa, e_blk)


def test_rmsnorm_identity_and_rotation():
    T, D, m, span = 64, 576, 4, 8
    kv, gate, bias = _case(T=T, D=D, seed=5)
    eps = 1e-6
    e = _compress(kv, gate, bias, [4], m=m, span=span, D=D, T=T, eps=eps)[0]
    e0 = _compress(kv, gate, bias, [4], m=m, span=span, D=D, T=T, eps=0.0)[0]
    # eps=0 gives unit RMS; with eps, ||e||^2 = D*ms/(ms+eps) where e = e0 * sqrt(ms/(ms+eps))
    assert np.mean(e0 ** 2) == pytest.approx(1.0, rel=1e-13)
    ratio = np.sum(e ** 2) / np.sum(e0 ** 2)
    sl = slice(12, 20)
    wts = scipy.special.softmax(_vals(gate)[sl] + bias.astype(np.float64), axis=0)
    pooled = (wts * _vals(kv)[sl]).sum(axis=0)
    ms = np.mean(pooled ** 2)
    assert ratio == pytest.approx(ms / (ms + eps), rel=1e-12)


@pytest.mark.parametrize("m,span", [(4, 8), (128, 128)])
def test_entry_depends_only_on_its_tokens(m, span):
    T, D = 1024, 128
    kv, gate, bias = _case(T=T, D=D, span=span, seed=6)
    i = 4
    base = _compress(kv, gate, bias, [i], m=m, span=span, D=D, T=T)[0]
    lo, hi = (i + 1) * m - span, (i + 1) * m
    for p in [lo - 1, hi, 0, T - 1]:
        if lo <= p < hi:
            continue
        kv2 = kv.copy()
        kv2[p] = _bits(np.full(D, 7.0))
        assert np.array_equal(_compress(kv2, gate, bias, [i], m=m, span=span, D=D, T=T)[0], base)
    for p in [lo, hi - 1]:
        kv2 = kv.copy()
        kv2[p] = _bits(np.full(D, 7.0))
        assert not np.array_equal(_compress(kv2, gate, bias, [i], m=m, span=span, D=D, T=T)[0], base)


def test_permuting_tokens_with_their_bias_rows():
    T, D, m, span = 64, 128, 4, 8
    kv, gate, bias = _case(T=T, D=D, seed=7)
    i = 6
    base = _compress(kv, gate, bias, [i], m=m, span=span, D=D, T=T)[0]
    perm = np.array([3, 7, 0, 5, 1, 6, 2, 4])
    lo = (i + 1) * m - span
    kv2, gate2 = kv.copy(), gate.copy()
    kv2[lo:lo + span] = kv[lo + perm]
    gate2[lo:lo + span] = gate[lo + perm]
    e = _compress(kv2, gate2, np.ascontiguousarray(bias[perm]), [i], m=m, span=span, D=D, T=T)[0]
    assert np.allclose(e, base, atol=1e-13)


def test_single_token_block_is_the_window_row_transform():
    # m = 1, span = 1: pooling one token is the identity, so an entry is that token RMSNormed
    # and RoPEd at its own position -- the transform the window rows get.
    T, D = 16, 128
    kv, gate, bias = _case(T=T, D=D, span=1, seed=8)
    for p in [0, 9]:
        e = _compress(kv, gate, bias, [p], m=1, span=1, D=D, T=T)[0]
        want = oracle.rope(oracle.rmsnorm(_vals(kv)[p]), float(p))
        assert np.allclose(e, want, atol=1e-13)


def test_raw_tail_storage_offsets():
    # the same entry computed from a full store and from a store that keeps only the tail
    T, D = 256, 128
    kv, gate, bias = _case(T=T, D=D, seed=9)
    full = _compress(kv, gate, bias, [62], m=4, span=8, D=D, T=T)[0]
    keep = 16
    _, tail = oracle.compress(kv[T - keep:], gate[T - keep:], bias, [0], [T - keep], [0], [0],
                              [62], m=4, span=8, D=D, n_entry_rows=T // 4)
    assert np.array_equal(full, tail[0])
