"""Pins for the oracle's lightning-indexer score and top-k selection (CPU only).

Exact integer brute force, an fp64 evaluation within the fp32 rounding bound, the fixed
head order of the fp32 accumulation, brute-force selection by Python's sort, ties,
padding, visibility and permutation."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _e4m3(x):
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _ints(rng, shape):
    return rng.integers(-3, 4, size=shape)


def _run(qI, qs, w, kI, ks, t, m=4, k=8, want_scores=True, ent_off=(0,)):
    HI, dI = qI.shape[-2], qI.shape[-1]
    Q = qI.shape[0]
    return oracle.indexer_topk(_e4m3(qI), qs, w, _e4m3(kI), ks, list(ent_off),
                               np.zeros(Q, np.int32), np.full(Q, t, np.int32), H_I=HI, d_I=dI,
                               m=m, k=k, want_scores=want_scores, ld_scores=kI.shape[0])


def test_integer_scores_equal_exact_brute_force():
    rng = np.random.default_rng(0)
    HI, dI, N = 4, 64, 256
    q = _ints(rng, (1, HI, dI))
    kk = _ints(rng, (N, dI))
    w = np.array([[1.0, 0.5, 0.25, 2.0 ** -7]], np.float32)        # dyadic: exact in fp32
    idx, s = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(N, np.float32), t=4 * N - 1)
    for i in range(N):
        exact = sum(Fraction(float(w[0, h])) * max(int(q[0, h] @ kk[i]), 0) for h in range(HI))
        assert Fraction(float(s[0, i])) == exact


def test_real_scores_within_fp32_bound_of_fp64():
    rng = np.random.default_rng(1)
    HI, dI, N = 64, 128, 300
    q = rng.standard_normal((1, HI, dI)) * 0.5
    kk = rng.standard_normal((N, dI)) * 0.5
    qs = rng.uniform(0.5, 2.0, (1, HI)).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, N).astype(np.float32)
    w = rng.uniform(0, 1, (1, HI)).astype(np.float32)
    _, s = _run(q, qs, w, kk, ks, t=4 * N - 1)
    qv = oracle.e4m3_value(_e4m3(q)).astype(np.float64)[0]
    kv = oracle.e4m3_value(_e4m3(kk)).astype(np.float64)
    d = kv @ qv.T                                                   # [N, HI] exact sums
    terms = np.maximum(d, 0) * (w[0].astype(np.float64) * qs[0].astype(np.float64))
    exact = terms.sum(axis=1) * ks.astype(np.float64)
    bound = (HI + 3) * 2.0 ** -24 * np.abs(terms).sum(axis=1) * ks + 1e-30
    assert np.all(np.abs(s[0] - exact) <= bound)


def test_heads_accumulate_in_ascending_order_in_fp32():
    # d = 1 for every head.  In ascending order: 1 + 2^-24 ties back to 1 (even), twice.
    # Any other order or a wider accumulator gives 1 + 2^-23.
    HI, dI = 3, 64
    q = np.zeros((1, HI, dI))
    q[0, :, 0] = 1.0
    kk = np.zeros((1, dI))
    kk[0, 0] = 1.0
    w = np.array([[1.0, 2.0 ** -24, 2.0 ** -24]], np.float32)
    _, s = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(1, np.float32), t=3, k=1)
    assert s[0, 0] == np.float32(1.0)
    w = np.array([[2.0 ** -24, 2.0 ** -24, 1.0]], np.float32)
    _, s = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(1, np.float32), t=3, k=1)
    assert s[0, 0] == np.float32(1.0 + 2.0 ** -23)


def test_relu_per_head():
    HI, dI = 2, 64
    q = np.zeros((1, HI, dI))
    q[0, 0, 0], q[0, 1, 0] = 2.0, -3.0
    kk = np.zeros((1, dI))
    kk[0, 0] = 1.0
    w = np.ones((1, HI), np.float32)
    _, s = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(1, np.float32), t=3, k=1)
    assert s[0, 0] == 2.0          # the negative head contributes 0, not -3


@pytest.mark.parametrize("k", [1, 17, 64, 200])
def test_topk_equals_python_sort_brute_force(k):
    rng = np.random.default_rng(2)
    HI, dI, N = 4, 64, 1024
    q, kk = _ints(rng, (1, HI, dI)), _ints(rng, (N, dI))
    w = rng.uniform(0, 1, (1, HI)).astype(np.float32)
    idx, s = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(N, np.float32), t=4 * N - 1, k=k)
    want = sorted(sorted(range(N), key=lambda i: (-float(s[0, i]), i))[:k])
    assert idx[0].tolist() == want


def test_ties_go_to_the_lower_index():
    rng = np.random.default_rng(3)
    HI, dI, N = 4, 64, 64
    base = _ints(rng, (8, dI))
    kk = base[rng.integers(0, 8, N)]                   # only 8 distinct keys -> many ties
    q = _ints(rng, (1, HI, dI))
    w = np.ones((1, HI), np.float32)
    idx, s = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(N, np.float32), t=4 * N - 1, k=20)
    order = sorted(range(N), key=lambda i: (-float(s[0, i]), i))
    assert idx[0].tolist() == sorted(order[:20])
    thr = s[0, order[19]]
    tied = [i for i in range(N) if s[0, i] == thr]
    chosen = [i for i in idx[0] if s[0, i] == thr]
    assert chosen == tied[: len(chosen)]               # lowest indices among the ties
    # all-equal scores: the first k indices
    kk = np.tile(base[:1], (N, 1))
    idx, _ = _run(q, np.ones((1, HI), np.float32), w, kk, np.ones(N, np.float32), t=4 * N - 1, k=20)
    assert idx[0].tolist() == list(range(20))


def test_visibility_and_padding():
    rng = np.random.default_rng(4)
    HI, dI, N = 4, 64, 40
    q, kk = _ints(rng, (1, HI, dI)), _ints(rng, (N, dI))
    w = np.ones((1, HI), np.float32)
    one = np.ones((1, HI), np.float32)
    # t = 4*10 - 2: entry 9 ends at position 39, not yet visible -> 9 entries
    idx = _run(q, one, w, kk, np.ones(N, np.float32), t=38, k=16, want_scores=False)
    assert idx[0, :9].tolist() == list(range(9)) and np.all(idx[0, 9:] == -1)
    idx = _run(q, one, w, kk, np.ones(N, np.float32), t=39, k=16, want_scores=False)
    assert idx[0, :10].tolist() == list(range(10)) and np.all(idx[0, 10:] == -1)
    # t < m - 1: nothing visible
    idx = _run(q, one, w, kk, np.ones(N, np.float32), t=2, k=4, want_scores=False)
    assert np.all(idx == -1)


def test_permuting_entries_permutes_the_selection():
    rng = np.random.default_rng(5)
    HI, dI, N = 4, 64, 512
    q = rng.standard_normal((1, HI, dI))
    kk = rng.standard_normal((N, dI))
    w = rng.uniform(0, 1, (1, HI)).astype(np.float32)
    one = np.ones((1, HI), np.float32)
    idx, s = _run(q, one, w, kk, np.ones(N, np.float32), t=4 * N - 1, k=50)
    top = np.sort(s[0])[::-1][:51]
    assert len(np.unique(top)) == 51                    # no tie at the cut: order-free case
    perm = rng.permutation(N)                           # new row r holds old row perm[r]
    idx2 = _run(q, one, w, kk[perm], np.ones(N, np.float32), t=4 * N - 1, k=50, want_scores=False)
    assert sorted(perm[idx2[0]].tolist()) == idx[0].tolist()


def test_sequences_are_independent():
    rng = np.random.default_rng(6)
    HI, dI = 4, 64
    kk = _ints(rng, (300, dI))
    q = _ints(rng, (2, HI, dI))
    w = rng.uniform(0, 1, (2, HI)).astype(np.float32)
    one = np.ones((2, HI), np.float32)
    # two sequences: entries 0..99 and 100..299; query 1 reads only its own rows
    idx = oracle.indexer_topk(_e4m3(q), one, w, _e4m3(kk), np.ones(300, np.float32), [0, 100],
                              np.array([0, 1], np.int32), np.array([399, 799], np.int32),
                              H_I=HI, d_I=dI, m=4, k=10)
    alone = oracle.indexer_topk(_e4m3(q[1:]), one[1:], w[1:], _e4m3(kk[100:]),
                                np.ones(200, np.float32), [0], np.array([0], np.int32),
                                np.array([799], np.int32), H_I=HI, d_I=dI, m=4, k=10)
    assert idx[1].tolist() == alone[0].tolist()
