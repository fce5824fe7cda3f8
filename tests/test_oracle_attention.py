"""Pins for the oracle's shared-KV MQA attention with window, sink and partial RoPE.

Closed forms (one key with a sink; uniform logits), limits (sink -> -inf is plain softmax,
checked against torch's scaled_dot_product_attention; sink -> +inf drives the output to 0),
sparse-with-every-entry equals dense, padding, visibility, and the shift invariance of the
whole compress + attend pipeline, which fixes the sign of the inverse RoPE."""
import math

import numpy as np
import pytest
import torch

import oracle


def _bits(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _vals(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


def _problem(T=300, D=128, H=4, n_ent=None, fmt=0, seed=0, m=4):
    rng = np.random.default_rng(seed)
    n_ent = T // m if n_ent is None else n_ent
    kv = _bits(rng.standard_normal((T, D)))
    rb = oracle.entry_row_bytes(fmt, D)
    ents = np.stack([oracle.entry_store(rng.standard_normal(D), fmt, D) for _ in range(n_ent)]) \
        if n_ent else np.zeros((0, rb), np.uint8)
    q = _bits(rng.standard_normal((1, H, D)))
    sink = rng.standard_normal(H).astype(np.float32)
    return kv, ents, q, sink


def _attn(kv, ents, q, sink, t, idx=None, *, D, H, W=128, m=4, fmt=0, scale=None):
    return oracle.attention(q, ents, fmt, [0], kv, [0], [0], [0], [t], idx, sink, H=H, D=D,
                            W=W, m=m, scale=scale)[0]


def _keys(kv, ents, t, ids, *, D, W, fmt=0):
    rows = [oracle.entry_load(ents[i], fmt, D) for i in ids]
    for p in range(max(0, t - W + 1), t + 1) if W else []:
        rows.append(oracle.rope(oracle.rmsnorm(_vals(kv[p])), float(p)))
    return np.array(rows).reshape(-1, D)


def test_single_entry_with_sink_closed_form():
    D, H = 128, 3
    kv, ents, q, _ = _problem(D=D, H=H, n_ent=1, seed=1)
    sink = np.array([-1.0, 0.0, 2.5], np.float32)
    t = 3                                      # entry 0 (block 0..3) is visible at t = 3
    o = _attn(kv, ents, q, sink, t, np.array([[0]], np.int32), D=D, H=H, W=0)
    v = oracle.entry_load(ents[0], 0, D)
    for h in range(H):
        l = (oracle.rope(_vals(q[0, h]), float(t)) @ v) / math.sqrt(D)
        want = oracle.rope(v / (1.0 + math.exp(float(sink[h]) - l)), -float(t))
        assert np.allclose(o[h], want, atol=1e-13)


@pytest.mark.parametrize("fmt,D", [(0, 128), (1, 576)])
def test_sink_to_minus_inf_is_plain_softmax_attention(fmt, D):
    H, T = 4, 400
    kv, ents, q, _ = _problem(T=T, D=D, H=H, fmt=fmt, seed=2)
    t = T - 1
    rng = np.random.default_rng(3)
    idx = np.sort(rng.choice(T // 4, 40, replace=False)).astype(np.int32)[None]
    sink = np.full(H, -1e30, np.float32)
    o = _attn(kv, ents, q, sink, t, idx, D=D, H=H, fmt=fmt)
    K = torch.from_numpy(_keys(kv, ents, t, idx[0], D=D, W=128, fmt=fmt))
    for h in range(H):
        qh = torch.from_numpy(oracle.rope(_vals(q[0, h]), float(t)))
        ref = torch.nn.functional.scaled_dot_product_attention(
            qh[None, None, None], K[None, None], K[None, None], scale=1.0 / math.sqrt(D))[0, 0, 0]
        assert np.allclose(o[h], oracle.rope(ref.numpy(), -float(t)), atol=1e-12)


def test_sink_to_plus_inf_drives_output_to_zero():
    D, H = 128, 2
    kv, ents, q, _ = _problem(D=D, H=H, seed=4)
    o = _attn(kv, ents, q, np.full(H, 1e4, np.float32), 299, None, D=D, H=H)
    assert np.max(np.abs(o)) < 1e-30
    o80 = _attn(kv, ents, q, np.full(H, 80.0, np.float32), 299, None, D=D, H=H)
    assert np.max(np.abs(o80)) < 1e-20


def test_uniform_logits_give_scaled_mean():
    D, H, T = 128, 2, 200
    kv, ents, _, sink = _problem(T=T, D=D, H=H, seed=5)
    q = _bits(np.zeros((1, H, D)))
    t = T - 1
    o = _attn(kv, ents, q, sink, t, None, D=D, H=H)
    K = _keys(kv, ents, t, range(T // 4), D=D, W=128)
    n = K.shape[0]
    assert n == T // 4 + 128
    for h in range(H):
        want = oracle.rope(K.mean(axis=0) * n / (n + math.exp(float(sink[h]))), -float(t))
        assert np.allclose(o[h], want, atol=1e-13)


def test_sparse_with_every_entry_equals_dense_and_padding_is_ignored():
    D, H, T = 128, 4, 300
    kv, ents, q, sink = _problem(T=T, D=D, H=H, seed=6)
    t = T - 1
    n = (t + 1) // 4
    dense = _attn(kv, ents, q, sink, t, None, D=D, H=H)
    full = np.arange(n, dtype=np.int32)[None]
    assert np.allclose(_attn(kv, ents, q, sink, t, full, D=D, H=H), dense, atol=1e-13)
    padded = np.concatenate([full, -np.ones((1, 9), np.int32)], axis=1)
    assert np.allclose(_attn(kv, ents, q, sink, t, padded, D=D, H=H), dense, atol=1e-13)
    shuffled = np.random.default_rng(7).permutation(full[0])[None].astype(np.int32)
    assert np.allclose(_attn(kv, ents, q, sink, t, shuffled, D=D, H=H), dense, atol=1e-13)


def test_dense_visibility_and_short_window():
    D, H, m = 128, 2, 128
    T = 128 * 3 + 50
    kv, ents, q, sink = _problem(T=T, D=D, H=H, m=m, seed=8)
    # at t = 382 only entries 0 and 1 are complete; entry 2 ends at 383
    t = 382
    o = _attn(kv, ents, q, sink, t, None, D=D, H=H, m=m)
    o2 = oracle.attention(q, ents[:2], 0, [0], kv, [0], [0], [0], [t], None, sink, H=H, D=D,
                          W=128, m=m)[0]
    assert np.array_equal(o, o2)
    # a query at t = 5 sees no entry and a window of 6 tokens
    o = _attn(kv, ents, q, sink, 5, None, D=D, H=H, m=m)
    K = _keys(kv, ents, 5, [], D=D, W=128)
    assert K.shape[0] == 6
    for h in range(H):
        qh = oracle.rope(_vals(q[0, h]), 5.0)
        lg = K @ qh / math.sqrt(D)
        M = max(lg.max(), float(sink[h]))
        p = np.exp(lg - M)
        want = oracle.rope((p @ K) / (math.exp(float(sink[h]) - M) + p.sum()), -5.0)
        assert np.allclose(o[h], want, atol=1e-13)
    with pytest.raises(ValueError):   # an index past the visible entries is an error
        oracle.attention(q, ents, 0, [0], kv, [0], [0], [0], [382], np.array([[2]], np.int32),
                         sink, H=H, D=D, W=128, m=m)


def test_shift_invariance_of_compress_then_attend():
    # Prepend 4*s tokens: every position moves by delta = 4*s.  Entries keep pooling the same
    # raw tokens, the window holds the same rows, so the output must not change.  A wrong
    # sign in the inverse RoPE, or RoPE at a wrong position, breaks this.
    D, H, T, s = 128, 4, 260, 25
    delta = 4 * s
    rng = np.random.default_rng(9)
    kv = _bits(rng.standard_normal((T + delta, D)))
    gate = _bits(rng.standard_normal((T + delta, D)))
    bias = (rng.standard_normal((8, D)) * 0.1).astype(np.float32)
    q = _bits(rng.standard_normal((1, H, D)))
    sink = rng.standard_normal(H).astype(np.float32)
    ids = np.array([1, 5, 9, 30, 64], np.int32)       # entries >= 1 pool only stored tokens
    outs = []
    for shift in (0, delta):
        base = delta - shift                          # first stored position maps to row base
        n_ent = (T + shift) // 4
        ents, _ = oracle.compress(kv[base:], gate[base:], bias, [0], [0], [0],
                                  np.zeros(n_ent, np.int32), np.arange(n_ent, dtype=np.int32),
                                  m=4, span=8, D=D, n_entry_rows=n_ent)
        idx = (ids + shift // 4)[None].astype(np.int32)
        outs.append(oracle.attention(q, ents, 0, [0], kv[base:], [0], [0], [0], [T + shift - 1],
                                     idx, sink, H=H, D=D, W=128, m=4)[0])
    # entries are stored in bf16 after RoPE, so the two runs differ only by storage rounding
    # (a few 1e-4 here); a wrong rotation of the output moves the RoPE dims by O(0.1)
    assert np.allclose(outs[0], outs[1], atol=1e-3)
    wrong = np.stack([oracle.rope(o, float(delta)) for o in outs[1]])
    assert np.max(np.abs(wrong[:, D - 64:] - outs[0][:, D - 64:])) > 3e-2


def test_window_rows_and_entries_are_both_attended():
    # An entry covering positions inside the window is still a separate key.
    D, H, T = 128, 2, 64
    kv, ents, q, sink = _problem(T=T, D=D, H=H, seed=10)
    t = T - 1
    o = _attn(kv, ents, q, sink, t, np.array([[15]], np.int32), D=D, H=H)
    K = _keys(kv, ents, t, [15], D=D, W=128)
    assert K.shape[0] == 1 + 64
    for h in range(H):
        qh = oracle.rope(_vals(q[0, h]), float(t))
        lg = K @ qh / math.sqrt(D)
        M = max(lg.max(), float(sink[h]))
        p = np.exp(lg - M)
        want = oracle.rope((p @ K) / (math.exp(float(sink[h]) - M) + p.sum()), -float(t))
        assert np.allclose(o[h], want, atol=1e-13)
