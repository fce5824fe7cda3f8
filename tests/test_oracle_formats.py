"""Pins for the oracle's number formats and RoPE (CPU only).

BF16 / E4M3 rounding is checked against torch's casts (library routines) and exhaustive
decode tables; saturation and RoPE against closed forms and invariants."""
import math

import numpy as np
import pytest
import torch

import oracle


def test_e4m3_decode_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.all(np.isnan(ours[nan]))
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(1)
    mag = 10.0 ** rng.uniform(-4.0, 2.64, 1_000_000)          # up to ~436 < 464
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    ours = oracle.e4m3_round(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch maps +-0 results of underflow with the input's sign; compare values then bits
    assert np.array_equal(oracle.e4m3_value(ours), oracle.e4m3_value(ref))
    nz = oracle.e4m3_value(ref) != 0
    assert np.array_equal(ours[nz], ref[nz])


def test_e4m3_ties_and_saturation_closed_form():
    # exact midpoints round to the even code
    assert oracle.e4m3_value(oracle.e4m3_round(np.array([1.0 + 1 / 16]))).item() == 1.0
    assert oracle.e4m3_value(oracle.e4m3_round(np.array([1.0 + 3 / 16]))).item() == 1.25
    assert oracle.e4m3_value(oracle.e4m3_round(np.array([2.0 ** -10]))).item() == 0.0
    assert oracle.e4m3_value(oracle.e4m3_round(np.array([3 * 2.0 ** -10]))).item() == 2.0 ** -8
    big = np.array([449.0, 464.0, 480.0, 1e6, 1e300, np.inf])
    assert np.all(oracle.e4m3_round(big) == 0x7E)
    assert np.all(oracle.e4m3_round(-big) == 0xFE)


def test_bf16_decode_exhaustive_and_encode_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ours = oracle.bf16_value(bits[::97])
    r = ref[::97]
    ok = ~np.isnan(r)
    assert np.array_equal(ours[ok], r[ok])
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(500_000),
        rng.standard_normal(200_000) * 1e-39,            # bf16 subnormals
        rng.standard_normal(100_000) * 1e37,
    ]).astype(np.float32)
    ours = oracle.bf16_round(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_overflow_and_ties():
    assert oracle.bf16_round(np.array([3.5e38]))[0] == 0x7F80     # rounds past max -> inf
    assert oracle.bf16_round(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80  # tie -> even (1.0)
    assert oracle.bf16_round(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82


@pytest.mark.parametrize("D", [128, 576])
def test_rope_closed_form_convention(D):
    theta = 10000.0
    # pair 0 rotates by pos * 1 rad; unit x-vector goes to (cos, sin)
    x = np.zeros(D)
    x[D - 64] = 1.0
    y = oracle.rope(x, 1.0, theta)
    assert y[D - 64] == pytest.approx(0.5403023058681398, abs=1e-15)
    assert y[D - 63] == pytest.approx(0.8414709848078965, abs=1e-15)
    # last pair (j = 31) rotates by pos * theta^(-62/64); unit y-vector -> (-sin, cos)
    x = np.zeros(D)
    x[D - 1] = 1.0
    pos = 1000.0
    ang = 10.0 ** -0.875                            # 1000 / 10000^(31/32)
    y = oracle.rope(x, pos, theta)
    assert y[D - 2] == pytest.approx(-math.sin(ang), abs=1e-14)
    assert y[D - 1] == pytest.approx(math.cos(ang), abs=1e-14)
    # the first D-64 dims are never touched
    x = np.random.default_rng(3).standard_normal(D)
    y = oracle.rope(x, 12345.0, theta)
    assert np.array_equal(y[: D - 64], x[: D - 64])


def test_rope_invariants():
    rng = np.random.default_rng(4)
    D = 128
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    for p in [0.0, 3.0, 1048575.0]:
        y = oracle.rope(q, p)
        assert np.linalg.norm(y) == pytest.approx(np.linalg.norm(q), rel=1e-13)   # rotation
        assert np.allclose(oracle.rope(y, -p), q, atol=1e-12)                     # inverse
    # <RoPE_a q, RoPE_b k> depends only on b - a
    d1 = oracle.rope(q, 100.0) @ oracle.rope(k, 137.0)
    d2 = oracle.rope(q, 1_000_000.0) @ oracle.rope(k, 1_000_037.0)
    assert d1 == pytest.approx(d2, abs=1e-9)
    assert oracle.rope(q, 0.0).tolist() == q.tolist()


def test_rmsnorm_closed_form():
    x = np.full(128, 3.0)
    y = oracle.rmsnorm(x, eps=0.0)
    assert np.allclose(y, 1.0, atol=1e-15)
    x = np.random.default_rng(5).standard_normal(576)
    ms = np.mean(x * x)
    y = oracle.rmsnorm(x, eps=1e-6)
    assert np.sum(y * y) == pytest.approx(576 * ms / (ms + 1e-6), rel=1e-13)


def test_entry_formats_round_trip():
    rng = np.random.default_rng(6)
    e = rng.standard_normal(576)
    row = oracle.entry_store(e, 1, 576)
    assert row.size == 656
    back = oracle.entry_load(row, 1, 576)
    for blk in range(4):
        sl = slice(128 * blk, 128 * blk + 128)
        scale = np.frombuffer(row[512 + 4 * blk: 516 + 4 * blk].tobytes(), np.float32)[0]
        assert scale == np.float32(np.abs(e[sl]).max() / 448.0)
        # the largest element lands on the top code
        assert np.max(np.abs(row[sl].astype(np.int32) & 0x7F)) == 0x7E
        # e4m3 relative step is 2^-3: error <= half a step of the value's binade
        err = np.abs(back[sl] - e[sl])
        assert np.all(err <= np.maximum(np.abs(e[sl]) * 2.0 ** -4, scale * 2.0 ** -10) + 1e-12)
    bf = oracle.bf16_value(oracle.bf16_round(e[512:]))
    assert np.array_equal(back[512:], bf)
    row0 = oracle.entry_store(e[:128], 0, 128)
    assert np.array_equal(oracle.entry_load(row0, 0, 128), oracle.bf16_value(oracle.bf16_round(e[:128])))
