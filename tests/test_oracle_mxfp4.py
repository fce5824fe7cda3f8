"""Pins for the oracle's MXFP4 lightning indexer and BF16 selector scores (CPU only).

"DeepSeek-V4 深度分析报告" Figure 2 / "其他注意力技术细节" (the indexer computes in FP4) and
section 3.4 (MXFP4 on the QK path of CSA; indexer scores quantised FP32 -> BF16 before the
top-k).  The E2M1 and E8M0 decodes are checked exhaustively against library dtypes
(ml_dtypes, torch); the score against the separately pinned FP8 oracle on inputs that both
formats hold exactly, and against an fp64 computation from the library decodes with wide
block-scale spreads; the BF16 selection against torch's BF16 cast and a brute-force
selection."""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle


def test_e2m1_decode_exhaustive_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = oracle.e2m1_value(codes)
    assert np.array_equal(ours, ref)
    # the high nibble is ignored by the decode
    assert np.array_equal(oracle.e2m1_value(codes | 0xA0), ref)
    assert ours.max() == 6.0 and ours[1] == 0.5


def test_e8m0_decode_exhaustive_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    ours = oracle.e8m0_value(codes)
    assert np.isnan(ref[255]) and np.isnan(ours[255])
    assert np.array_equal(ours[:255], ref[:255])
    assert ours[127] == 1.0 and ours[0] == 2.0 ** -127 and ours[254] == 2.0 ** 127


def _pack(codes):
    """[..., d] 4-bit codes -> [..., d/2] bytes, element 2j in the low nibble."""
    lo = codes[..., 0::2].astype(np.uint8)
    hi = codes[..., 1::2].astype(np.uint8)
    return (lo | (hi << 4)).astype(np.uint8)


def _values(codes):
    return codes.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _case(rng, Q, HI, dI, T, exp_lo, exp_hi, m=4):
    B = len(T)
    n_ent = [t // m for t in T]
    ent_off = np.concatenate([[0], np.cumsum(n_ent)[:-1]]).astype(np.int64)
    rows = int(sum(n_ent))
    qc = rng.integers(0, 16, (Q, HI, dI)).astype(np.uint8)
    kc = rng.integers(0, 16, (rows, dI)).astype(np.uint8)
    qe = rng.integers(exp_lo, exp_hi + 1, (Q, HI, dI // 32)).astype(np.uint8)
    ke = rng.integers(exp_lo, exp_hi + 1, (rows, dI // 32)).astype(np.uint8)
    w = rng.standard_normal((Q, HI)).astype(np.float32)
    q_seq = rng.integers(0, B, Q).astype(np.int32)
    q_pos = np.array([rng.integers(0, T[b]) for b in q_seq], np.int32)
    q_pos[0] = T[q_seq[0]] - 1
    return dict(qc=qc, kc=kc, qe=qe, ke=ke, w=w, ent_off=ent_off, q_seq=q_seq, q_pos=q_pos,
                rows=rows, m=m)


@pytest.mark.parametrize("dI", [128, 64])
def test_scores_match_the_fp8_oracle_on_common_values(dI):
    # block exponents within +-2: every element value * block scale is an e4m3 value, so the
    # FP8 oracle (unit row and head scales) scores the same vectors; the two oracles must
    # agree bit for bit.  The test packs the nibbles itself (element 2j low).
    rng = np.random.default_rng(7)
    HI, k = 8, 64
    c = _case(rng, Q=6, HI=HI, dI=dI, T=[9001, 4000, 13], exp_lo=125, exp_hi=129)
    qv = _values(c["qc"]) * np.repeat(2.0 ** (c["qe"].astype(np.float64) - 127), 32, axis=-1)
    kv = _values(c["kc"]) * np.repeat(2.0 ** (c["ke"].astype(np.float64) - 127), 32, axis=-1)
    q8 = torch.from_numpy(qv.astype(np.float32)).to(torch.float8_e4m3fn)
    k8 = torch.from_numpy(kv.astype(np.float32)).to(torch.float8_e4m3fn)
    assert np.array_equal(q8.to(torch.float64).numpy(), qv)
    assert np.array_equal(k8.to(torch.float64).numpy(), kv)
    ones_q = np.ones((qv.shape[0], HI), np.float32)
    ones_k = np.ones(c["rows"], np.float32)
    i8, s8 = oracle.indexer_topk(q8.view(torch.uint8).numpy(), ones_q, c["w"],
                                 k8.view(torch.uint8).numpy(), ones_k, c["ent_off"], c["q_seq"],
                                 c["q_pos"], H_I=HI, d_I=dI, m=c["m"], k=k, want_scores=True)
    i4, s4 = oracle.indexer_topk_mxfp4(_pack(c["qc"]), c["qe"], c["w"], _pack(c["kc"]), c["ke"],
                                       c["ent_off"], c["q_seq"], c["q_pos"], H_I=HI, d_I=dI,
                                       m=c["m"], k=k, want_scores=True)
    assert np.array_equal(i4, i8)
    vis = ~np.isnan(s8)
    assert np.array_equal(vis, ~np.isnan(s4))
    assert np.array_equal(s4[vis].view(np.int32), s8[vis].view(np.int32))


def test_wide_scale_spread_against_fp64_from_library_decodes():
    # one head, w = 1: the score is max(dot, 0) rounded to fp32.  Block exponents spread over
    # 2^-10 .. 2^10 on each side.  A block's dot is a multiple of 1/4 below 2^11 (13 bits)
    # times 2^(eq + ek - 254), the exponents of the four blocks lie within 40 of each other,
    # so their fp64 sum is exact and the float32 conversion is the only rounding.  The
    # reference is formed from the library decodes.
    rng = np.random.default_rng(8)
    dI = 128
    c = _case(rng, Q=4, HI=1, dI=dI, T=[4000], exp_lo=117, exp_hi=137)
    c["w"][:] = 1.0
    _, s4 = oracle.indexer_topk_mxfp4(_pack(c["qc"]), c["qe"], c["w"], _pack(c["kc"]), c["ke"],
                                      c["ent_off"], c["q_seq"], c["q_pos"], H_I=1, d_I=dI,
                                      m=c["m"], k=16, want_scores=True)
    qv, kv = _values(c["qc"]), _values(c["kc"])
    qs = torch.from_numpy(c["qe"]).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    ks = torch.from_numpy(c["ke"]).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    checked = rounded = 0
    for qq in range(4):
        n = (int(c["q_pos"][qq]) + 1) // c["m"]
        for i in range(n):
            row = int(c["ent_off"][c["q_seq"][qq]]) + i
            blocks = [float(np.dot(qv[qq, 0, 32 * b:32 * b + 32], kv[row, 32 * b:32 * b + 32]))
                      * qs[qq, 0, b] * ks[row, b] for b in range(dI // 32)]
            exact = sum(blocks)
            ref = np.float32(max(exact, 0.0))
            assert s4[qq, i].view(np.int32) == ref.view(np.int32), (qq, i)
            checked += 1
            rounded += float(ref) != max(exact, 0.0)
    assert checked > 1000 and rounded > 100   # the fp32 rounding is exercised


def test_bf16_selection_is_the_top_k_of_torch_rounded_scores():
    # integer-ish inputs make many scores collide once rounded to 8 significant bits
    rng = np.random.default_rng(9)
    HI, dI, k = 4, 64, 100
    c = _case(rng, Q=5, HI=HI, dI=dI, T=[12000, 3001], exp_lo=126, exp_hi=128)
    args = (_pack(c["qc"]), c["qe"], c["w"], _pack(c["kc"]), c["ke"], c["ent_off"], c["q_seq"],
            c["q_pos"])
    kw = dict(H_I=HI, d_I=dI, m=c["m"], k=k, want_scores=True)
    i32, s32 = oracle.indexer_topk_mxfp4(*args, select_bf16=False, **kw)
    i16, s16 = oracle.indexer_topk_mxfp4(*args, select_bf16=True, **kw)
    ties = 0
    for qq in range(5):
        n = (int(c["q_pos"][qq]) + 1) // c["m"]
        r = torch.from_numpy(s32[qq, :n].copy()).to(torch.bfloat16).to(torch.float32).numpy()
        assert np.array_equal(s16[qq, :n].view(np.int32), r.view(np.int32))
        order = np.lexsort((np.arange(n), -r.astype(np.float64)))
        want = np.sort(order[:k]) if n > k else np.arange(n)
        got = i16[qq][i16[qq] >= 0]
        assert np.array_equal(got, want), qq
        ties += n - np.unique(r).size
    assert ties > 1000
    # the FP32 and BF16 selections are different sets here (the rounding matters)
    assert not np.array_equal(i32, i16)


def test_nan_block_scale_and_nan_weight():
    # a NaN block scale makes that entry's dot products NaN, which max(., 0) (fmaxf) maps
    # to 0, as in the FP8 indexer: the entry scores +0.  A NaN head weight makes the score
    # NaN, which is reported.
    rng = np.random.default_rng(10)
    c = _case(rng, Q=2, HI=2, dI=64, T=[800], exp_lo=126, exp_hi=128)
    c["ke"][5, 1] = 255
    c["q_pos"][:] = 799
    args = [_pack(c["qc"]), c["qe"], c["w"], _pack(c["kc"]), c["ke"], c["ent_off"], c["q_seq"],
            c["q_pos"]]
    _, s = oracle.indexer_topk_mxfp4(*args, H_I=2, d_I=64, m=4, k=8, want_scores=True)
    assert np.all(s[:, 5].view(np.int32) == 0)
    args[2] = c["w"].copy()
    args[2][1, 0] = np.nan
    with pytest.raises(ValueError, match="-2"):
        oracle.indexer_topk_mxfp4(*args, H_I=2, d_I=64, m=4, k=8)
