"""Host-side helpers of the benchmark: which entries a step compresses, the prefill
chunk's indexer FLOP count (checked against the count of causal query-entry pairs), the
decode steps' algorithmic indexer bytes (checked against the key-row sizes), and the rule
that a recorded DRAM traffic figure is reported only while its kernel sources are
unchanged."""
import torch

import bench
from long_context_compressed_04_b200 import synth

P = "csa_prefill_8k_on_64k"


def test_prefill_step_compresses_the_entries_that_pool_new_tokens():
    wl = bench.make_workload(P, 0, "cpu")
    seq, ent = bench.step_items(wl, P, "cpu")
    # tokens 65536 .. 73727 are new; entry i pools positions up to (i + 1) * 4 - 1
    assert seq.tolist() == [0] * 2048
    assert ent.tolist() == list(range(16384, 18432))
    assert (16384 + 1) * 4 - 1 >= 65536 > 16384 * 4 - 1


def test_prefill_indexer_flops_count_every_causal_pair():
    wl = bench.make_workload(P, 0, "cpu")
    # query at position t sees floor((t + 1) / 4) entries, t = 65536 .. 73727
    pairs = sum((t + 1) // 4 for t in range(65536, 65536 + 8192))
    assert pairs == 142_604_288
    assert bench.indexer_flops(wl) == pairs * 64 * 128 * 2


def test_decode_step_compresses_the_newest_entry_of_each_sequence():
    wl = synth.make_workload("t", B=3, T=[4096, 5001, 3003], D=128, H=16, m=4, span=8,
                             H_I=4, d_I=64, k=64, seed=3, device="cpu")
    seq, ent = bench.step_items(wl, "csa_decode_128k_b32", "cpu")
    assert seq.tolist() == [0, 1, 2]
    assert ent.tolist() == [4096 // 4 - 1, 5001 // 4 - 1, 3003 // 4 - 1]
    assert torch.equal(ent, (wl.n_ent - 1).to(torch.int32))


def _decode_shape(**kw):
    # the attributes algorithmic_bytes reads, without allocating a 1M-token workload
    from types import SimpleNamespace
    B = kw.get("B", 8)
    base = dict(B=B, Q=B, q_pos=torch.full((B,), (1 << 20) - 1, dtype=torch.int32), m=4,
                fmt=1, D=576, W=128, H=128, span=8, H_I=64, d_I=128, k=1024, kI4=None)
    base.update(kw)
    return SimpleNamespace(**base)


def test_headline_indexer_bytes_are_every_key_row_and_scale():
    # 8 queries x 262,144 visible entries x (128 fp8 bytes + 4 scale bytes), and 64 heads x
    # (128 bytes + query scale + weight) per query
    _, keys = bench.algorithmic_bytes(_decode_shape())
    assert keys == 8 * 262_144 * 132 + 8 * 64 * 136 == 276_893_696


def test_mxfp4_indexer_bytes_are_packed_codes_and_block_scales():
    # 64 packed bytes + 4 UE8M0 scale bytes per key; the heads the same plus a fp32 weight
    _, keys = bench.algorithmic_bytes(_decode_shape(kI4=object()))
    assert keys == 8 * 262_144 * 68 + 8 * 64 * 72 == 142_643_200


def test_measured_traffic_only_while_the_sources_are_unchanged(monkeypatch):
    files = ["long_context_compressed_04_b200/csrc/topk.cu"]
    import hashlib, os
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(os.path.dirname(bench.__file__), f), "rb").read())
    good = {"bytes": 123, "files": files, "sha": h.hexdigest()[:16]}
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("w", "k"), good)
    assert bench.measured_traffic("w", "k") == 123
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("w", "k"), dict(good, sha="0" * 16))
    assert bench.measured_traffic("w", "k") is None
    assert bench.measured_traffic("no such workload", "k") is None
