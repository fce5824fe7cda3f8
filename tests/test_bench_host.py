"""Host-side helpers of the benchmark: which entries a step compresses, and the prefill
chunk's indexer FLOP count (checked against the count of causal query-entry pairs)."""
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
