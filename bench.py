"""Benchmark of the CSA / HCA decode hot path on B200.

One step = one pass of the whole hot path over one batch: compress each sequence's newest
entry, lightning indexer + top-k (CSA), sparse (CSA) or dense (HCA) attention.  The
default workload is CSA decode at 1,048,576 tokens: 8 sequences, 128 query heads over
576-dim entries (512 FP8 channels with 1x128 scales + 64 bf16 RoPE channels), a 64 x 128
FP8 indexer and top-1024.  The same run also measures CSA decode with 32 sequences of
131072 +- 1024 tokens (64 heads of dim 128, top-512) and HCA decode with 16 sequences of
1,048,576 tokens, reported under "also".  Inputs are synthetic and seeded; the compressed
cache is built with the library itself before timing.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--no-also]
                  [--impl reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own batch (sequences
shard across GPUs with no data-path collective; weak scaling); the timed region is
bracketed by barriers and device syncs and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "CSA/HCA decode query-tokens/s at 128K–1M ctx; % of HBM roofline"
UNIT = "query-tokens/s"

WORKLOADS = {
    "csa_decode_128k_b32": dict(kind="csa", B=32, T=131072, jitter=1024, D=128, H=64, H_I=64,
                                d_I=128, k=512, fmt=0),
    "hca_decode_1m_b16": dict(kind="hca", B=16, T=1 << 20, jitter=0, D=128, H=64, fmt=0),
    "csa_decode_1m_b8_fp8": dict(kind="csa", B=8, T=1 << 20, jitter=0, D=576, H=128, H_I=64,
                                 d_I=128, k=1024, fmt=1),
    # the 1M decode step with the pages' FP4 indexer: MXFP4 query heads and keys (N(0,1)
    # quantised per 32-element block) and the top-k taken on BF16-rounded scores
    "csa_decode_1m_b8_mxfp4": dict(kind="csa", B=8, T=1 << 20, jitter=0, D=576, H=128,
                                   H_I=64, d_I=128, k=1024, fmt=1, indexer_fmt="mxfp4",
                                   select_bf16=True),
    # a causal prefill chunk: 8192 new query tokens after 65536 prior tokens; the step
    # compresses the 2048 entries that pool new tokens, then scores, selects and attends
    "csa_prefill_8k_on_64k": dict(kind="csa_prefill", B=1, T=65536 + 8192, jitter=0, D=128,
                                  H=64, H_I=64, d_I=128, k=1024, fmt=0, n_new=8192),
}


# DRAM traffic (read + write, bytes per launch) of the dominant kernel from the ncu captures
# summarised in profiles/ (the launch lists of the two 1M workloads), valid only while the kernel's
# sources are byte-identical to the ones captured (sha256 of the files, first 16 hex digits).
MEASURED_TRAFFIC = {
    ("csa_decode_1m_b8_fp8", "indexer_score_tc"): {
        "bytes": 281_108_224,
        "files": ["long_context_compressed_04_b200/csrc/indexer_tc.cu",
                  "long_context_compressed_04_b200/csrc/indexer_items.cuh",
                  "long_context_compressed_04_b200/csrc/sm100.cuh",
                  "long_context_compressed_04_b200/csrc/common.cuh"],
        "sha": "381e8d13a9b6edc5",
    },
    ("csa_decode_1m_b8_mxfp4", "indexer_score_fp4"): {
        "bytes": 146_638_080,
        "files": ["long_context_compressed_04_b200/csrc/indexer_fp4.cu",
                  "long_context_compressed_04_b200/csrc/indexer_items.cuh",
                  "long_context_compressed_04_b200/csrc/sm100.cuh",
                  "long_context_compressed_04_b200/csrc/common.cuh"],
        "sha": "461b40acd17541e5",
    },
}


def measured_traffic(workload: str, kernel: str):
    import hashlib
    rec = MEASURED_TRAFFIC.get((workload, kernel))
    if not rec:
        return None
    h = hashlib.sha256()
    for f in rec["files"]:
        h.update(open(os.path.join(HERE, f), "rb").read())
    return rec["bytes"] if h.hexdigest()[:16] == rec["sha"] else None


def _peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _tensor_peak_fp8():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return round(2.0 * float(d["bf16_tflops_sustained"]), 1), \
            "measured bf16_tflops_sustained x 2 (nominal fp8 / bf16 ratio)"
    return round(2.0 * 1400.0, 1), "fallback sustained bf16 1400 TFLOP/s x 2 (nominal fp8 / bf16 ratio)"


def rank_lengths(name: str, rank: int):
    """Context lengths of the sequences rank `rank` owns: every rank draws its own jittered
    lengths (and its own inputs, seeded by the rank), so the ranks' sequences are disjoint
    units of the same shape (weak scaling, no data-path collective)."""
    from long_context_compressed_04_b200 import synth
    c = WORKLOADS[name]
    if c["jitter"]:
        return synth.jittered_lengths(c["B"], c["T"], c["jitter"], 1000 + rank)
    return [c["T"]] * c["B"]


def max_over_ranks(x: float, dist, device) -> float:
    """The largest `x` over the ranks (x itself on one process): a run's time is that of its
    slowest rank."""
    t = torch.tensor([x], device=device, dtype=torch.float64)
    if dist:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, steps: int, ms: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return units_per_rank * world * steps / (ms / 1e3)


def make_workload(name: str, rank: int, device, keep_raw=None):
    from long_context_compressed_04_b200 import synth
    c = WORKLOADS[name]
    if c["kind"] == "csa_prefill":
        return synth.make_workload(name, B=c["B"], T=c["T"], D=c["D"], H=c["H"], m=4, span=8,
                                   W=128, fmt=c["fmt"], H_I=c["H_I"], d_I=c["d_I"], k=c["k"],
                                   indexer="fp8", queries="prefill", n_new=c["n_new"],
                                   seed=rank, device=device)
    T = rank_lengths(name, rank) if c["jitter"] else c["T"]
    if c["kind"] == "csa":
        fp4 = c.get("indexer_fmt") == "mxfp4"
        wl = synth.make_workload(name, B=c["B"], T=T, D=c["D"], H=c["H"], m=4, span=8, W=128,
                                 fmt=c["fmt"], H_I=c["H_I"], d_I=c["d_I"], k=c["k"],
                                 indexer="int" if fp4 else "fp8", keep_raw=keep_raw, seed=rank,
                                 device=device)
        if fp4:
            wl.qI4, wl.qsf4, wl.kI4, wl.ksf4 = synth.mxfp4_indexer(wl, "normal", seed=rank)
            wl.select_bf16 = bool(c.get("select_bf16", False))
            wl.kI = wl.ks = wl.qI = wl.qs = None
        return wl
    return synth.make_workload(name, B=c["B"], T=T, D=c["D"], H=c["H"], m=128, span=128, W=128,
                               fmt=c["fmt"], keep_raw=keep_raw, seed=rank, device=device)


def new_tokens(wl, name):
    """Tokens that are new in one step: the last one of every sequence (decode), or the
    last n_new of every sequence (prefill)."""
    return WORKLOADS[name].get("n_new", 1)


def step_items(wl, name, device):
    """(item_seq, item_ent): the entries one step compresses, i.e. those that pool a new
    token (entry i pools positions up to (i+1)m - 1)."""
    from long_context_compressed_04_b200 import pipeline
    nn = new_tokens(wl, name)
    if nn == 1:
        return pipeline.newest_entry_items(wl, device)
    seqs, ents = [], []
    for b in range(wl.B):
        T_b = int(wl.T[b]) if wl.T.dim() else int(wl.T)
        first = T_b - nn
        i0 = max(0, -(-(first + 1) // wl.m) - 1)
        n_b = int(wl.n_ent[b])
        ents.append(torch.arange(i0, n_b, dtype=torch.int32))
        seqs.append(torch.full((n_b - i0,), b, dtype=torch.int32))
    return torch.cat(seqs).to(device), torch.cat(ents).to(device)


def indexer_flops(wl):
    """Multiply-adds x 2 of the indexer's dot products: every visible (query, entry) pair,
    every indexer head."""
    n_vis = ((wl.q_pos.cpu().to(torch.int64) + 1) // wl.m)
    return int(n_vis.sum()) * wl.H_I * wl.d_I * 2


def algorithmic_bytes(wl):
    """Bytes the method must move per step (each counted once): indexer keys + scales of
    every visible entry, the selected (or all, for HCA) entry rows, the window's raw rows,
    q, out and the index sets; plus the newest block's raw rows for compression."""
    from long_context_compressed_04_b200 import csa_entry_row_bytes
    n_vis = ((wl.q_pos.cpu().to(torch.int64) + 1) // wl.m)
    rb = csa_entry_row_bytes(wl.fmt, wl.D)
    win = torch.clamp(wl.q_pos.cpu().to(torch.int64) + 1, max=wl.W)
    qo = wl.Q * wl.H * wl.D * 2 * 2
    comp = wl.B * (wl.span * wl.D * 2 * 2 + rb)
    if wl.H_I and wl.kI4 is not None:
        # MXFP4: d_I / 2 element bytes + d_I / 32 scale bytes per key; the same per head
        # plus its fp32 weight
        row4 = wl.d_I // 2 + wl.d_I // 32
        keys = int(n_vis.sum()) * row4 + wl.Q * wl.H_I * (row4 + 4)
        sel = int(torch.clamp(n_vis, max=wl.k).sum()) * rb + wl.Q * wl.k * 4
    elif wl.H_I:
        keys = int(n_vis.sum()) * (wl.d_I + 4) + wl.Q * wl.H_I * (wl.d_I + 8)
        sel = int(torch.clamp(n_vis, max=wl.k).sum()) * rb + wl.Q * wl.k * 4
    else:
        keys = 0
        sel = int(n_vis.sum()) * rb
    total = keys + sel + int(win.sum()) * wl.D * 2 + qo + comp
    return total, keys


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_index_for_smi(dev: int) -> str:
    try:
        props = torch.cuda.get_device_properties(dev)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            dv = getattr(props, "pci_device_id", 0)
            return f"{dom:08x}:{bus:02x}:{dv:02x}.0"
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[dev]
    return str(dev)


CPU_SAMPLE_SEQS = {"csa_decode_128k_b32": 32, "hca_decode_1m_b16": 16, "csa_decode_1m_b8_fp8": 8,
                   "csa_decode_1m_b8_mxfp4": 8,
                   "csa_prefill_8k_on_64k": 64}   # prefill: sampled queries of the chunk


def cpu_baseline(name: str, n_seq: int | None = None):
    """The oracle, as it stands, on a bounded sample of the workload: n_seq sequences of
    the workload's shape, one decode step each (compress the newest entry, score every
    visible entry and select, attend).  The sample's cache rows are synthetic stored-format
    rows (untimed set-up); the timed step recompresses the newest entry itself."""
    n_seq = n_seq or CPU_SAMPLE_SEQS[name]
    import numpy as np
    import oracle
    from oracle import workload as _orc
    from long_context_compressed_04_b200 import synth

    c = WORKLOADS[name]
    if c["kind"] == "csa_prefill":
        # the chunk's entry compression plus n_seq of its queries, spread over the chunk
        import dataclasses
        wl = make_workload(name, 0, "cpu")
        sel = torch.linspace(0, wl.Q - 1, n_seq).round().long()
        ws = dataclasses.replace(wl, q_seq=wl.q_seq[sel], q_pos=wl.q_pos[sel], q=wl.q[sel],
                                 qI=wl.qI[sel], qs=wl.qs[sel], w=wl.w[sel])
        rows, _ = _orc.compress(wl)                      # the cache (untimed set-up)
        iseq, ient = step_items(wl, name, "cpu")
        t0 = time.perf_counter()
        _orc.compress(wl, iseq.numpy(), ient.numpy(), entries=rows)
        idx = _orc.indexer(ws, want_scores=False)
        _orc.attention(ws, rows, idx)
        dt = time.perf_counter() - t0
        return {"value": n_seq / dt, "unit": UNIT, "cores": min(oracle.num_threads(), n_seq),
                "kind": "oracle",
                "sample": f"{n_seq} of the {wl.Q} prefill queries of {name} with the chunk's "
                          f"{int(iseq.numel())} new entries compressed (indexer over every "
                          f"visible entry, top-k, attention), {dt:.2f} s"}
    T = synth.jittered_lengths(n_seq, c["T"], c["jitter"], 99) if c["jitter"] else [c["T"]] * n_seq
    fp4 = None
    if c["kind"] == "csa":
        wl = synth.make_workload(name, B=n_seq, T=T, D=c["D"], H=c["H"], m=4, span=8, W=128,
                                 fmt=c["fmt"], H_I=c["H_I"], d_I=c["d_I"], k=c["k"],
                                 indexer="fp8", keep_raw=256, seed=7)
        if c.get("indexer_fmt") == "mxfp4":
            fp4 = synth.mxfp4_indexer(wl, "normal", seed=7)
    else:
        wl = synth.make_workload(name, B=n_seq, T=T, D=c["D"], H=c["H"], m=128, span=128, W=128,
                                 fmt=c["fmt"], keep_raw=256, seed=7)
    # cache of entries for the sample (the raw store keeps only the tail, so the cache is
    # filled with stored-format rows drawn directly; the step recompresses the newest one)
    g = torch.Generator().manual_seed(5)
    rows = synth.random_entries(max(wl.ent_rows, 1), wl.fmt, wl.D, g, "cpu").numpy().copy()
    n = _orc.i64(wl.n_ent)
    item_seq = np.arange(wl.B, dtype=np.int32)
    item_ent = (n - 1).astype(np.int32)
    t0 = time.perf_counter()
    oracle.compress(_orc.u16(wl.kv), _orc.u16(wl.gate), _orc.f32(wl.bias), _orc.i64(wl.kv_off),
                    _orc.i64(wl.kv_pos0), _orc.i64(wl.ent_off), item_seq, item_ent, m=wl.m,
                    span=wl.span, D=wl.D, fmt=wl.fmt, entries=rows)
    if fp4 is not None:
        idx = _orc.indexer_mxfp4(wl, fp4, select_bf16=bool(c.get("select_bf16")),
                                 want_scores=False)
    else:
        idx = _orc.indexer(wl, want_scores=False) if wl.H_I else None
    _orc.attention(wl, rows, idx)
    dt = time.perf_counter() - t0
    return {"value": wl.Q / dt, "unit": UNIT, "cores": min(oracle.num_threads(), wl.Q),
            "kind": "oracle",
            "sample": f"{wl.Q} decode queries of {name} (one step each: newest-entry compress, "
                      f"indexer over all visible entries, top-k, attention), {dt:.2f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    samples = []
    for _ in range(args.warmup):
        cpu_baseline(args.workload, n_seq=1)
    for _ in range(args.steps):
        samples.append(cpu_baseline(args.workload, n_seq=1))
    v = sum(s["value"] for s in samples) / len(samples)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, **WORKLOADS[args.workload]},
            "cpu_baseline": {"value": v, "unit": UNIT, "kind": "oracle",
                             "cores": samples[0]["cores"], "sample": samples[0]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


DEFAULT_WORKLOAD = "csa_decode_1m_b8_fp8"
# measured in the same run as the default workload and reported under "also"
ALSO_WORKLOADS = ("csa_decode_128k_b32", "hca_decode_1m_b16", "csa_decode_1m_b8_mxfp4")


def fp8_gemm_peak(dev, n: int = 8192, seconds: float = 4.0):
    """Dense e4m3 GEMM rate of this GPU (torch._scaled_mm, n x n x n, fp32 scales, bf16
    out): best of 10 single launches (burst) and the mean over `seconds` of back-to-back
    launches (sustained), in TFLOP/s."""
    a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
    b = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)  # noqa: E731
    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1) / 1e3)
    reps = 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_end = time.time() + seconds
    e0.record()
    while time.time() < t_end:
        for _ in range(20):
            mm()
        reps += 20
        torch.cuda.synchronize()
    e1.record()
    torch.cuda.synchronize()
    sustained = flop * reps / (e0.elapsed_time(e1) / 1e3) / 1e12
    return {"burst": round(flop / best / 1e12, 1), "sustained": round(sustained, 1),
            "how": f"torch._scaled_mm e4m3 {n}^3, bf16 out: best of 10 (burst), "
                   f"{seconds:.0f} s back to back (sustained)"}


def measure(name: str, args, dist, dev, rank: int, world: int, full: bool):
    """Times K steps of workload `name` (graph replay, L2 flushed before each), then the
    per-kernel device times in a second replayed graph; with `full`, also the end-to-end
    rate through host buffers.  Returns the fields of the JSON line."""
    import long_context_compressed_04_b200 as L
    from long_context_compressed_04_b200 import pipeline

    raw_tail = getattr(args, "raw_tail", False) and WORKLOADS[name]["kind"] != "csa_prefill"
    wl = make_workload(name, rank, dev, keep_raw=256 if raw_tail else None)
    buf = pipeline.alloc(wl, dev)
    if raw_tail:
        # the raw store keeps each sequence's last 256 tokens (the window and the newest
        # block); the compressed cache before the step is drawn as stored-format rows
        from long_context_compressed_04_b200 import synth
        g = torch.Generator(device=dev).manual_seed(1000 + rank)
        buf.entries.copy_(synth.random_entries(buf.entries.shape[0], wl.fmt, wl.D, g, dev))
    else:
        all_seq, all_ent = pipeline.all_entry_items(wl, dev)
        pipeline.compress(wl, buf, all_seq, all_ent)      # build the compressed cache
        del all_seq, all_ent
    new_seq, new_ent = step_items(wl, name, dev)
    torch.cuda.synchronize()

    def step_eager(b=buf, w=wl):
        pipeline.step(w, b, new_seq, new_ent)

    # the step's launches are captured once into a CUDA graph and replayed, so the timed
    # region measures device work rather than Python/ctypes launch overhead
    for _ in range(args.warmup):
        step_eager()
    torch.cuda.synchronize()
    graph = None
    kernels_per_step = 0
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        c0 = L.csa_launch_count()
        with torch.cuda.graph(graph):
            step_eager()
        kernels_per_step = L.csa_launch_count() - c0   # libcsa kernels in the graph
        torch.cuda.synchronize()

    def step():
        if graph is not None:
            graph.replay()
        else:
            step_eager()

    # L2 flush between timed steps: write 256 MB (> the 126 MB L2), then read another
    # 256 MB so that the dirty flush lines are written back here, outside the timed region,
    # and L2 holds neither workload data nor pending write-backs when a step starts
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    def barrier():
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    launches0 = L.csa_launch_count()
    with ClockSampler(gpu_index_for_smi(dev.index)) as clk:
        barrier()
        for i in range(K):
            flush_l2()
            ev[i][0].record()
            step()
            ev[i][1].record()
        barrier()
    launches = L.csa_launch_count() - launches0 + kernels_per_step * K
    ms_max = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dist, dev)
    assert int(buf.dev_status.item()) == 0, f"device status flagged during the {name} run"

    # second pass: the same step captured into a CUDA graph with a CUDA event pair around
    # every libcsa kernel (recorded on the launching stream); each replay re-records them,
    # so the device time of each kernel is read after every replay
    L.csa_profile_collect()
    L.csa_profile_enable(True)
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph):
        step_eager()
    L.csa_profile_enable(False)
    torch.cuda.synchronize()
    per_kernel = {}
    for i in range(K):
        flush_l2()
        pgraph.replay()
        torch.cuda.synchronize()
        for kname, (n_l, tot_ms) in L.csa_profile_collect(keep_pending=True).items():
            c, t_ = per_kernel.get(kname, (0, 0.0))
            per_kernel[kname] = (c + n_l, t_ + tot_ms)
    del pgraph
    L.csa_profile_collect()

    e2e = None
    if full:
        e2e = measure_e2e(name, wl, buf, new_seq, new_ent, args, dist, dev, world, flush_l2,
                          barrier)

    peak, peak_kind = _peaks()
    total_bytes, key_bytes = algorithmic_bytes(wl)
    value = whole_job_rate(wl.Q, world, K, ms_max)
    step_s = ms_max / K / 1e3
    # the dominant kernel is the one that moves the method's dominant bytes: the indexer
    # (every visible key, each step) for CSA decode, the attention (every entry) for HCA
    alg_of = {"indexer_score_tc": key_bytes,
              "indexer_score_fp4": key_bytes,
              "attn_tc": total_bytes - key_bytes, "attn_simt": total_bytes - key_bytes}
    dom_name = next((n for n in (["indexer_score_tc", "indexer_score_fp4"]
                                 if wl.H_I else [])
                     + ["attn_tc", "attn_simt"] if n in per_kernel), None)
    roof = None
    if WORKLOADS[name]["kind"] == "csa_prefill" and "indexer_score_tc" in per_kernel:
        # prefill: the indexer's FP8 dot products bound it (tensor pipe); the peak is this
        # GPU's e4m3 GEMM rate, measured here (sustained: the indexer runs for milliseconds)
        n_l, tot_ms = per_kernel["indexer_score_tc"]
        avg_s = tot_ms / n_l / 1e3
        fl = indexer_flops(wl)
        fp8 = fp8_gemm_peak(dev)
        ach = fl / avg_s / 1e12
        roof = {"bound": "tensor", "kernel": "indexer_score_tc", "achieved": round(ach, 1),
                "peak": fp8["sustained"], "unit": "TFLOP/s",
                "frac": round(ach / fp8["sustained"], 4), "traffic": None,
                "peak_source": "measured in this run (sustained); " + fp8["how"],
                "fp8_gemm_burst": fp8["burst"], "algorithmic_flops_per_launch": fl,
                "avg_launch_us": round(avg_s * 1e6, 2)}
    elif dom_name:
        n_l, tot_ms = per_kernel[dom_name]
        avg_s = tot_ms / n_l / 1e3
        alg = alg_of[dom_name]
        ach = alg / avg_s / 1e9
        roof = {"bound": "hbm", "kernel": dom_name, "achieved": round(ach, 1), "peak": peak,
                "unit": "GB/s", "frac": round(ach / peak, 4),
                "traffic": measured_traffic(name, dom_name),
                "peak_source": f"{peak_kind} hbm_gbs (copy)",
                "algorithmic_bytes_per_launch": alg, "avg_launch_us": round(avg_s * 1e6, 2)}
    out = {
        "value": value, "ms_per_step": ms_max / K,
        "config": {"workload": name, **WORKLOADS[name], "queries_per_gpu": wl.Q,
                   **({"cache": "stored rows drawn directly; raw store keeps the last 256 tokens"}
                      if raw_tail else {}),
                   "l2": "flushed before every timed step (256 MB write, then 256 MB read)",
                   "indexer_inputs": ("mxfp4 (e2m1, one UE8M0 scale per 32) from N(0,1)"
                                      + ("; top-k on BF16-rounded scores" if wl.select_bf16
                                         else "")) if wl.kI4 is not None
                   else "fp8 e4m3 N(0,1), 1x128 scales"},
        "roofline": roof,
        "step_roofline": {"algorithmic_bytes": total_bytes,
                          "achieved_gbs": round(total_bytes / step_s / 1e9, 1),
                          "frac": round(total_bytes / step_s / 1e9 / peak, 4)},
        "kernels": {k2: {"launches": v[0], "avg_us": round(v[1] / v[0] * 1e3, 2),
                         "share": round(v[1] / sum(x[1] for x in per_kernel.values()), 4)}
                    for k2, v in per_kernel.items()},
        "gpu_launches": launches,
        "launch": "cuda graph replay" if graph is not None else "eager",
        "clocks": clk.summary(),
    }
    if e2e is not None:
        out["e2e"] = e2e
    del graph, buf, wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def measure_e2e(name, wl, buf, new_seq, new_ent, args, dist, dev, world, flush_l2, barrier):
    """The same metric through the public API with host buffers.  Every step copies its
    inputs from pinned host memory (the query heads, the indexer's query heads, scales and
    weights, and the new tokens' raw KV and gate rows) and copies its output back.  The
    copies are double-buffered on a second stream: step i+1's inputs go up and step i-1's
    output comes down while step i computes.  A run of E steps is captured into one CUDA
    graph (the two streams forked and joined inside it) and replayed; the rate is E steps
    over the replay's device time."""
    from long_context_compressed_04_b200 import pipeline
    import dataclasses

    nn = new_tokens(wl, name)
    last_rows = torch.cat([(wl.kv_off[b] + (wl.T.to(dev)[b] - nn - wl.kv_pos0[b]))
                           + torch.arange(nn, device=dev) for b in range(wl.B)]).long()
    nr = last_rows.numel()
    fields = [f for f in ("q", "qI", "qs", "qI4", "qsf4", "w") if getattr(wl, f) is not None]
    pinned = {f: torch.empty(getattr(wl, f).shape, dtype=getattr(wl, f).dtype,
                             pin_memory=True).copy_(getattr(wl, f).cpu()) for f in fields}
    pin_kv = torch.empty((nr, wl.D), dtype=wl.kv.dtype, pin_memory=True).copy_(wl.kv[last_rows].cpu())
    pin_gate = torch.empty((nr, wl.D), dtype=wl.gate.dtype, pin_memory=True).copy_(wl.gate[last_rows].cpu())
    # two sets of device inputs and outputs; the compressed cache and raw KV are shared
    sets = []
    for j in range(2):
        dev_in = {f: torch.empty_like(getattr(wl, f)) for f in fields}
        w_j = dataclasses.replace(wl, **dev_in)
        b_j = dataclasses.replace(buf, out=torch.empty_like(buf.out),
                                  idx=None if buf.idx is None else torch.empty_like(buf.idx),
                                  workspace=torch.empty_like(buf.workspace))
        sets.append(dict(wl=w_j, buf=b_j, kv=torch.empty((nr, wl.D), dtype=wl.kv.dtype, device=dev),
                         gate=torch.empty((nr, wl.D), dtype=wl.gate.dtype, device=dev),
                         up=torch.cuda.Event(), done=torch.cuda.Event(),
                         down=torch.cuda.Event(),
                         host_out=torch.empty(buf.out.shape, dtype=buf.out.dtype,
                                              pin_memory=True)))
    h2d = sum(v.numel() * v.element_size() for v in pinned.values()) + 2 * pin_kv.numel() * 2
    d2h = sets[0]["host_out"].numel() * sets[0]["host_out"].element_size()
    copy = torch.cuda.Stream()

    def upload(st):
        for f in fields:
            getattr(st["wl"], f).copy_(pinned[f], non_blocking=True)
        st["kv"].copy_(pin_kv, non_blocking=True)
        st["gate"].copy_(pin_gate, non_blocking=True)
        st["up"].record(copy)

    def run(E):
        comp = torch.cuda.current_stream()   # the capture stream while a graph is captured
        # fork: the copy stream joins the capture
        copy.wait_stream(comp)
        with torch.cuda.stream(copy):
            upload(sets[0])
        for i in range(E):
            st, nxt = sets[i % 2], sets[(i + 1) % 2]
            if i + 1 < E:
                with torch.cuda.stream(copy):
                    if i >= 1:
                        copy.wait_event(nxt["down"])    # step i-1's output is read back
                    upload(nxt)
            comp.wait_event(st["up"])
            wl.kv.index_copy_(0, last_rows, st["kv"])
            wl.gate.index_copy_(0, last_rows, st["gate"])
            pipeline.step(st["wl"], st["buf"], new_seq, new_ent)
            st["done"].record(comp)
            with torch.cuda.stream(copy):
                copy.wait_event(st["done"])
                st["host_out"].copy_(st["buf"].out, non_blocking=True)
                st["down"].record(copy)
        comp.wait_stream(copy)                          # join

    E = 16
    run(E)
    torch.cuda.synchronize()
    egraph = None
    if not args.no_graph:
        egraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(egraph):
            run(E)
        torch.cuda.synchronize()
    R = max(args.steps // E, 4)
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(R)]
    barrier()
    for i in range(R):
        flush_l2()
        ee[i][0].record()
        if egraph is not None:
            egraph.replay()
        else:
            run(E)
        ee[i][1].record()
    barrier()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ee), dist, dev)
    for st in sets:
        assert int(st["buf"].dev_status.item()) == 0
    return {"value": whole_job_rate(wl.Q, world, R * E, e2e_ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": e2e_ms / (R * E),
            "how": f"pinned h2d of each step's inputs and d2h of its output on a second stream, "
                   f"double-buffered; {E} pipelined steps per captured graph, {R} replays"}


def measure_cp(world: int, args, dev):
    """Context-parallel decode of the headline workload, its W ranks' slices on this one GPU
    (long_context_compressed_04_b200.cp).  On W GPUs the slices' selections run at once, so
    each part is timed on its own, from a CUDA graph, with L2 flushed before it: every
    rank's selection (the slowest is the step's share), the merge, every rank's row pack and
    the attention over the gathered rows.  The two exchanges run here as stand-ins (a copy
    and a sum) outside the timed parts; their bytes per rank are reported, with the time
    they take at the measured peer bandwidth (770 GB/s per direction), launch latency not
    included.  The cache is drawn as stored rows (the raw store keeps the last 256 tokens)."""
    from long_context_compressed_04_b200 import cp, pipeline, synth
    name = DEFAULT_WORKLOAD
    wl = make_workload(name, 0, dev, keep_raw=256)
    g = torch.Generator(device=dev).manual_seed(1000)
    rows = synth.random_entries(wl.ent_rows, wl.fmt, wl.D, g, dev)
    ent_off = wl.ent_off.cpu()
    ranks = []
    for r in range(world):
        kI, ks, ents, off, base = [], [], [], [], 0
        for b in range(wl.B):
            lo, hi = cp.slice_bounds(int(wl.n_ent[b]), world, r)
            r0 = int(ent_off[b])
            kI.append(wl.kI[r0 + lo:r0 + hi])
            ks.append(wl.ks[r0 + lo:r0 + hi])
            ents.append(rows[r0 + lo:r0 + hi])
            off.append(base)
            base += hi - lo
        sl = cp.make_slice(wl, world, r, torch.tensor(off, dtype=torch.int64))
        ranks.append((sl, torch.cat(kI).contiguous(), torch.cat(ks).contiguous(),
                      torch.cat(ents).contiguous(), cp.alloc(wl, sl, world, dev)))
    one = pipeline.alloc(wl, dev)
    one.entries.copy_(rows)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def graph(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        return gr

    reps = max(args.steps, 10)

    def timed(gr):
        ts = []
        for _ in range(reps):
            flush.zero_()          # still running when the graph is launched behind it
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gr.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(ts)

    sel_g = [graph(lambda sl=sl, kI=kI, ks=ks, buf=buf: cp.select_local(wl, sl, kI, ks, buf))
             for sl, kI, ks, _e, buf in ranks]
    sel_us = [timed(gr) for gr in sel_g]
    cands = torch.stack([buf.cand for *_x, buf in ranks])
    for *_x, buf in ranks:
        cp.exchange_candidates(buf, all_gather=lambda out, inp: out.copy_(cands))
    buf0 = ranks[0][4]
    merge_us = timed(graph(lambda: cp.merge(wl, buf0)))
    for *_x, buf in ranks[1:]:
        buf.idx.copy_(buf0.idx)
    pack_us = [timed(graph(lambda sl=sl, ents=ents, buf=buf: cp.pack(wl, sl, ents, buf)))
               for sl, _k, _s, ents, buf in ranks]
    total = torch.stack([buf.packed.view(torch.int32) for *_x, buf in ranks]).sum(
        0, dtype=torch.int32)
    cp.exchange_rows(buf0, all_reduce=lambda t: t.copy_(total))
    attn_us = timed(graph(lambda: cp.attend(wl, buf0)))
    one_sel_us = timed(graph(lambda: pipeline.indexer_topk(wl, one)))
    one_attn_us = timed(graph(lambda: pipeline.attend(wl, one)))
    torch.cuda.synchronize()
    ok = (all(int(buf.dev_status.item()) == 0 for *_x, buf in ranks)
          and int(one.dev_status.item()) == 0)
    same = bool(torch.equal(one.idx, buf0.idx)) and bool(
        torch.equal(one.out.view(torch.int16), buf0.out.view(torch.int16)))
    cand_b, rows_b = cp.exchange_bytes(wl, world)
    # all_gather: each rank receives (W - 1) buffers; ring all_reduce: 2 (W - 1) / W x size
    xfer = (world - 1) * cand_b + 2 * (world - 1) / world * rows_b
    xfer_us = xfer / 770e9 * 1e6
    step_us = max(sel_us) + merge_us + max(pack_us) + attn_us
    return {"mode": "context-parallel, the ranks' parts timed in turn on one GPU",
            "workload": name, "world": world,
            "slice_select_us": [round(x, 1) for x in sel_us], "merge_us": round(merge_us, 1),
            "pack_us": [round(x, 1) for x in pack_us], "attention_us": round(attn_us, 1),
            "rank_compute_us": round(step_us, 1),
            "exchange_bytes_in_per_rank": int(xfer), "exchange_us_at_770GBps": round(xfer_us, 1),
            "one_gpu_select_us": round(one_sel_us, 1), "one_gpu_attention_us": round(one_attn_us, 1),
            "bitwise_equal_one_gpu": same, "dev_status_clean": ok,
            "timing": f"median of {reps} graph replays, each behind a 256 MB L2 flush, "
                      "CUDA events"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", action="store_true",
                    help="measure only --workload (not the other decode workloads)")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    ap.add_argument("--raw-tail", action="store_true",
                    help="keep only each sequence's last 256 raw tokens and draw the compressed "
                         "cache as stored rows (the same step, a few GB on the device; for "
                         "profiling)")
    ap.add_argument("--cp", type=int, default=0,
                    help="time context-parallel decode of the headline workload over this many "
                         "slices, the ranks in turn on one GPU (a separate JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)
    if args.cp:
        torch.cuda.set_device(0)
        print(json.dumps(measure_cp(args.cp, args, torch.device("cuda", 0))), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    head = measure(args.workload, args, dist, dev, rank, world, full=True)
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
    }
    line.update({k: v for k, v in head.items() if k not in ("value", "ms_per_step")})
    if args.workload == DEFAULT_WORKLOAD and not args.no_also:
        # every rank measures the same workloads in the same order
        line["also"] = {}
        for name in ALSO_WORKLOADS:
            r = measure(name, args, dist, dev, rank, world, full=False)
            line["also"][name] = {
                "value": r["value"], "unit": UNIT, "ms_per_step": r["ms_per_step"],
                "step_frac": r["step_roofline"]["frac"],
                "dominant_kernel": None if r["roofline"] is None else r["roofline"]["kernel"],
                "dominant_frac": None if r["roofline"] is None else r["roofline"]["frac"],
                "kernels": r["kernels"], "gpu_launches": r["gpu_launches"],
                "clocks": r["clocks"]}
            line["gpu_launches"] += r["gpu_launches"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
