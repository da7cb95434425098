#!/usr/bin/env python3
"""Benchmark of the KDA layer core on B200.

One step = one prefill call of the 8K-token workload (prefill_bf16_T8192_H32:
1 sequence x 8192 tokens x 32 heads x d=128, bf16 q/k/v, fp32 log-decay and
beta, zero initial state, final state returned) through the library's C ABI.
The decode step of the 256-sequence x 34-layer workload (one layer per call,
rotating over the 34 state slabs) is timed the same way and reported in the
``decode`` object.  Inputs are synthetic and seeded (gated_delta_rule_152_b200.inputs).

Multi-GPU: one process per GPU (torchrun).  Sequences and heads are
independent, so every rank runs its own replica of the workload (weak
scaling) with no collective on the data path; the timed region is bracketed by
a barrier and the max over ranks is reported.

``--impl reference`` times the fp64 CPU oracle (the only reference that
exists for this method) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_152_b200 import inputs as kin  # noqa: E402

METRIC = "KDA prefill tokens/s and decode seq-steps/s per layer on 1 B200; % of roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
TF32_OVER_BF16 = 1.1 / 2.25          # nominal dense tf32 : bf16 tensor-core ratio
D = 128
# Algorithmic HBM bytes per token-head of the prefill, as the method's
# workload fixes them: q, k, v bf16 (3 x 256), g fp32 (512), beta (4), and o
# in v's dtype (256) = 1540 B.  Per (sequence, head) add the final state write
# (64 KiB) and, when given, the initial state read (64 KiB).  The roofline
# fraction is taken on these bytes.
PREFILL_BYTES_PER_TOKEN_HEAD = 3 * 2 * D + 4 * D + 4 + 2 * D
# This library writes o in fp32, 256 B more per token-head (bf16 rounding of
# the exact output alone would exceed the 2e-2 x RMS bound); those are the
# bytes the kernel actually moves, reported beside the fraction.
PREFILL_BYTES_PER_TOKEN_HEAD_AS_WRITTEN = PREFILL_BYTES_PER_TOKEN_HEAD + 2 * D
STATE_BYTES = 4 * D * D
# Dense contraction flops per token-head of the 64-token chunk form:
# 5 x (2 C^2 d) + 3 x (2 C d^2) + C^3 / 3 per chunk of C = 64 tokens.
PREFILL_FLOPS_PER_TOKEN_HEAD = (5 * 2 * 64 * 64 * D + 3 * 2 * 64 * D * D + 64 ** 3 // 3) // 64
# Decode: state read + write, plus q, k, v (bf16), g (fp32), beta and o in v's
# dtype = 132,612 B per (sequence, head); o is written in fp32 (+256 B).
DECODE_BYTES_PER_SEQ_HEAD = 2 * STATE_BYTES + 3 * 2 * D + 4 * D + 4 + 2 * D
DECODE_BYTES_PER_SEQ_HEAD_AS_WRITTEN = DECODE_BYTES_PER_SEQ_HEAD + 2 * D
# One prefill call of the 8K workload (one sequence, full workspace) launches
# two kernels: the chunk index and the overlapped prep/state kernel.  The
# prefill roofline is taken over the whole call (algorithmic bytes of the
# call / its CUDA-event time); the ncu launch list gives each kernel's share.
PREFILL_KERNELS = ("kda_chunk_index_kernel", "kda_chunk_overlap_kernel")
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the dominant kernel, from the ncu capture named here, and a hash of the
# kernel sources it was taken on: when the sources differ, the figure no
# longer describes the kernel and the line reports traffic as null.
MEASURED_TRAFFIC = {
    # 336,875,008 B read + 121,080,576 B written (one-pass capture)
    "prefill": {"bytes": 457955584,
                "capture": "profiles/kda_chunk_overlap_kernel__prefill_bf16_T8192_H32.md",
                "sources_sha": "04e0894bf777ae0d",
                "files": ("kda_chunk2.cu", "kda_tile.cuh", "sm100.cuh", "kda_common.cuh", "kda_launch.h")},
    # 547,409,408 B read + 483,761,920 B written
    "decode": {"bytes": 1031171328,
               "capture": "profiles/kda_decode_kernel__decode_bf16_256seq_H32_one_layer.md",
               "sources_sha": "db3decae6f041942",
               "files": ("kda_decode.cu", "kda_common.cuh", "kda_launch.h")},
}


def sources_sha(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "gated_delta_rule_152_b200", "csrc", f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kind):
    t = MEASURED_TRAFFIC[kind]
    if t["bytes"] is None or t["sources_sha"] != sources_sha(t["files"]):
        return None, None
    return t["bytes"], t["capture"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.out = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", 0)
            devn = getattr(props, "pci_device_id", 0)
            self.target = f"{dom:08x}:{bus:02x}:{devn:02x}.0" if bus is not None else str(device_index)
        except Exception:
            self.target = str(device_index)

    def start(self):
        try:
            self.out = open(os.devnull, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.target, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            text = ""
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in text.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sms.append(float(parts[0]))
                maxs.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs), "reasons": sorted(reasons),
                "samples": len(sms)}


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU baseline
def oracle_prefill_sample(x: kin.PrefillInputs, tokens: int, threads: int = 0):
    """Run the fp64 oracle on the first `tokens` tokens of the workload (all
    heads); returns (seconds, tokens)."""
    import oracle
    sl = slice(0, tokens)
    t0 = time.perf_counter()
    oracle.kda_forward(x.q[sl], x.k[sl], x.v[sl], x.g[sl], x.beta[sl], [0, tokens], None, threads=threads)
    return time.perf_counter() - t0, tokens


def _oracle_rate(fn, units, min_s):
    """Run fn() (one bounded sample of `units` units) until min_s seconds have
    passed; returns (units per second, seconds, repetitions)."""
    reps, total = 0, 0.0
    while reps == 0 or (total < min_s and reps < 64):
        t0 = time.perf_counter()
        fn()
        total += time.perf_counter() - t0
        reps += 1
    return units * reps / total, total, reps


def cpu_baseline(x: kin.PrefillInputs, min_s: float = 3.0):
    """The fp64 oracle on the host cores: the headline figure is the 8K
    workload on all cores; ``by_config`` adds one thread and all threads on
    bounded samples of the tiny, 8K, varlen and decode workloads (each
    sample's extent stated), about 10-20 s of CPU work in all."""
    import oracle
    cores = oracle.max_threads()
    rows = []
    f64 = oracle.to_f64   # inputs converted once, outside the timed calls

    def prefill_row(name, xs, tokens, threads, what):
        sl = slice(0, tokens)
        q, k, v, g, b = (f64(t)[sl] for t in (xs.q, xs.k, xs.v, xs.g, xs.beta))
        cu = [0, tokens] if xs.cu_seqlens.numel() == 2 else xs.cu_seqlens.tolist()
        s0 = None if xs.initial_state is None else f64(xs.initial_state)
        fn = lambda: oracle.kda_forward(q, k, v, g, b, cu, s0, threads=threads)
        rate, secs, reps = _oracle_rate(fn, tokens, min_s)
        rows.append({"workload": name, "threads": threads, "value": rate, "unit": "tokens/s",
                     "sample": f"{what}; {reps} pass(es), {secs:.1f} s"})
        return rate, secs, reps

    # 8K workload: all threads over whole passes (the headline), one thread on its first 256 tokens
    rate8k, secs8k, reps8k = prefill_row(kin.PREFILL_8K.name, x, x.total_T, cores,
                                         f"all {x.total_T} tokens x {x.heads} heads")
    prefill_row(kin.PREFILL_8K.name, x, 256, 1, f"first 256 of {x.total_T} tokens x {x.heads} heads")
    # tiny fp32 workload: whole (two heads, so at most two threads have work)
    xt = kin.make_prefill(kin.TINY_FP32)
    for th in (1, cores):
        prefill_row(kin.TINY_FP32.name, xt, xt.total_T, th, f"all {xt.total_T} tokens x {xt.heads} heads")
    # varlen workload: its first two sequence lengths (all heads, initial states) on all
    # threads; the first 512 tokens of its first sequence on one thread
    lens = kin.seq_lengths(kin.VARLEN_16)
    xv = kin.make_prefill(kin.VARLEN_16, lengths=lens[:2])
    prefill_row(kin.VARLEN_16.name, xv, xv.total_T, cores,
                f"sequences of lengths {lens[0]} and {lens[1]} (the first two of 16) x {xv.heads} heads")
    xv1 = kin.make_prefill(kin.VARLEN_16, lengths=[512])
    prefill_row(kin.VARLEN_16.name, xv1, 512, 1, f"512 tokens of one sequence x {xv1.heads} heads")
    # decode workload: 8 sequences x 4 of its layer slabs x 32 heads
    spec = kin.DECODE_256x34
    toks = [[f64(t) for t in (tk.q, tk.k, tk.v, tk.g, tk.beta)]
            for tk in (kin.make_decode_tokens(spec, layer, n_seqs=8) for layer in range(4))]
    states = [f64(kin.make_decode_state(spec, layer, n_seqs=8)) for layer in range(4)]
    for th in (1, cores):
        def dec():
            for t, st in zip(toks, states):
                oracle.kda_decode(*t, st, threads=th)
        rate, secs, reps = _oracle_rate(dec, 8 * 4, min_s / 3)
        rows.append({"workload": spec.name, "threads": th, "value": rate, "unit": "seq-steps/s/layer",
                     "sample": f"8 sequences x 4 layer slabs x {spec.heads} heads; {reps} pass(es), {secs:.1f} s"})
    # indexer selection: 4 of the top-k workload's 64 query rows (numpy's sort, one thread)
    from oracle.topk import topk_indices
    sc = torch.randn(4, TOPK_N, generator=torch.Generator().manual_seed(2048)).numpy()
    rate, secs, reps = _oracle_rate(lambda: topk_indices(sc, TOPK_K), 4, min_s / 3)
    rows.append({"workload": TOPK_WORKLOAD, "threads": 1, "value": rate, "unit": "query rows/s",
                 "sample": f"4 of {TOPK_ROWS} rows x {TOPK_N} scores; {reps} pass(es), {secs:.1f} s"})
    return {"value": rate8k, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps8k} passes over all {x.total_T} tokens x {x.heads} heads of {kin.PREFILL_8K.name}, "
                      f"fp64, {cores} OpenMP threads over (sequence, head) pairs, {secs8k:.1f} s",
            "by_config": rows}


# ---------------------------------------------------------------- GPU arm
def time_prefill_config(spec, dev, stream, steps, warmup, hbm, world):
    """Device time of one prefill call on another synthetic prefill config
    (inputs resident in HBM, larger than L2), with its own clock record."""
    from gated_delta_rule_152_b200 import kda
    x = kin.make_prefill(spec)
    xd = x.to(dev)
    T, H = x.total_T, x.heads
    N = x.cu_seqlens.numel() - 1
    o = torch.empty(T, H, D, device=dev)
    sT = torch.empty(N, H, D, D, device=dev)
    ws = torch.empty(max(kda.kda_chunk_fwd_workspace_size(N, T, H), 256), dtype=torch.uint8, device=dev)

    def step():
        kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, initial_state=xd.initial_state,
                          final_state=sT, o=o, workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    state_io = N * H * STATE_BYTES * (2 if x.initial_state is not None else 1)
    nbytes = T * H * PREFILL_BYTES_PER_TOKEN_HEAD + state_io
    nbytes_written = T * H * PREFILL_BYTES_PER_TOKEN_HEAD_AS_WRITTEN + state_io
    gbs = nbytes / (ms / 1e3) / 1e9
    overlapped = H <= 96   # the overlapped launch serves any number of sequences up to 96 heads
    del xd, o, sT, ws
    torch.cuda.empty_cache()
    return {"workload": spec.name, "value": world * T / (ms / 1e3), "unit": "tokens/s", "ms_per_call": ms,
            "sequences": N, "tokens": T, "heads": H, "steps": steps, "warmup": warmup,
            "path": "overlapped" if overlapped else "two-launch (index, prep, state kernels)",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "bytes_per_launch": nbytes, "bytes_per_launch_as_written": nbytes_written,
                         "frac_as_written": nbytes_written / (ms / 1e3) / 1e9 / hbm},
            "clocks": clk}, steps * (2 if overlapped else 3)


# The lightning indexer's selection step on one decode step's worth of
# queries: 64 query rows, each over the scores of 1,048,576 past tokens, the
# 2,048 highest kept (page "GLM-5.3-FLASH", section "How can a layer search
# the whole history selectively?").  Scores ~ N(0, 1), seeded.
TOPK_ROWS, TOPK_N, TOPK_K = 64, 1 << 20, 2048
TOPK_WORKLOAD = f"indexer_topk{TOPK_K}_rows{TOPK_ROWS}_n{TOPK_N}"
TOPK_KERNELS = 5   # init, hist0, pick0, split, finish (plus one memset of the error word)


def time_topk(dev, stream, steps, warmup, hbm, world):
    """Device time of one top-k selection call (scores resident in HBM,
    256 MB > L2); the roofline bytes are the scores read once and the indices
    written once."""
    from gated_delta_rule_152_b200 import kda
    g = torch.Generator().manual_seed(2048)
    scores = torch.randn(TOPK_ROWS, TOPK_N, generator=g).to(dev)
    idx = torch.empty(TOPK_ROWS, TOPK_K, dtype=torch.int32, device=dev)
    ws = torch.empty(kda.kda_topk_workspace_size(TOPK_ROWS, TOPK_N, TOPK_K), dtype=torch.uint8, device=dev)
    call = lambda: kda.kda_topk_indices(scores, TOPK_K, indices=idx, workspace=ws, stream=stream)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    nbytes = TOPK_ROWS * TOPK_N * 4 + TOPK_ROWS * TOPK_K * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    del scores, idx, ws
    torch.cuda.empty_cache()
    return {"workload": TOPK_WORKLOAD, "value": world * TOPK_ROWS / (ms / 1e3), "unit": "query rows/s",
            "ms_per_call": ms, "steps": steps, "warmup": warmup,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "bytes_per_launch": nbytes,
                         "note": "scores read once + indices written once; the kernels read the scores "
                                 "twice when the cut's bin holds <= 16,384 tokens of a row"}}, steps * TOPK_KERNELS


def bench_gpu(args, world, rank, local):
    from gated_delta_rule_152_b200 import kda
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)

    # ---------------- prefill (8K-token workload) --------------------------
    x = kin.make_prefill(kin.PREFILL_8K)
    xd = x.to(dev)
    T, H = x.total_T, x.heads
    o = torch.empty(T, H, D, device=dev)
    sT = torch.empty(1, H, D, D, device=dev)
    ws = torch.empty(max(kda.kda_chunk_fwd_workspace_size(1, T, H), 256), dtype=torch.uint8, device=dev)

    def step():
        kda.kda_chunk_fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.cu_seqlens, initial_state=None,
                          final_state=sT, o=o, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    # SM clocks are sampled from here to the end of the last timed region
    clocks = ClockSampler(dev.index)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    prefill_tok_s = world * T / (ms / 1e3)
    bytes_per_launch = T * H * PREFILL_BYTES_PER_TOKEN_HEAD + H * STATE_BYTES
    bytes_written = T * H * PREFILL_BYTES_PER_TOKEN_HEAD_AS_WRITTEN + H * STATE_BYTES
    achieved_gbs = bytes_per_launch / (ms / 1e3) / 1e9
    flops_per_launch = T * H * PREFILL_FLOPS_PER_TOKEN_HEAD
    tf32_peak = bf16 * TF32_OVER_BF16
    achieved_tflops = flops_per_launch / (ms / 1e3) / 1e12

    # end to end: pinned host inputs -> device, call, o + final state -> host,
    # every step.  Inputs, outputs and their host copies are double-buffered:
    # step i+1's inputs come in on one copy stream while step i computes, and
    # step i's results leave on another (PCIe is full duplex); an event orders
    # every reuse of a buffer after its last reader.
    pin = lambda t: t.pin_memory()
    hins = [pin(t) for t in (x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens)]
    ho = [torch.empty(T, H, D).pin_memory() for _ in range(2)]
    hs = [torch.empty(1, H, D, D).pin_memory() for _ in range(2)]
    do = [o, torch.empty(T, H, D, device=dev)]
    ds = [sT, torch.empty(1, H, D, D, device=dev)]
    dins = [[torch.empty_like(t, device=dev) for t in hins] for _ in range(2)]
    in_stream, out_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    out_done = [torch.cuda.Event(), torch.cuda.Event()]
    for ev in comp_done:
        ev.record(stream)
    for ev in out_done:
        ev.record(out_stream)

    def e2e_step(i):
        b = i & 1
        in_stream.wait_event(comp_done[b])   # step i-2's call has read input set b
        with torch.cuda.stream(in_stream):
            for d_, h_ in zip(dins[b], hins):
                d_.copy_(h_, non_blocking=True)
        in_done[b].record(in_stream)
        stream.wait_event(in_done[b])
        stream.wait_event(out_done[b])       # step i-2's results have left output set b
        dq, dk, dv, dg, db, dcu = dins[b]
        kda.kda_chunk_fwd(dq, dk, dv, dg, db, dcu, final_state=ds[b], o=do[b], workspace=ws, stream=stream)
        comp_done[b].record(stream)
        out_stream.wait_event(comp_done[b])
        with torch.cuda.stream(out_stream):
            ho[b].copy_(do[b], non_blocking=True)
            hs[b].copy_(ds[b], non_blocking=True)
        out_done[b].record(out_stream)

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    in_stream.wait_event(e0)   # the first timed copies start inside the timed region
    for i in range(args.steps):
        e2e_step(i)
    for ev in out_done:   # the last results are on the host
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    h2d = sum(t.numel() * t.element_size() for t in hins)
    d2h = ho[0].numel() * 4 + hs[0].numel() * 4
    del xd, dins, do, ds
    torch.cuda.empty_cache()

    # ---------------- decode (256 seq x 34 layers) -------------------------
    spec = kin.DECODE_256x34
    L = spec.layers if not args.quick else 4
    N = spec.n_seqs
    states = torch.empty(L, N, spec.heads, D, D, device=dev)

    def fill(layer):   # each layer slab has its own seed; drawn on the host in parallel
        states[layer].copy_(kin.make_decode_state(spec, layer))
        return layer

    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=max(1, min(8, (os.cpu_count() or 1) // world))) as pool:
        list(pool.map(fill, range(L)))
    torch.cuda.synchronize(dev)
    toks = [kin.make_decode_tokens(spec, layer).to(dev) for layer in range(L)]
    od = torch.empty(N, spec.heads, D, device=dev)

    def dstep(i):
        t = toks[i % L]
        kda.kda_decode_step(t.q, t.k, t.v, t.g, t.beta, states[i % L], o=od, stream=stream)

    dsteps = max(args.steps, L)
    for i in range(max(args.warmup, 3)):
        dstep(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for i in range(dsteps):
        dstep(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    dms = max_over_ranks(e0.elapsed_time(e1) / dsteps, world)
    dec_rate = world * N / (dms / 1e3)
    dec_bytes = N * spec.heads * DECODE_BYTES_PER_SEQ_HEAD
    dec_bytes_written = N * spec.heads * DECODE_BYTES_PER_SEQ_HEAD_AS_WRITTEN
    dec_gbs = dec_bytes / (dms / 1e3) / 1e9
    del states
    torch.cuda.empty_cache()

    # ---------------- the indexer's top-k selection -------------------------
    topk, topk_launches = time_topk(dev, stream, max(args.steps, 20), max(args.warmup, 3), hbm, world)

    # ---------------- the other prefill configs (one GPU, not in --quick) ---
    # their host inputs take about 10 GB each, too much to hold once per rank
    extras, extra_launches = {}, 0
    if not args.quick and world == 1:
        for key, xspec in (("long_context", kin.PREFILL_128K), ("varlen", kin.VARLEN_16)):
            extras[key], n_l = time_prefill_config(xspec, dev, stream, 30, max(args.warmup, 3), hbm, world)
            extra_launches += n_l

    traffic_prefill, traffic_prefill_src = measured_traffic("prefill")
    traffic_decode, traffic_decode_src = measured_traffic("decode")
    line = {
        "metric": METRIC,
        "value": prefill_tok_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "tf32",
        "data": "synthetic (seeded; no dataset or weights involved)",
        "config": {"workload": kin.PREFILL_8K.name, "sequences": 1, "tokens": T, "heads": H, "d": D,
                   "qkv_dtype": "bf16", "o_dtype": "fp32", "parallelism": f"replicas x{world}",
                   "l2": "inputs 471 MB > 126 MB L2, no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                     "frac": achieved_gbs / hbm, "traffic": traffic_prefill,
                     "traffic_capture": traffic_prefill_src,
                     "peak_source": f"{peak_src} hbm_gbs",
                     "scope": "whole prefill call: " + " + ".join(PREFILL_KERNELS),
                     "bytes_per_launch": bytes_per_launch,
                     "bytes_per_launch_as_written": bytes_written,
                     "frac_as_written": bytes_written / (ms / 1e3) / 1e9 / hbm,
                     "as_written_note": "o is written in fp32, 256 B per token-head more than the "
                                        "1540 B the fraction is taken on",
                     "tensor": {"achieved_tflops": achieved_tflops, "peak_tflops_tf32": tf32_peak,
                                "frac": achieved_tflops / tf32_peak,
                                "flops_per_launch": flops_per_launch}},
        "decode": {"workload": spec.name, "value": dec_rate, "unit": "seq-steps/s/layer",
                   "ms_per_call": dms, "layers_rotated": L,
                   "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm, "unit": "GB/s",
                                "frac": dec_gbs / hbm, "traffic": traffic_decode,
                                "traffic_capture": traffic_decode_src,
                                "bytes_per_launch": dec_bytes, "bytes_per_launch_as_written": dec_bytes_written,
                                "frac_as_written": dec_bytes_written / (dms / 1e3) / 1e9 / hbm}},
        "e2e": {"value": world * T / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "topk": topk,
        "gpu_launches": args.steps * 2 * len(PREFILL_KERNELS) + dsteps + topk_launches + extra_launches,
        "clocks": clk,
    }
    line.update(extras)
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x)
    return line


def bench_reference(args, world, rank):
    """The reference arm: the fp64 oracle on the host cores, same metric."""
    if rank != 0:
        return None
    import oracle
    x = kin.make_prefill(kin.PREFILL_8K)
    tokens = args.ref_tokens
    for _ in range(args.warmup):
        oracle_prefill_sample(x, 64)
    t_total = 0.0
    for _ in range(args.steps):
        dt, _ = oracle_prefill_sample(x, tokens)
        t_total += dt
    rate = tokens * args.steps / t_total
    cores = oracle.max_threads()
    sample = (f"first {tokens} of 8192 tokens x 32 heads of prefill_bf16_T8192_H32 per step, fp64, "
              f"{cores} OpenMP threads")
    return {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": kin.PREFILL_8K.name, "sequences": 1, "tokens": 8192, "heads": 32, "d": D},
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-tokens", type=int, default=1024)
    ap.add_argument("--quick", action="store_true", help="decode over 4 layer slabs instead of 34")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = bench_reference(args, world, rank)
        else:
            line = bench_gpu(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
