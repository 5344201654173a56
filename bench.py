"""Benchmark of the MapFlow hot path on B200.

One step = one pass of the whole path over one sender layer and one receiver
layer of the workload: block statistics (lse + block masses), selection and
extraction of the kept blocks, and the fused map-mix x V.  Inputs are seeded
and synthetic (shapes of the 32K-token workload by default) and already
resident in HBM when the timed region starts; the kept map (tens of GB) is far
larger than L2, so no separate L2 flush is done.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--mode path|rounds|overlap]

With N > 1 (torchrun), the layer's query blocks are split across the ranks
with no data-path collective (every query block's work is independent): a
single sequence in zig-zag pairs (qb, nqb-1-qb), a varlen batch by whole
sequences balanced by causal cost.  The total work is fixed as N grows
(strong scaling); time = max over ranks.
`--impl reference` times the CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).

Two more measurements, one GPU each, print their own line:
`--mode rounds` the round-level selection (multi-turn workload: selection at
the watershed layer, then extraction and the fused kernel on every later
layer); `--mode overlap` a receiver prefill that fetches a mapped layer's
cache from pinned host memory while it recomputes its first layers, against
the same calls issued serially.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from cross_model_attention_block_b200 import partition  # noqa: E402
from cross_model_attention_block_b200 import synth  # noqa: E402

METRIC = ("mapped-AV GB/s & % HBM roofline; compress tokens/s & % tensor peak; "
          "layer-prefill ms")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ traffic

KERNEL_SOURCES = {
    "mapped_av": "cross_model_attention_block_b200/csrc/tc_mapped_av.cu",
    "block_stats": "cross_model_attention_block_b200/csrc/tc_qk.cu",
    "select_extract": "cross_model_attention_block_b200/csrc/tc_qk.cu",
}


def kernel_traffic(kernel, workload):
    """DRAM bytes per launch (read + write) of a kernel from profiles/traffic.json,
    or None when no capture exists for it or its source changed since."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel, {}).get(workload)
    if not rec:
        return None
    with open(os.path.join(ROOT, KERNEL_SOURCES[kernel]), "rb") as f:
        sha = hashlib.sha1(f.read()).hexdigest()
    return rec["bytes_per_launch"] if rec.get("source_sha1") == sha else None


# ------------------------------------------------------------ reference arm

def bench_reference(args, wl):
    """Time the CPU oracle on bounded samples of the workload (rank 0)."""
    from oracle import mapflow_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = len(os.sched_getaffinity(0))
    x = synth.single_layer(wl)
    L = wl.lengths[0]
    B = wl.B
    nqb = (L + B - 1) // B
    per_step = 2
    picks = [int((k + 0.5) * nqb / (per_step * (args.steps + args.warmup)))
             for k in range(per_step * (args.steps + args.warmup))]
    W = orc._f64(x.W)

    def one(qb):
        i1 = min(L, (qb + 1) * B)
        Qs, Ks, Vs = orc._f64(x.Q[:i1]), orc._f64(x.K[:i1]), orc._f64(x.V[:i1])
        r = orc.run_sequence(Qs, Ks, Vs, W, wl.Hkv, B, wl.tau, wl.band_bias, wl.band_width,
                             qbs=[qb])
        return r[qb]["O"].shape[0]

    it = iter(picks)
    for _ in range(args.warmup):
        for _ in range(per_step):
            one(next(it))
    t0 = time.perf_counter()
    rows = 0
    for _ in range(args.steps):
        for _ in range(per_step):
            rows += one(next(it))
    dt = time.perf_counter() - t0
    value = rows / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": L, "Hs": wl.Hs, "Hr": wl.Hr,
                   "Hkv": wl.Hkv, "d": wl.d, "B": wl.B, "tau": wl.tau},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} query blocks per step spread evenly over "
                                   f"the {nqb} query blocks (causal cost averages out); "
                                   f"full path per block"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(wl, x, budget_s=20.0):
    """The oracle on evenly spread query blocks until about budget_s of CPU work."""
    from oracle import mapflow_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = len(os.sched_getaffinity(0))
    L, B = wl.lengths[0], wl.B
    nqb = (L + B - 1) // B
    order = [int((k + 0.5) * nqb / 8) for k in range(8)]
    W = orc._f64(x.W)
    rows, done = 0, []
    t0 = time.perf_counter()
    for qb in order:
        i1 = min(L, (qb + 1) * B)
        r = orc.run_sequence(orc._f64(x.Q[:i1]), orc._f64(x.K[:i1]), orc._f64(x.V[:i1]), W,
                             wl.Hkv, B, wl.tau, wl.band_bias, wl.band_width, qbs=[qb])
        rows += r[qb]["O"].shape[0]
        done.append(qb)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"query blocks {done} of {nqb} (rows {rows} of {L}), whole path "
                      f"per block, {dt:.1f} s"}


# ----------------------------------------------------------------- our arm

def rank_plan(wl, rank, world):
    """Global query-block ranges [(begin, end), ...] this rank runs: the whole
    context at N = 1; zig-zag pairs of one sequence, or whole sequences of a
    varlen batch balanced by causal cost, at N > 1."""
    nq = [(L + wl.B - 1) // wl.B for L in wl.lengths]
    if world == 1:
        return [(0, sum(nq))]
    if len(wl.lengths) == 1:
        return partition.zigzag_ranges(nq[0], world, rank)
    cu = np.concatenate([[0], np.cumsum(nq)])
    out = []
    for s in partition.balance_sequences(wl.lengths, world, rank):
        a, b = int(cu[s]), int(cu[s + 1])
        if a == b:
            continue
        if out and out[-1][1] == a:
            out[-1] = (out[-1][0], b)
        else:
            out.append((a, b))
    return out


def plan_units(wl, ranges):
    """(rows, causal (i, j) pairs) of the query blocks in `ranges`."""
    nq = [(L + wl.B - 1) // wl.B for L in wl.lengths]
    cu = np.concatenate([[0], np.cumsum(nq)])
    rows = pairs = 0
    for a, b in ranges:
        for g in range(a, b):
            s = int(np.searchsorted(cu, g, side="right") - 1)
            L, qb = wl.lengths[s], g - int(cu[s])
            i0, i1 = qb * wl.B, min(L, (qb + 1) * wl.B)
            rows += i1 - i0
            pairs += (i1 * (i1 + 1) - i0 * (i0 + 1)) // 2
    return rows, pairs


def algorithmic(wl, nnz, ranges=None):
    """Algorithmic bytes / flops of the three kernels over the query blocks of
    `ranges` (the whole context by default): one launch each at N = 1."""
    rows, pairs = plan_units(wl, ranges or [(0, sum((L + wl.B - 1) // wl.B
                                                    for L in wl.lengths))])
    el = 2 if wl.dtype == "bf16" else 4
    nqb = sum((l + wl.B - 1) // wl.B for l in wl.lengths)
    map_bytes = nnz * wl.Hs * wl.B * wl.B * el
    av_bytes = (map_bytes + wl.ntok * wl.Hkv * wl.d * el + rows * wl.Hr * wl.d * el
                + wl.Hr * wl.Hs * el + 4 * nnz + 8 * (nqb + 1))
    stats_flops = 2.0 * wl.d * pairs * wl.Hs          # one QK^T over the causal triangle
    extract_bytes = map_bytes
    av_flops = 2.0 * nnz * wl.B * wl.B * (wl.Hs * wl.Hr + wl.d * wl.Hr)
    return dict(av_bytes=av_bytes, stats_flops=stats_flops, extract_bytes=extract_bytes,
                av_flops=av_flops, map_bytes=map_bytes, rows=rows)


def dense_attention_ms(wl, dev, stream, ev, warmup, steps):
    """Mean time of torch's causal SDPA for the receiver layer (Hr query heads,
    Hkv KV heads, d) over the workload's sequences; a library call, reported
    beside the fused kernel as context, never on our path."""
    import torch.nn.functional as F
    g = torch.Generator(device=dev).manual_seed(7)
    dt = wl.torch_dtype
    seqs = []
    for L in wl.lengths:
        q = torch.randn(1, wl.Hr, L, wl.d, device=dev, dtype=dt, generator=g)
        k = torch.randn(1, wl.Hkv, L, wl.d, device=dev, dtype=dt, generator=g)
        v = torch.randn(1, wl.Hkv, L, wl.d, device=dev, dtype=dt, generator=g)
        seqs.append((q, k, v))

    def run():
        for q, k, v in seqs:
            F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(steps):
        run()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def max_over_ranks(x, world, device):
    """The largest value of x over all ranks (every rank gets it); x itself at N=1."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_env():
    """(rank, world, local_rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def layer_jobs(wl, rank, world):
    """The layers this rank runs: (sender layers [index], receiver layers
    [(receiver, layer, sender index)]).  One-layer workloads: sender 0 and
    its receiver; the multi-receiver workload: every sender layer and every
    receiver layer through the layer table at N = 1, whole sender layers with
    the receiver layers that read them at N > 1."""
    if wl.sender_layers == 1:
        return [0], [(0, 0, 0)]
    if world == 1:
        senders = list(range(wl.sender_layers))
        readers = [(r, l) for r, (_, n, _) in enumerate(wl.receivers) for l in range(n)]
    else:
        senders, readers = partition.layer_split(wl.sender_layers, wl.receivers, world, rank)
    return senders, [(r, l, wl.receivers[r][2][l]) for r, l in readers]


def layer_inputs(wl, senders, receivers):
    """Host tensors: {sender layer: (Q, K)}, {(receiver, layer): (V, W)}."""
    if wl.sender_layers == 1:
        x = synth.single_layer(wl)
        return {0: (x.Q, x.K)}, {(0, 0): (x.V, x.W)}
    return ({s: synth.sender_layer(wl, s) for s in senders},
            {(r, l): synth.receiver_layer(wl, r, l) for r, l, _ in receivers})


def bench_ours(args, wl, rank, world, local_rank):
    from cross_model_attention_block_b200 import mapflow as mfb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ctx = mfb.Context.make(wl.lengths, wl.Hs, wl.d, wl.B, wl.band_bias, wl.band_width,
                           wl.torch_dtype, device=dev)
    nqb, nblocks = ctx.layout_sizes()
    senders, receivers = layer_jobs(wl, rank, world)
    host_s, host_r = layer_inputs(wl, senders, receivers)
    # query-block ranges of a sender layer on this rank: the rank's share of a
    # one-layer workload, the whole layer when layers are split
    plan = rank_plan(wl, rank, world) if wl.sender_layers == 1 else [(0, nqb)]
    # V in its page pool where the workload says so (16-token pages, a random
    # permutation of the pages of the whole batch)
    host_pages = {}
    contig_v = {key: V for key, (V, W) in host_r.items()}  # the oracle's V
    if wl.paged:
        for key, (V, W) in host_r.items():
            pool, table = synth.paged_v(V, wl.lengths, synth.page_rng(wl))
            host_r[key] = (pool, W)
            host_pages[key] = table
    # per step, the inputs: Q, K of every sender layer, V (or its pool) and W
    # of every receiver layer, and the page tables
    in_keys = ([("Q", s) for s in senders] + [("K", s) for s in senders]
               + [("V", k) for k in host_r] + [("W", k) for k in host_r]
               + [("T", k) for k in host_pages])
    host_in = {}
    for s in senders:
        host_in[("Q", s)], host_in[("K", s)] = host_s[s]
    for k, (V, W) in host_r.items():
        host_in[("V", k)], host_in[("W", k)] = V, W
    for k, t in host_pages.items():
        host_in[("T", k)] = t
    dev_in = {k: host_in[k].to(dev) for k in in_keys}
    lse = torch.empty((wl.Hs, wl.ntok), dtype=torch.float32, device=dev)
    mass = torch.empty((nblocks,), dtype=torch.float32, device=dev)
    # one cache per (sender layer, range), sized to the range's causal blocks
    caches = {(s, r): mfb.Cache(ctx, capacity=ctx.range_blocks(*r), device=dev)
              for s in senders for r in plan}
    outs = {(r, l): torch.empty((wl.ntok, wl.Hr, wl.d), dtype=wl.torch_dtype, device=dev)
            for r, l, _ in receivers}
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def run(din, dout, marks=None):
        """One step: every sender layer's statistics, then its selection and
        extraction (range by range), then every receiver layer's fused
        kernel on its sender layer's cache.  marks: list collecting
        (stage, start event, end event)."""
        def timed(stage, fn):
            if marks is None:
                fn()
                return
            a, b = ev(), ev()
            a.record(stream)
            fn()
            b.record(stream)
            marks.append((stage, a, b))

        for s in senders:
            Qd, Kd = din[("Q", s)], din[("K", s)]
            timed(0, lambda: [mfb.block_stats(ctx, Qd, Kd, lse=lse, mass=mass, qb_range=r)
                              for r in plan])
            timed(1, lambda: [mfb.select_extract(ctx, Qd, Kd, lse, mass, wl.tau,
                                                 cache=caches[(s, r)], qb_range=r)
                              for r in plan])
        for rr, l, s in receivers:
            key = (rr, l)
            table = din.get(("T", key))

            def av():
                for r in plan:
                    c = caches[(s, r)]
                    mfb.mapped_av(c, wl.Hr, din[("W", key)], din[("V", key)], wl.Hkv,
                                  page_table=table, O=dout[key],
                                  workspace=getattr(c, "_av_ws", None), qb_range=r)
            timed(2, av)

    def step(marks=None):
        run(dev_in, outs, marks)

    for _ in range(args.warmup):
        step()
    mfb.sync_status()
    nnz = {s: sum(caches[(s, r)].nnz for r in plan) for s in senders}
    alg_s = [algorithmic(wl, nnz[s], plan) for s in senders]
    alg = {"stats_flops": sum(a["stats_flops"] for a in alg_s),
           "extract_bytes": sum(a["extract_bytes"] for a in alg_s),
           "av_bytes": sum(algorithmic(wl, nnz[s], plan)["av_bytes"] for _, _, s in receivers),
           "map_bytes": sum(a["map_bytes"] for a in alg_s)}

    marks = [[] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for k in range(args.steps):
        step(marks[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    ms = t_start.elapsed_time(t_end)
    stage = np.zeros((args.steps, 3))
    for k, m in enumerate(marks):
        for st, a, b in m:
            stage[k, st] += a.elapsed_time(b)
    stage_ms = stage.mean(axis=0)
    ms = max_over_ranks(ms, world, dev)
    mfb.sync_status()

    # context only: dense causal GQA attention of the same receiver layer
    # (torch scaled_dot_product_attention, bf16, per sequence), the cost the
    # fused kernel stands in for (per receiver layer)
    dense_ms = dense_attention_ms(wl, dev, stream, ev, args.warmup, min(args.steps, 10))
    dense_ms = max_over_ranks(dense_ms, world, dev)

    # end to end through the C ABI: every step copies its inputs in from
    # pinned host memory and its outputs back, as a serving loop would: the
    # copies run on two copy streams into double-buffered device tensors, so
    # step k's H2D and step k-1's D2H overlap step k-1's and k's kernels
    hIn = {k: host_in[k].pin_memory() for k in in_keys}
    hOut = {k: torch.empty(o.shape, dtype=o.dtype).pin_memory() for k, o in outs.items()}
    dIn = [dev_in, {k: torch.empty_like(t) for k, t in dev_in.items()}]
    dOut = [outs, {k: torch.empty_like(o) for k, o in outs.items()}]
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    in_ready = [ev() for _ in range(2)]
    used = [ev() for _ in range(2)]      # step's kernels done with buffer set b
    out_read = [ev() for _ in range(2)]  # outputs b copied back

    def e2e_run(nsteps):
        def h2d(b):
            with torch.cuda.stream(h2d_s):
                for k in in_keys:
                    dIn[b][k].copy_(hIn[k], non_blocking=True)
                in_ready[b].record(h2d_s)

        h2d_s.wait_stream(stream)  # nothing starts before the timed region does
        h2d(0)
        for k in range(nsteps):
            b = k % 2
            if k + 1 < nsteps:
                if k >= 1:
                    h2d_s.wait_event(used[1 - b])  # step k-1 is done with the other set
                h2d(1 - b)
            stream.wait_event(in_ready[b])
            if k >= 2:
                stream.wait_event(out_read[b])     # step k-2's outputs have been read back
            run(dIn[b], dOut[b])
            used[b].record(stream)
            d2h_s.wait_event(used[b])
            with torch.cuda.stream(d2h_s):
                for key, o in dOut[b].items():
                    hOut[key].copy_(o, non_blocking=True)
                out_read[b].record(d2h_s)
        stream.wait_stream(d2h_s)

    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    mfb.sync_status()
    h2d = sum(t.numel() * t.element_size() for t in hIn.values())
    d2h = sum(t.numel() * t.element_size() for t in hOut.values())
    # the CPU baseline's inputs: the first sender layer and its first reader
    s0 = senders[0]
    k0 = next((rr, l) for rr, l, s in receivers if s == s0)
    x = synth.LayerInputs(*host_s[s0], contig_v[k0], host_r[k0][1])

    if rank != 0:
        return
    peaks, src = load_peaks()
    ms_step = ms / args.steps
    tokens = wl.ntok  # the context of one step, split across the ranks
    t_stats, t_sel, t_av = stage_ms
    av_gbs = alg["av_bytes"] / (t_av * 1e-3) / 1e9
    stats_tf = alg["stats_flops"] / (t_stats * 1e-3) / 1e12
    ext_gbs = alg["extract_bytes"] / (t_sel * 1e-3) / 1e9
    hbm = peaks["hbm_gbs"]
    # the statistics kernel runs for milliseconds at a time between the other
    # stages, at the clocks of a short burst: its fraction is taken of the
    # burst cuBLAS figure; the sustained (power-capped) figure is given beside it
    tens = peaks["bf16_tflops"]
    tens_sust = peaks["bf16_tflops_sustained"]
    kernels = {
        "mapped_av": {"bound": "hbm", "achieved": av_gbs, "peak": hbm, "unit": "GB/s",
                      "frac": av_gbs / hbm, "ms": t_av,
                      "algorithmic_bytes": alg["av_bytes"]},
        "block_stats": {"bound": "tensor", "achieved": stats_tf, "peak": tens,
                        "unit": "TFLOP/s", "frac": stats_tf / tens, "ms": t_stats,
                        "peak_kind": "burst bf16",
                        "frac_of_sustained_peak": stats_tf / tens_sust,
                        "algorithmic_flops": alg["stats_flops"]},
        "select_extract": {"bound": "hbm", "achieved": ext_gbs, "peak": hbm, "unit": "GB/s",
                           "frac": ext_gbs / hbm, "ms": t_sel,
                           "algorithmic_bytes": alg["extract_bytes"]},
    }
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    roof = {k: v for k, v in kernels[dom].items() if k in ("bound", "achieved", "peak", "unit",
                                                            "frac")}
    roof["kernel"] = dom
    roof["peak_source"] = f"{src} (MEASURED_PEAKS.json)" if src == "measured" else src
    roof["traffic"] = kernel_traffic(dom, wl.name)
    line = {
        "metric": METRIC, "value": tokens / (ms_step * 1e-3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.ntok, "Hs": wl.Hs, "Hr": wl.Hr,
                   "Hkv": wl.Hkv, "d": wl.d, "B": wl.B, "tau": wl.tau,
                   "sender_layers": len(senders), "receiver_layers": len(receivers),
                   "paged_v": bool(wl.paged),
                   "kept_blocks": sum(nnz.values()), "causal_blocks": nblocks * len(senders),
                   "map_gb": alg["map_bytes"] / 1e9,
                   "l2": "inputs larger than L2 (kept map >> 126 MB); no flush",
                   "parallelism": ("single GPU" if world == 1 else
                                   f"query-block ranges x{world} (rank 0: {plan})"
                                   if wl.sender_layers == 1 else
                                   f"sender layers with their readers x{world} "
                                   f"(rank 0: {senders})")},
        "mapped_av_gbs": av_gbs, "mapped_av_hbm_frac": av_gbs / hbm,
        "compress_tokens_per_s": wl.ntok * len(senders) / ((t_stats + t_sel) * 1e-3),
        "stats_tensor_frac": stats_tf / tens,
        "stats_tensor_frac_of_sustained": stats_tf / tens_sust,
        "layer_prefill_ms": t_av / len(receivers),
        "dense_sdpa_ms_context": dense_ms,
        "stage_ms": {"block_stats": t_stats, "select_extract": t_sel, "mapped_av": t_av},
        "roofline": roof, "kernels": kernels,
        "clocks": clk,
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * len(plan) * (LAUNCHES_COMPRESS * len(senders)
                                                  + LAUNCHES_MAPPED * len(receivers)),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample(wl, x)
    print(json.dumps(line), flush=True)


# kernels of ours launched per query-block range and step: per sender layer,
# stats (meta, stats, mass reduce) and select and extract (meta, qb map,
# select, scan, fill, extract); per receiver layer, mapped AV (group meta, V
# regrouping, fused kernel)
LAUNCHES_COMPRESS = 9
LAUNCHES_MAPPED = 3


def bench_rounds(args):
    """Round-level selection on the multi-turn workload (one GPU)."""
    from cross_model_attention_block_b200 import mapflow as mfb
    wl = synth.workloads()["multi_turn_rounds_n8192"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    ctx = mfb.Context.make(wl.lengths, wl.Hs, wl.d, wl.B, wl.band_bias, wl.band_width,
                           wl.torch_dtype, device=dev)
    layers = [tuple(t.to(dev) for t in synth.sender_layer(wl, l) + synth.receiver_layer(wl, 0, l))
              for l in range(wl.sender_layers)]
    nqb, nblocks = ctx.layout_sizes()
    lse = torch.empty((wl.Hs, wl.ntok), dtype=torch.float32, device=dev)
    mass = torch.empty((nblocks,), dtype=torch.float32, device=dev)
    cache = mfb.Cache(ctx, device=dev)
    blocks = mfb.Cache(ctx, device=dev)
    O = torch.empty((wl.ntok, wl.Hr, wl.d), dtype=wl.torch_dtype, device=dev)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    mapped = range(wl.watershed, wl.sender_layers)

    def step(m=None):
        rec = (lambda i: m[i].record(stream)) if m else (lambda i: None)
        Qw, Kw = layers[wl.watershed][:2]
        rec(0)
        mfb.block_stats(ctx, Qw, Kw, lse=lse, mass=mass)
        mfb.select_rounds(ctx, mass, wl.rounds[0], wl.tau, cache=cache)
        rec(1)
        for l in mapped:
            Q, K, V, W = layers[l]
            mfb.block_stats(ctx, Q, K, lse=lse, mass=mass)
            mfb.extract(ctx, Q, K, lse, cache)
            mfb.mapped_av(cache, wl.Hr, W, V, wl.Hkv, O=O, workspace=getattr(cache, "_av_ws", None))
        rec(2)

    for _ in range(args.warmup):
        step()
    mfb.sync_status()
    marks = [[ev() for _ in range(3)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    for k in range(args.steps):
        step(marks[k])
    torch.cuda.synchronize()
    clk = clocks.stop()
    mfb.sync_status()
    t = np.array([[m[0].elapsed_time(m[1]), m[1].elapsed_time(m[2])] for m in marks]).mean(0)
    # the block selection of the watershed layer at the same tau, for the kept fraction
    Qw, Kw = layers[wl.watershed][:2]
    mfb.block_stats(ctx, Qw, Kw, lse=lse, mass=mass)
    mfb.select_extract(ctx, Qw, Kw, lse, mass, wl.tau, cache=blocks)
    mfb.sync_status()
    ms = float(t.sum())
    line = {
        "mode": "rounds", "metric": "round-level selection: tokens/s of one step (selection at "
        "the watershed layer, then statistics, extraction and the fused kernel on every later "
        "layer)", "value": wl.ntok / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.ntok, "rounds": len(wl.rounds[0]) - 1,
                   "sender_layers": wl.sender_layers, "watershed": wl.watershed,
                   "mapped_layers": len(mapped), "Hs": wl.Hs, "Hr": wl.Hr, "Hkv": wl.Hkv,
                   "B": wl.B, "tau": wl.tau},
        "stage_ms": {"watershed_stats_and_round_selection": float(t[0]),
                     "mapped_layers": float(t[1]),
                     "per_mapped_layer": float(t[1]) / len(mapped)},
        "kept_blocks": {"rounds": cache.nnz, "blocks_same_tau": blocks.nnz,
                        "causal": nblocks},
        "cache_gb_per_layer": {"rounds": cache.nnz * wl.Hs * wl.B * wl.B * 2 / 1e9,
                               "blocks_same_tau": blocks.nnz * wl.Hs * wl.B * wl.B * 2 / 1e9},
        "clocks": clk,
        "gpu_launches": args.steps * (9 + len(mapped) * 9),
    }
    print(json.dumps(line), flush=True)


def bench_overlap(args):
    """Receiver prefill: fetch of a mapped layer's cache from pinned host memory
    overlapped with the recompute of the receiver's first layers (one GPU)."""
    import torch.nn.functional as F
    from cross_model_attention_block_b200 import mapflow as mfb
    from cross_model_attention_block_b200 import overlap as ov
    wl = synth.workloads()["multi_receiver_n16384"]
    n_recompute, chunks = 2, 8
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    ctx = mfb.Context.make(wl.lengths, wl.Hs, wl.d, wl.B, wl.band_bias, wl.band_width,
                           wl.torch_dtype, device=dev)
    Q, K = (t.to(dev) for t in synth.sender_layer(wl, 0))
    lse, mass = mfb.block_stats(ctx, Q, K)
    src = mfb.select_extract(ctx, Q, K, lse, mass, wl.tau)
    mfb.sync_status()
    nnz = src.nnz
    host = mfb.Cache(ctx, capacity=nnz, device="cpu", pin=True)
    mfb.cache_offload(src, host)
    torch.cuda.synchronize()
    del src, Q, K
    target = mfb.Cache(ctx, capacity=nnz, device=dev)
    V, W = (t.to(dev) for t in synth.receiver_layer(wl, 0, 0))
    O = torch.empty((wl.ntok, wl.Hr, wl.d), dtype=wl.torch_dtype, device=dev)
    layer = ov.MappedLayer(host, target, W, V, O)
    g = torch.Generator(device=dev).manual_seed(11)
    q = torch.randn(1, wl.Hr, wl.ntok, wl.d, device=dev, dtype=wl.torch_dtype, generator=g)
    kv = torch.randn(1, wl.Hkv, wl.ntok, wl.d, device=dev, dtype=wl.torch_dtype, generator=g)
    # stand-in for one of the receiver's own first layers (dense causal attention)
    recompute = [lambda: F.scaled_dot_product_attention(q, kv, kv, is_causal=True,
                                                        enable_gqa=True)] * n_recompute
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    copy = torch.cuda.Stream()

    def timed(fn):
        a, b = ev(), ev()
        a.record(stream)
        out = fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b), a, out

    res = {"serial": [], "overlapped": [], "fetch": [], "recompute": [], "mapped": []}
    for k in range(args.warmup + args.steps):
        t_s, _, _ = timed(lambda: ov.prefill(recompute, [layer], wl.Hr, wl.Hkv, chunks,
                                             serial=True))
        t_o, a, evs = timed(lambda: ov.prefill(recompute, [layer], wl.Hr, wl.Hkv, chunks,
                                               copy_stream=copy))
        t_f = a.elapsed_time(evs[-1])          # start to the last range landed
        t_r, _, _ = timed(lambda: [f() for f in recompute])
        t_m, _, _ = timed(lambda: [mfb.mapped_av(target, wl.Hr, W, V, wl.Hkv, O=O, qb_range=r)
                                   for r in ov.chunk_ranges(target.nqb, chunks)])
        if k >= args.warmup:
            for key, v in (("serial", t_s), ("overlapped", t_o), ("fetch", t_f),
                           ("recompute", t_r), ("mapped", t_m)):
                res[key].append(v)
    mfb.sync_status()
    med = {k: float(np.median(v)) for k, v in res.items()}
    fetch_bytes = (nnz * wl.Hs * wl.B * wl.B * 2 + 4 * nnz + 16 * (target.nqb + 1))
    line = {
        "mode": "overlap", "metric": "receiver prefill ms: cache fetch from host memory "
        "overlapped with the early-layer recompute, against the same calls in series",
        "value": med["overlapped"], "unit": "ms", "higher_is_better": False, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.ntok, "recompute_layers": n_recompute,
                   "recompute_stand_in": "torch causal SDPA (Hr query heads, Hkv KV heads)",
                   "mapped_layers": 1, "chunks": chunks, "fetch_gb": fetch_bytes / 1e9,
                   "source": "pinned host memory"},
        "serial_ms": med["serial"], "overlapped_ms": med["overlapped"],
        "saved_ms": med["serial"] - med["overlapped"],
        "fetch_ms": med["fetch"], "fetch_gbs": fetch_bytes / (med["fetch"] * 1e-3) / 1e9,
        "recompute_ms": med["recompute"], "mapped_ms": med["mapped"],
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_bf16_n32768")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", choices=["path", "rounds", "overlap"], default="path")
    args = ap.parse_args(argv)
    if args.mode != "path" and args.impl == "ours":
        return bench_rounds(args) if args.mode == "rounds" else bench_overlap(args)
    wl = synth.workloads()[args.workload]
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        if rank == 0:
            bench_reference(args, wl)
        return 0
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        bench_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
