#!/usr/bin/env python
"""Benchmark of the W4 path on B200: prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (``value``): W4A16 GEMV HBM GB/s at M=1 over the 8B decode sweep -- one step is
one M=1 GEMV through each of the four (K, N) shapes {(4096,4096), (4096,1024),
(4096,14336), (14336,4096)} (asymmetric INT4, group 128, weights quantized with the
20-ratio clip search), i.e. 73.6 MB of algorithmic bytes. The weights rotate over R
prepacked copies whose total size is at least 3x the 126 MB L2, so no step reads weights
from L2. Every other row of the path is measured in ``rows`` with its own roofline: the W4A8
prefill GEMM (M=4096, both shapes), the FP8 row quant, the quantizer on the full 8B weight
set (6.98e9 weights, 20 ratios), the MoE grouped GEMM and the GEMV at M=4 and 16.

Multi-GPU: every rank runs the same per-GPU work on its own weights (weak scaling, no
collective on the data path); timings are CUDA events, max over ranks.
``--impl reference`` times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "W4A16 GEMV HBM GB/s (M=1) & W4A8 GEMM TFLOP/s; % of B200 roofline"
DECODE_SHAPES = [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)]  # (K, N)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# DRAM bytes per launch of the roofline kernels, from one ncu capture each
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by kernel and shape, with the SHA-1 of
# the kernel's source file at capture time: a number is reported only while the source is
# unchanged (otherwise the counters describe a different kernel and "traffic" is null).
NCU_TRAFFIC = {
    # profiles/w4a16_gemv_m1_k14336_n4096_full.md: the kernel's own bytes (a chain of launches
    # without the L2 prefetch of the next launch's weights, caches flushed between launches)
    "w4a16_gemv M1 K14336xN4096": {"bytes": 31290624, "sha1": "b089e61bdc768133cc203b6be361c562219a81f8"},
    # profiles/w4a16_tc_m4_k14336_n4096_full.md: w4a16_gemm_tc at M = 4 (one launch)
    "w4a16_tc M4 K14336xN4096": {"bytes": 32818432, "sha1": "9fc6804e09b9a30d55bf9586da1ef1ca258aba9e"},
    # profiles/w4a8_gemm_prefill_traffic.md (median of 11 launches per shape)
    "w4a8_gemm M4096 K3840xN15360": {"bytes": 153379840, "sha1": "2fc13ed112d7918580956d35db9107959347192d"},
    "w4a8_gemm M4096 K15360xN3840": {"bytes": 179415552, "sha1": "2fc13ed112d7918580956d35db9107959347192d"},
}


# Warp instructions issued per weight by the quantizer (smsp__inst_executed.sum of one launch
# over the weights it quantized), from one ncu capture, with the SHA-1 of its source file.
QUANT_ISSUE = {
    # profiles/w4_quantize_q_proj_4096x4096_full.md: 177,504,361 / 16,777,216 weights
    "w4_quantize g128 asym 20 ratios": {"inst_per_weight": 10.5801, "sha1": "699b710fb8687d7611083e0cc6c3af238594311d"},
}


def source_sha1(rel):
    import hashlib
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()


def traffic_for(key, rel):
    t = NCU_TRAFFIC.get(key)
    if not t or t["sha1"] != source_sha1(rel):
        return None
    return t["bytes"]


def gemv_bytes(M, N, K, g=128):
    """Algorithmic bytes of one W4A16 GEMV: packed codes, 2+2 bytes of scale and zero per
    group, the bf16 activations and the bf16 output."""
    return N * K // 2 + N * (K // g) * 4 + 2 * M * K + 2 * M * N


# ------------------------------------------------------------------ clocks

class Clocks:
    """Samples SM clock and clock-event reasons with NVML every ~2 ms while the timed
    region runs (from just before its first launch until after its final synchronize)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.mhz, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:  # no NVML: report no samples
            self.nv = None
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.mhz.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *exc):
        self._stop.set()
        if self.nv:
            self.t.join(timeout=2)

    def summary(self):
        return {"sm_mhz": float(np.median(self.mhz)) if self.mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.mhz)}


# ------------------------------------------------------------------ timing helpers

def max_over_ranks(vals, dev):
    """Element-wise maximum of a list of floats over all ranks (the job's time is its
    slowest rank's); identity without a process group."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return list(vals)
    t = torch.tensor(vals, dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world, units_per_rank_step, ms_step):
    """Whole-job throughput: the units all ranks processed per step over the (max) step time."""
    return world * units_per_rank_step / (ms_step * 1e-3)


def time_region(fn, iters, stream=None, lead=None):
    """Device time (ms) of `iters` calls of fn, CUDA events on the launching stream.
    lead: GPU work (an L2 flush) enqueued after the synchronisation and before the start
    event. The host-side work of the first call (argument marshalling, tensor-map encoding,
    the launch) then overlaps it instead of leaving the GPU idle inside the timed interval,
    so that a single timed launch measures the kernel's device time."""
    stream = stream or torch.cuda.current_stream()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if lead is not None:
        lead()
    s.record(stream)
    for i in range(iters):
        fn(i)
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e)


def flush_l2(buf):
    buf.add_(1)


# ------------------------------------------------------------------ our arm

class Decode:
    """The decode sweep: quantize (GPU), prepack R copies per shape, M=1 activations.
    Step i runs one GEMV per shape on weight copy i % R; each step is captured once in a
    CUDA graph (the decode loop replays graphs, as serving engines do)."""

    def __init__(self, M, seed, dev, copies=None, tc=False):
        """tc: the tensor-core W4A16 (w4a16_gemm_tc, layout W4_LAYOUT_TC) instead of the GEMV."""
        from bit_gemm_wise_b200 import synth, w4
        self.w4 = w4
        self.M = M
        self.tc = tc
        layout = w4.W4_LAYOUT_TC if tc else w4.W4_LAYOUT_GEMV
        g = 128
        grid = synth.clip_grid_20()
        self.shapes = DECODE_SHAPES
        self.bytes_per_step = sum(gemv_bytes(M, N, K) for K, N in self.shapes)
        packed_per_step = sum(w4.w4_prepack_bytes(N, K, g, layout) for K, N in self.shapes)
        self.R = copies or max(2, -(-3 * L2_BYTES // packed_per_step))
        self.packed, self.x, self.y, self.ws = [], [], [], []
        # all shapes' activations and outputs live in one buffer each (16-byte aligned views),
        # so that a step's host copies are one copy in and one copy out
        xo = [0]
        yo = [0]
        for K, N in self.shapes:
            xo.append(xo[-1] + (M * K + 7) // 8 * 8)
            yo.append(yo[-1] + (M * N + 7) // 8 * 8)
        # two sets, so that a pipelined serving loop can copy step i + 1's activations in and
        # step i - 1's outputs out while step i runs (set 0 is the one the other rows use)
        self.xbufs = [torch.empty(xo[-1], dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.ybufs = [torch.empty(yo[-1], dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.xbuf, self.ybuf = self.xbufs[0], self.ybufs[0]
        self.xs, self.ys = [[], []], [[], []]
        for si, (K, N) in enumerate(self.shapes):
            W = synth.decode_weight(K, N, seed, device=dev)
            codes, scales, zeros, _ = w4.alloc_quantized(N, K, g, "asym", device=dev, chosen=False)
            w4.w4_quantize(W, N, K, g, "asym", grid, codes, scales, zeros, None)
            nb = w4.w4_prepack_bytes(N, K, g, layout)
            p = torch.empty(self.R * nb, dtype=torch.uint8, device=dev)
            w4.w4_prepack(codes, scales, zeros, N, K, g, "asym", layout, p[:nb])
            for r in range(1, self.R):
                p[r * nb:(r + 1) * nb].copy_(p[:nb])
            self.packed.append((p, nb))
            for b in range(2):
                xv = self.xbufs[b][xo[si]:xo[si] + M * K].view(M, K)
                xv.copy_(synth.decode_activation(M, K, seed, device=dev))
                self.xs[b].append(xv)
                self.ys[b].append(self.ybufs[b][yo[si]:yo[si] + M * N].view(M, N))
            self.x.append(self.xs[0][si])
            self.y.append(self.ys[0][si])
            self.ws.append(w4.alloc_tc_workspace(N, K, g, device=dev) if tc else
                           w4.alloc_gemv_workspace(N, K, g, device=dev))
            del W, codes, scales, zeros
        # each weight copy as a tensor view, made once (a call of the decode loop only looks it up)
        self.wviews = [[p[r * nb:(r + 1) * nb] for r in range(self.R)] for p, nb in self.packed]
        self.launches_per_step = len(self.shapes)
        self.graphs = None
        # consecutive GEMVs may overlap: each streams its weights while its predecessor
        # finishes (programmatic dependent launch); activations are read after it completes
        self.flags = w4.W4_OVERLAP_PREVIOUS

    def weights(self, si, i):
        return self.wviews[si][i % self.R]

    def gemv(self, si, i, next_si=None, prefetch=True, buf=0):
        """GEMV si of step i. It names the weights of the GEMV that follows it on the stream
        (the step's next shape, or the first shape of step i + 1; with next_si given, that
        shape's copy for step i + 1), which it brings into L2 once its own are requested."""
        (K, N) = self.shapes[si]
        x, y = self.xs[buf][si], self.ys[buf][si]
        if self.tc:
            self.w4.w4a16_gemm_tc(x, self.M, self.weights(si, i), N, K, 128, "asym", y, self.flags, self.ws[si])
            return
        if not prefetch:
            self.w4.w4a16_gemv(x, self.M, self.weights(si, i), N, K, 128, "asym", y, self.flags, self.ws[si])
            return
        if next_si is None:
            nsi, ni = (si + 1, i) if si + 1 < len(self.shapes) else (0, i + 1)
        else:
            nsi, ni = next_si, i + 1
        self.w4.w4a16_gemv_prefetch_next(x, self.M, self.weights(si, i), N, K, 128, "asym", y, self.flags,
                                         self.ws[si], self.weights(nsi, ni))

    def step_eager(self, i, buf=0):
        for si in range(len(self.shapes)):
            self.gemv(si, i, buf=buf)

    def step_grouped(self, i):
        """The step's four GEMVs as one grouped launch (w4a16_gemv_grouped)."""
        self.w4.w4a16_gemv_grouped(self.x, self.M, [p[(i % self.R) * nb:] for p, nb in self.packed],
                                   [N for K, N in self.shapes], [K for K, N in self.shapes], 128, "asym", self.y,
                                   self.flags)

    def graph_of(self, n_steps, first=0):
        """One CUDA graph holding n_steps consecutive decode steps (weights rotate over the
        copies), the GEMVs chained with programmatic dependent launches, as a decode graph
        holding a model's layers would be."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.side):
            for i in range(n_steps):
                self.step_eager(first + i)
        return g

    def shape_graph(self, si, n_launches):
        """n_launches GEMVs of one shape back to back (rotating weight copies)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.side):
            for i in range(n_launches):
                self.gemv(si, i, next_si=si)
        return g

    def capture(self, steps, warmup):
        self.step_eager(0)  # first calls set kernel attributes outside the capture
        torch.cuda.synchronize()
        self.side = torch.cuda.Stream()
        self.g_warm = self.graph_of(max(1, warmup))
        self.g_steps = self.graph_of(steps, first=warmup)
        torch.cuda.synchronize()


def run_ours(args, rank, world, dev):
    from bit_gemm_wise_b200 import synth, w4
    pk = peaks()
    dist = world > 1
    stream = torch.cuda.current_stream()

    dec = Decode(1, args.seed, dev)
    dec.capture(args.steps, args.warmup)
    dec.g_warm.replay()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # the timed region is exactly `steps` decode steps (one graph replay); it is repeated
    # (each repeat bracketed by synchronisations) until the clock sampler has seen enough of
    # the load, and the median repeat is reported with the spread
    reps, region_ms = 0, []
    with Clocks(torch.cuda.current_device()) as clk:
        t_end = time.perf_counter() + args.min_seconds
        while reps < args.min_repeats or time.perf_counter() < t_end:
            region_ms.append(time_region(lambda i: dec.g_steps.replay(), 1, stream))
            reps += 1
    if dist:
        torch.distributed.barrier()
    ms = max_over_ranks([float(np.median(region_ms))], dev)[0]
    ms_step = ms / args.steps
    value = job_throughput(world, dec.bytes_per_step, ms_step) / 1e9

    # per-shape launch times: a graph of many launches of one shape (rotating weight copies,
    # chained like the decode step), events around each replay, time per launch
    per_shape = {}
    for si, (K, N) in enumerate(dec.shapes):
        n_l = 8 * dec.R
        gs = dec.shape_graph(si, n_l)
        gs.replay()
        t_ms = float(np.median([time_region(lambda i: gs.replay(), 1, stream) for _ in range(9)])) / n_l
        per_shape[f"K{K}xN{N}"] = {"us": round(t_ms * 1e3, 3),
                                   "GBps": round(gemv_bytes(1, N, K) / (t_ms * 1e-3) / 1e9, 1)}
        del gs

    # roofline of the dominant kernel: the shape whose GEMV launch takes longest;
    # algorithmic bytes of one launch over its event-timed duration
    dom = max(per_shape, key=lambda k: per_shape[k]["us"])
    dK, dN = (int(v) for v in dom[1:].split("xN"))
    dbytes = gemv_bytes(1, dN, dK)
    dach = dbytes / (per_shape[dom]["us"] * 1e-6) / 1e9
    roofline = {"bound": "hbm", "achieved": round(dach, 1), "peak": pk["hbm"], "unit": "GB/s",
                "frac": round(dach / pk["hbm"], 4),
                "traffic": traffic_for(f"w4a16_gemv M1 {dom}", "bit_gemm_wise_b200/csrc/w4a16_gemv.cu"),
                "kernel": f"w4a16_gemv M=1 {dom}", "bytes_per_launch": dbytes,
                "peak_source": f"{pk['src']} copy bandwidth (of {pk['src']})",
                "frac_of_spec_8000": round(dach / 8000.0, 4),
                "step_frac": round(value / world / pk["hbm"], 4)}

    # e2e through the public Python API with host buffers, every step: pinned h2d of the
    # activations (the four shapes' vectors packed in one buffer: one copy), the four
    # w4a16_gemv_prefetch_next calls, d2h of the outputs (one buffer, one copy)
    xh = dec.xbuf.cpu().pin_memory()
    yh = torch.empty(dec.ybuf.shape, dtype=dec.ybuf.dtype).pin_memory()
    h2d = xh.numel() * 2
    d2h = yh.numel() * 2

    def e2e_step(i):
        dec.xbuf.copy_(xh, non_blocking=True)
        dec.step_eager(i)
        yh.copy_(dec.ybuf, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    eager_ms = time_region(e2e_step, args.steps, stream) / args.steps
    # the same step captured once per weight copy as a CUDA graph (pinned-host copies of x in,
    # the four API calls, copies of y out), replayed as a serving loop would
    e2e_graphs = []
    torch.cuda.synchronize()
    for r in range(dec.R):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=dec.side):
            e2e_step(r)
        e2e_graphs.append(gr)
    for i in range(args.warmup):
        e2e_graphs[i % dec.R].replay()
    serial_ms = time_region(lambda i: e2e_graphs[i % dec.R].replay(), args.steps, stream) / args.steps
    del e2e_graphs
    # the serving loop pipelined over two streams, `steps` steps in one graph: every step still
    # copies its activations in from pinned host memory and its outputs out, but step i + 1's
    # copy in and step i's copy out run on a copy stream while the GEMVs of the neighbouring
    # step run (two device buffer sets; events order each buffer's reuse)
    yhs = [yh, torch.empty(dec.ybuf.shape, dtype=dec.ybuf.dtype).pin_memory()]
    ts = torch.cuda.Stream()

    def pipelined(first):
        cs = torch.cuda.current_stream()
        n = args.steps
        x_in = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        fork, join = torch.cuda.Event(), torch.cuda.Event()
        fork.record(cs)
        ts.wait_stream(cs)
        with torch.cuda.stream(ts):
            dec.xbufs[0].copy_(xh, non_blocking=True)
            x_in[0].record(ts)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                with torch.cuda.stream(ts):
                    if i >= 1:
                        ts.wait_event(done[i - 1])  # step i - 1 used the set step i + 1 fills
                    dec.xbufs[(i + 1) % 2].copy_(xh, non_blocking=True)
                    x_in[i + 1].record(ts)
            cs.wait_event(x_in[i])
            dec.step_eager(first + i, buf=b)
            done[i].record(cs)
            with torch.cuda.stream(ts):
                ts.wait_event(done[i])
                yhs[b].copy_(dec.ybufs[b], non_blocking=True)
        join.record(ts)
        cs.wait_event(join)

    torch.cuda.synchronize()
    g_pipe = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_pipe, stream=dec.side):
        pipelined(args.warmup)
    g_pipe.replay()
    torch.cuda.synchronize()
    e2e_ms = float(np.median([time_region(lambda i: g_pipe.replay(), 1, stream) for _ in range(5)])) / args.steps
    del g_pipe
    e2e_ms, eager_ms, serial_ms = max_over_ranks([e2e_ms, eager_ms, serial_ms], dev)
    e2e_val = job_throughput(world, dec.bytes_per_step, e2e_ms) / 1e9
    eager_val = job_throughput(world, dec.bytes_per_step, eager_ms) / 1e9
    serial_val = job_throughput(world, dec.bytes_per_step, serial_ms) / 1e9

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 x int4 -> fp32 accumulate", "data": "synthetic (seeded; no checkpoint or dataset)",
        "config": {"workload": "decode GEMV sweep (K,N) in {(4096,4096),(4096,1024),(4096,14336),(14336,4096)}, "
                               "M=1, INT4 asym group 128, 20-ratio MSE clip",
                   "bytes_per_step": dec.bytes_per_step, "weight_copies": dec.R,
                   "l2": f"inputs larger than L2: weights rotate over {dec.R} copies "
                         f"({dec.R * sum(nb for _, nb in dec.packed) / 1e6:.0f} MB > 3 x L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "per_shape": per_shape,
        "gpu_launches": dec.launches_per_step * args.steps,
        "clocks": clk.summary(),
        "timing": {"repeats": reps, "region_ms_median": round(float(np.median(region_ms)), 5),
                   "region_ms_min": round(min(region_ms), 5), "region_ms_max": round(max(region_ms), 5),
                   "how": "each repeat: one graph replay of exactly `steps` decode steps, CUDA events on the "
                          "launching stream, synchronised on both sides; value from the median repeat"},
        "e2e": {"value": round(e2e_val, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "per step: one pinned-host copy of the four activation vectors in, the four "
                       "w4a16_gemv_prefetch_next API calls, one copy of the four outputs out; `steps` steps "
                       "in one CUDA graph, the copies on a second stream overlapping the neighbouring steps' "
                       "GEMVs (two device buffer sets), median of 5 replays",
                "serial_value": round(serial_val, 1),
                "serial_how": "the same step with its copies in line, one graph per step",
                "eager_value": round(eager_val, 1)},
    }
    # the other rows are single-GPU measurements: taken at N = 1 only, so that a scaling run
    # times the headline alone
    if not args.headline_only and world == 1:
        out["rows"] = measure_rows(args, dev, pk)
    del dec
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(args.seed, budget_s=args.cpu_seconds)
    return out


ROW_GROUPS = ("gemv", "prefill", "moe", "quantize")


def measure_rows(args, dev, pk):
    """Every other row of the path, each timed with CUDA events (after warm-up)."""
    from bit_gemm_wise_b200 import synth, w4
    rows = {}
    fp8_peak = 2.0 * pk["bf16"]  # dense FP8 = 2x dense BF16 (nominal ratio), burst
    want = set(args.rows.split(",")) if args.rows else set(ROW_GROUPS)

    # GEMV at M = 4 and 16 (bound by the CUDA cores' issue rate): GB/s, and the FMA work as a
    # fraction of the CUDA-core fp32 FMA peak (148 SMs x 128 lanes x 2 flop x 1965 MHz)
    fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12
    if "gemv" in want:
        # the same M = 1 decode step as one grouped launch of its four independent GEMVs (the
        # per-launch phases paid once per step instead of once per GEMV), graph-replayed
        d = Decode(1, args.seed, dev)
        d.step_grouped(0)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        n = 8 * d.R
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=side):
            for i in range(n):
                d.step_grouped(i)
        gr.replay()
        ms = float(np.median([time_region(lambda i: gr.replay(), 1) for _ in range(9)])) / n
        gbps = d.bytes_per_step / (ms * 1e-3) / 1e9
        rows["w4a16_gemv_grouped_step_M1"] = {
            "value": round(gbps, 1), "unit": "GB/s", "us_per_step": round(ms * 1e3, 2),
            "roofline": {"bound": "hbm", "achieved": round(gbps, 1), "peak": pk["hbm"], "unit": "GB/s",
                         "frac": round(gbps / pk["hbm"], 4)},
            "note": "the headline's four decode GEMVs (same bytes) as one w4a16_gemv_grouped launch per step"}
        del d, gr
    for M in ((4, 16) if "gemv" in want else ()):
        d = Decode(M, args.seed, dev)
        d.capture(6 * d.R, 3)
        d.g_warm.replay()
        ms = float(np.median([time_region(lambda i: d.g_steps.replay(), 1) for _ in range(5)])) / (6 * d.R)
        flops = sum(2.0 * M * N * K for K, N in d.shapes)
        rows[f"w4a16_gemv_M{M}"] = {"value": round(d.bytes_per_step / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                                    "us_per_step": round(ms * 1e3, 2),
                                    "frac_hbm": round(d.bytes_per_step / (ms * 1e-3) / 1e9 / pk["hbm"], 4),
                                    "fp32_fma_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                                    "frac_fp32_fma_peak": round(flops / (ms * 1e-3) / 1e12 / fp32_peak, 4)}
        del d

    # the same decode sweep through the tensor-core W4A16 (w4a16_gemm_tc): one expansion per
    # weight for all M activation rows; bound by HBM like the M = 1 GEMV
    for M in ((1, 4, 16) if "gemv" in want else ()):
        d = Decode(M, args.seed, dev, tc=True)
        d.capture(6 * d.R, 3)
        d.g_warm.replay()
        ms = float(np.median([time_region(lambda i: d.g_steps.replay(), 1) for _ in range(5)])) / (6 * d.R)
        gbps = d.bytes_per_step / (ms * 1e-3) / 1e9
        shapes_us = {}
        for si, (K, N) in enumerate(d.shapes):
            n_l = 8 * d.R
            gs = d.shape_graph(si, n_l)
            gs.replay()
            t_ms = float(np.median([time_region(lambda i: gs.replay(), 1) for _ in range(5)])) / n_l
            shapes_us[f"K{K}xN{N}"] = round(t_ms * 1e3, 3)
            del gs
        dom_us = shapes_us["K14336xN4096"]
        rows[f"w4a16_tc_M{M}"] = {
            "value": round(gbps, 1), "unit": "GB/s", "us_per_step": round(ms * 1e3, 2), "per_shape_us": shapes_us,
            "roofline": {"bound": "hbm", "achieved": round(gbps, 1), "peak": pk["hbm"], "unit": "GB/s",
                         "frac": round(gbps / pk["hbm"], 4),
                         "launch_K14336xN4096": {
                             "achieved": round(gemv_bytes(M, 4096, 14336) / (dom_us * 1e-6) / 1e9, 1),
                             "traffic": traffic_for(f"w4a16_tc M{M} K14336xN4096",
                                                    "bit_gemm_wise_b200/csrc/w4a16_tc.cu")}},
            "note": "w4a16_gemm_tc (tcgen05, W4_LAYOUT_TC), same four decode shapes and bytes as w4a16_gemv_M*"}
        del d

    # NF4 comparator at M = 1 over the same decode shapes: normal-quantile levels, blocks of 64
    # with an fp32 absmax, a table lookup per code byte (the format the pages compare with)
    if "gemv" in want:
        nf = []
        per_copy = sum(N * K // 2 + N * (K // 64) * 4 for K, N in DECODE_SHAPES)
        R = max(2, -(-3 * L2_BYTES // per_copy))  # weight copies: more than 3x L2 in all
        for K, N in DECODE_SHAPES:
            W = synth.decode_weight(K, N, args.seed, device=dev)
            codes = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
            am = torch.empty(N, K // 64, dtype=torch.float32, device=dev)
            w4.w4_nf4_quantize(W, N, K, codes, am)
            nf.append((K, N, [codes] + [codes.clone() for _ in range(R - 1)], [am] + [am.clone() for _ in range(R - 1)],
                       synth.decode_activation(1, K, args.seed, device=dev), torch.empty(1, N, dtype=torch.bfloat16, device=dev)))
            del W
        nbytes = sum(N * K // 2 + N * (K // 64) * 4 + 2 * K + 2 * N for K, N, *_ in nf)

        def nf_step(i):
            for K, N, cs, ams, x, y in nf:
                w4.w4_nf4_gemv(x, 1, cs[i % R], ams[i % R], N, K, y, w4.W4_OVERLAP_PREVIOUS)

        nf_step(0)
        side = torch.cuda.Stream()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=side):
            for i in range(4 * R):
                nf_step(i)
        gr.replay()
        ms = float(np.median([time_region(lambda i: gr.replay(), 1) for _ in range(9)])) / (4 * R)
        rows["nf4_gemv_M1"] = {"value": round(nbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                               "us_per_step": round(ms * 1e3, 2), "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm"], 4),
                               "note": "NF4 comparator (normal-quantile levels, blocks of 64, fp32 absmax), same four "
                                       "decode shapes, one graph of launches"}
        del nf, gr

    # single linear layer (K=576, N=1536, group 32 symmetric, M=1): launch-latency-dominated,
    # reported in microseconds
    if "gemv" in want:
        c = synth.SINGLE_LAYER
        N, K, g = c["N"], c["K"], c["group"]
        W, x = synth.single_layer(args.seed, device=dev)
        codes, scales, _, _ = w4.alloc_quantized(N, K, g, "sym", device=dev, chosen=False)
        w4.w4_quantize(W, N, K, g, "sym", [1.0], codes, scales, None, None)
        packed = w4.alloc_packed(N, K, g, w4.W4_LAYOUT_GEMV, device=dev)
        w4.w4_prepack(codes, scales, None, N, K, g, "sym", w4.W4_LAYOUT_GEMV, packed)
        y = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
        ws = w4.alloc_gemv_workspace(N, K, g, device=dev)

        def one(i):
            w4.w4a16_gemv(x, 1, packed, N, K, g, "sym", y, 0, ws)

        one(0)
        gr = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        with torch.cuda.graph(gr, stream=side):
            for _ in range(20):
                one(0)
        gr.replay()
        us = time_region(lambda i: gr.replay(), 10) / 200 * 1e3
        rows["w4a16_gemv_single_layer"] = {"value": round(us, 2), "unit": "us per call",
                                           "GBps": round(gemv_bytes(1, N, K, g) / (us * 1e-6) / 1e9, 1),
                                           "note": "0.5 MB problem: launch and latency bound, not a roofline row"}
        del W, x, codes, scales, packed, y, ws

    # context for the FP8 rows: cuBLAS FP8 GEMM (torch._scaled_mm, e4m3, 8192^3, best of 10)
    fp8_cublas = None
    if "prefill" in want or "moe" in want:
        fp8_cublas = measure_fp8_cublas(dev)
        rows["fp8_dense_cublas_8192"] = {"value": round(fp8_cublas, 1), "unit": "TFLOP/s",
                                         "note": "context: torch._scaled_mm e4m3 8192^3, best of 10"}

    # W4A8 prefill GEMM (M=4096) and the FP8 row quant feeding it
    for K, N in (synth.PREFILL_SHAPES if "prefill" in want else ()):
        M = synth.PREFILL_M
        W = synth.prefill_weight(K, N, args.seed, device=dev)
        codes, scales, zeros, _ = w4.alloc_quantized(N, K, 128, "asym", device=dev, chosen=False)
        w4.w4_quantize(W, N, K, 128, "asym", [1.0], codes, scales, zeros, None)
        packed = w4.alloc_packed(N, K, 128, w4.W4_LAYOUT_GEMM, device=dev)
        w4.w4_prepack(codes, scales, zeros, N, K, 128, "asym", w4.W4_LAYOUT_GEMM, packed)
        X = synth.prefill_activation(M, K, args.seed, device=dev)
        X8, sa, _, gop = w4.alloc_row_quant(M, K, 128, device=dev, group_sums=False)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        ws = w4.alloc_gemm_workspace(M, N, K, 128, device=dev)
        sched = w4.w4a8_gemm_schedule(M, N, K, 128, torch.cuda.get_device_properties(dev).multi_processor_count)

        def rq(i):
            w4.fp8_row_quant(X, M, K, 128, X8, sa, None, gop)

        def gemm(i):
            w4.w4a8_gemm(X8, sa, gop, M, packed, N, K, 128, "asym", Y, 0, ws)

        # the same row quant and GEMM in one launch from the bf16 activations (the memset that
        # clears its row flags is inside the timed interval)
        fws = w4.alloc_gemm_rowquant_workspace(M, N, K, 128, device=dev)

        def fused(i):
            w4.w4a8_gemm_rowquant(X, M, packed, N, K, 128, "asym", Y, 0, fws)

        rq(0); gemm(0); fused(0)
        n = 10
        t_rq = t_gemm = t_fused = 0.0
        for i in range(n):
            t_rq += time_region(rq, 1, lead=lambda: flush_l2(flush))
            t_gemm += time_region(gemm, 1, lead=lambda: flush_l2(flush))
            t_fused += time_region(fused, 1, lead=lambda: flush_l2(flush))
        t_rq /= n
        t_gemm /= n
        t_fused /= n
        flops = 2.0 * M * N * K
        tf = flops / (t_gemm * 1e-3) / 1e12
        rq_bytes = M * K * 2 + M * K + M * 4 + gop.numel() * 2
        # algorithmic bytes of one launch: the prepacked weight (codes, scales, zero-point
        # operand), E4M3 activations, row scales, group-sum operand, bf16 output
        alg_bytes = packed.numel() + X8.numel() + sa.numel() * 4 + gop.numel() * 2 + Y.numel() * 2
        rows[f"w4a8_gemm_{K}x{N}"] = {
            "value": round(tf, 1), "unit": "TFLOP/s", "us": round(t_gemm * 1e3, 1),
            "tiles": sched["tiles"], "split_tiles": sched["split_tiles"],
            "bytes_per_launch": alg_bytes,
            "traffic": traffic_for(f"w4a8_gemm M{M} K{K}xN{N}", "bit_gemm_wise_b200/csrc/w4a8_gemm.cu"),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(tf / fp8_peak, 4),
                         "peak_source": f"{pk['src']} bf16 burst x 2 (dense FP8/BF16 nominal ratio)",
                         "frac_of_cublas_fp8": round(tf / fp8_cublas, 4) if fp8_cublas else None,
                         "frac_of_spec_4500": round(tf / 4500.0, 4)}}
        rows[f"fp8_row_quant_{M}x{K}"] = {
            "value": round(rq_bytes / (t_rq * 1e-3) / 1e9, 1), "unit": "GB/s", "us": round(t_rq * 1e3, 1),
            "frac_hbm": round(rq_bytes / (t_rq * 1e-3) / 1e9 / pk["hbm"], 4)}
        rows[f"w4a8_rowquant_plus_gemm_{K}x{N}"] = {
            "value": round(flops / ((t_gemm + t_rq) * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "us": round((t_gemm + t_rq) * 1e3, 1)}
        tff = flops / (t_fused * 1e-3) / 1e12
        rows[f"w4a8_gemm_rowquant_{K}x{N}"] = {
            "value": round(tff, 1), "unit": "TFLOP/s", "us": round(t_fused * 1e3, 1),
            "note": "row quant + GEMM in one launch (w4a8_gemm_rowquant) from bf16 activations",
            "time_vs_gemm_alone": round(t_fused / t_gemm, 4),
            "time_vs_two_launches": round(t_fused / (t_gemm + t_rq), 4),
            "roofline": {"bound": "tensor", "achieved": round(tff, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(tff / fp8_peak, 4)}}
        del W, codes, scales, zeros, packed, X, X8, sa, gop, Y, flush, ws, fws
        torch.cuda.empty_cache()

    # MoE grouped GEMM (32 experts, top-4 of 4096 tokens, group 32)
    if "moe" in want:
        moe_rows(args, dev, fp8_peak, rows)
    if "quantize" in want:
        rows["w4_quantize_8b_set"] = quantizer_full_set(args, dev)
    return rows


def measure_fp8_cublas(dev, n=8192, reps=10):
    """Dense FP8 GEMM throughput of cuBLAS on this GPU (context for the FP8 rows)."""
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    one = torch.tensor(1.0, device=dev)

    def mm(i):
        torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    mm(0)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    best = min(time_region(mm, 1, lead=lambda: flush_l2(flush)) for _ in range(reps))
    del a, b, flush
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def moe_rows(args, dev, fp8_peak, rows):
    """The 32-expert, top-4 layer of 4096 tokens (2880 -> 5760 -> 2880, group 32): each
    grouped GEMM alone, and the whole layer -- route, gathered row quant, gate_up GEMM, SwiGLU
    with the row quant of its result, down GEMM, weighted combine -- as one stream of
    launches (L2 flushed before each timed region)."""
    from bit_gemm_wise_b200 import synth, w4
    c = synth.MOE
    E, k, T, K, H, g = c["E"], c["top_k"], c["tokens"], c["K"], c["N_down"], c["group"]
    gl = torch.Generator().manual_seed(args.seed * 1000 + 60)
    logits = torch.rand(T, E, generator=gl).to(dev)
    X = synth.moe_activation(args.seed, device=dev)
    R = T * k
    ex = torch.empty(T, k, dtype=torch.int32, device=dev)
    gt = torch.empty(T, k, dtype=torch.float32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    tor = torch.empty(R, dtype=torch.int32, device=dev)
    row_of = torch.empty(T, k, dtype=torch.int32, device=dev)
    route_ws = w4.alloc_moe_route_workspace(T, E, device=dev)
    # group 32: the grouped GEMMs take the fp16 copy of the E4M3 activations (exact), which
    # the two row quants write instead of the codes
    X16 = torch.empty(R, K, dtype=torch.float16, device=dev)
    sa = torch.empty(R, dtype=torch.float32, device=dev)
    Ygu = torch.empty(R, 2 * H, dtype=torch.bfloat16, device=dev)
    H16 = torch.empty(R, H, dtype=torch.float16, device=dev)
    sh = torch.empty(R, dtype=torch.float32, device=dev)
    Yd = torch.empty(R, K, dtype=torch.bfloat16, device=dev)
    y = torch.empty(T, K, dtype=torch.bfloat16, device=dev)
    packs = {}
    for kind, N, Kk in (("gate_up", 2 * H, K), ("down", K, H)):
        nb = w4.w4_prepack_bytes(N, Kk, g, w4.W4_LAYOUT_GEMM)
        packed = torch.empty(E * nb, dtype=torch.uint8, device=dev)
        for e in range(E):
            W = synth.moe_weight(kind, e, args.seed, device=dev)
            codes, scales, zeros, _ = w4.alloc_quantized(N, Kk, g, "asym", device=dev, chosen=False)
            w4.w4_quantize(W, N, Kk, g, "asym", [1.0], codes, scales, zeros, None)
            w4.w4_prepack(codes, scales, zeros, N, Kk, g, "asym", w4.W4_LAYOUT_GEMM, packed[e * nb:])
        packs[kind] = packed

    def route(i):
        w4.w4_moe_route(logits, T, E, k, ex, gt, off, tor, row_of, route_ws)

    def dispatch(i):
        w4.fp8_row_quant_gather(X, T, K, g, tor, R, None, sa, x16=X16)

    def gate_up(i):
        w4.w4a8_grouped_gemm(None, sa, None, off, E, R, packs["gate_up"], 2 * H, K, g, "asym", Ygu, X16=X16)

    def swiglu(i):
        w4.w4_moe_swiglu_quant(Ygu, R, H, g, None, sh, x16=H16)

    def down(i):
        w4.w4a8_grouped_gemm(None, sh, None, off, E, R, packs["down"], K, H, g, "asym", Yd, X16=H16)

    def combine(i):
        w4.w4_moe_combine(Yd, K, R, row_of, gt, T, k, y)

    steps = [route, dispatch, gate_up, swiglu, down, combine]

    def layer(i):
        for f in steps:
            f(i)

    layer(0)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    per = {}
    for f in steps:
        per[f.__name__] = float(np.median([time_region(f, 1, lead=lambda: flush_l2(flush)) for _ in range(5)]))
    ms = float(np.median([time_region(layer, 1, lead=lambda: flush_l2(flush)) for _ in range(5)]))
    fl = {"gate_up": 2.0 * R * 2 * H * K, "down": 2.0 * R * K * H}
    for kind in ("gate_up", "down"):
        tf = fl[kind] / (per[kind] * 1e-3) / 1e12
        rows[f"w4a8_grouped_{kind}"] = {
            "value": round(tf, 1), "unit": "TFLOP/s", "us": round(per[kind] * 1e3, 1),
            "path": "group 32: exact fp16 split of the dequantized weight, fp16 tensor cores",
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(tf / fp8_peak, 4),
                         "frac_of_fp16_split_cap": round(tf / (fp8_peak / 4.0), 4)}}
    rows["moe_layer_32x_top4"] = {
        "value": round((fl["gate_up"] + fl["down"]) / (ms * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
        "us": round(ms * 1e3, 1), "us_per_step": {kk: round(v * 1e3, 1) for kk, v in per.items()},
        "note": "route, gathered row quant, gate_up GEMM, SwiGLU + row quant, down GEMM, combine; 4096 tokens"}
    del packs, flush
    torch.cuda.empty_cache()


def quantizer_full_set(args, dev):
    from bit_gemm_wise_b200 import synth, w4
    grid = synth.clip_grid_20()
    layer = synth.LLAMA8B_LAYER
    n_layers = args.quant_layers
    mats = []
    for L in range(n_layers):
        for name, N, K in layer:
            W = synth.llama8b_weight(L, name, args.seed, device=dev)
            out = w4.alloc_quantized(N, K, 128, "asym", device=dev, chosen=False)
            mats.append((W, N, K, out))
    weights = sum(N * K for _, N, K, _ in mats)

    def q(i):
        for W, N, K, (codes, scales, zeros, _) in mats:
            w4.w4_quantize(W, N, K, 128, "asym", grid, codes, scales, zeros, None)

    q(0)
    with Clocks(torch.cuda.current_device()) as clk:
        ms = time_region(q, 1)
    ck = clk.summary()
    wps = weights / (ms * 1e-3)
    res = {"value": round(wps / 1e9, 2), "unit": "G weights/s",
           "input_GBps": round(2 * weights / (ms * 1e-3) / 1e9, 1), "ms": round(ms, 2),
           "weights": weights, "layers": n_layers, "bound": "alu", "clocks": ck}
    # issue-rate roofline: warp instructions per weight (ncu) x weights/s against one warp
    # instruction per clock on each of the 148 x 4 sub-partitions at the clock seen
    rec = QUANT_ISSUE.get("w4_quantize g128 asym 20 ratios")
    mhz = ck.get("sm_mhz") or ck.get("sm_max_mhz")
    if rec and rec["sha1"] == source_sha1("bit_gemm_wise_b200/csrc/w4_quantize.cu") and mhz:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        peak = sms * 4 * mhz * 1e6 / 1e12
        ach = rec["inst_per_weight"] * wps / 1e12
        res["roofline"] = {"bound": "alu", "achieved": round(ach, 3), "peak": round(peak, 3),
                           "unit": "T warp-instructions/s", "frac": round(ach / peak, 4),
                           "inst_per_weight": rec["inst_per_weight"]}
    del mats
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ CPU oracle

def oracle_decode_inputs(seed):
    """Synthetic quantized decode weights for timing the oracle GEMV (values do not affect
    its speed): random codes, fp16 scales, zeros in 0..15, and bf16 activations."""
    import oracle  # noqa: F401
    from bit_gemm_wise_b200 import synth
    rng = np.random.default_rng(seed)
    items = []
    for K, N in DECODE_SHAPES:
        codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
        scales = np.full((N, K // 128), 0x2100, np.uint16)
        zeros = rng.integers(0, 16, (N, K // 128)).astype(np.int16)
        x = synth.bf16_bits(synth.decode_activation(1, K, seed))
        items.append((K, N, codes, scales, zeros, x))
    return items


def cpu_baseline(seed, budget_s=12.0):
    import oracle
    items = oracle_decode_inputs(seed)
    oracle.gemv_ref(items[1][5], *items[1][2:5], 128, "asym")  # warm (build, page-in)
    t0 = time.perf_counter()
    nbytes = 0
    steps = 0
    while True:
        for K, N, codes, scales, zeros, x in items:
            oracle.gemv_ref(x, codes, scales, zeros, 128, "asym")
            nbytes += gemv_bytes(1, N, K)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": f"{steps} full decode steps (4 M=1 GEMVs, fp64 scalar C, OpenMP over rows)",
            "seconds": round(dt, 2)}


def run_reference(args):
    import oracle
    items = oracle_decode_inputs(args.seed)
    oracle.gemv_ref(items[1][5], *items[1][2:5], 128, "asym")
    step_bytes = sum(gemv_bytes(1, N, K) for K, N in DECODE_SHAPES)
    # a bounded sample per step: the first shape set that fits ~2 s
    def step():
        for K, N, codes, scales, zeros, x in items:
            oracle.gemv_ref(x, codes, scales, zeros, 128, "asym")
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    val = step_bytes * args.steps / dt / 1e9
    cores = os.cpu_count()
    return {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "decode GEMV sweep, M=1 (CPU oracle)"},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": "full decode steps (4 M=1 GEMVs), fp64 scalar C, OpenMP over rows"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--rows", default="", help="comma-separated subset of " + ",".join(ROW_GROUPS))
    ap.add_argument("--rows-only", action="store_true", help="skip the headline; measure --rows only")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--quant-layers", type=int, default=32)
    ap.add_argument("--min-repeats", type=int, default=25, help="repeats of the timed region (median reported)")
    ap.add_argument("--min-seconds", type=float, default=0.3, help="keep repeating the timed region this long")
    ap.add_argument("--profile-chain", default="", metavar="K,N",
                    help="only run --launches chained M=1 GEMVs of decode shape (K, N), each naming the next "
                         "weight copy (a short, bounded run for a profiler); prints one line")
    ap.add_argument("--profile-tc", default="", metavar="K,N",
                    help="only run --launches w4a16_gemm_tc calls of decode shape (K, N) at M = --tc-m "
                         "(rotating weight copies, chained like the decode step)")
    ap.add_argument("--tc-m", type=int, default=4)
    ap.add_argument("--launches", type=int, default=8)
    ap.add_argument("--no-prefetch", action="store_true",
                    help="with --profile-chain: plain w4a16_gemv calls (the kernel's own DRAM traffic)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        from bit_gemm_wise_b200 import w4
        w4.lib()
        if args.profile_tc:
            K, N = (int(v) for v in args.profile_tc.split(","))
            dec = Decode(args.tc_m, args.seed, dev, tc=True)
            si = dec.shapes.index((K, N))
            for i in range(args.launches):
                dec.gemv(si, i)
            torch.cuda.synchronize()
            from bit_gemm_wise_b200 import w4 as w4_
            assert w4_.w4_device_status() == 0
            out = {"profile_tc": f"K{K}xN{N}", "M": args.tc_m, "launches": args.launches,
                   "bytes_per_launch": gemv_bytes(args.tc_m, N, K)}
        elif args.profile_chain:
            K, N = (int(v) for v in args.profile_chain.split(","))
            dec = Decode(1, args.seed, dev)
            si = dec.shapes.index((K, N))
            for i in range(args.launches):
                dec.gemv(si, i, next_si=si, prefetch=not args.no_prefetch)
            torch.cuda.synchronize()
            from bit_gemm_wise_b200 import w4 as w4_
            assert w4_.w4_device_status() == 0
            out = {"profile_chain": f"K{K}xN{N}", "launches": args.launches, "prefetch": not args.no_prefetch,
                   "bytes_per_launch": gemv_bytes(1, N, K)}
        elif args.rows_only:
            out = {"rows": measure_rows(args, dev, peaks())}
        else:
            out = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
