#!/usr/bin/env python
"""Benchmark of the Spense hybrid 2:4-sparse + dense FP8 GEMM on B200.

Workload (default): the attention projections of a 32B-class decoder (hidden
5120): q_proj 8192x5120, k_proj and v_proj 1024x5120, o_proj 5120x8192, FP8
e4m3 weights with the last 25% of the input columns dense, M = 16 decode
tokens. One step = the four GEMMs of one layer. Eight layers' packed weights
(542 MB, more than the 126 MB L2) are rotated so every step streams its
weights from HBM. Inputs are seeded synthetic tensors (no model weights).

Metric: weight-stream GB/s = algorithmic bytes (packed values + 2-bit
metadata + dense columns + scales + activations + bf16 output) / time; also
the speedup over the same kernel on the dense FP8 matrix (dense_frac = 1).

Prints one JSON line (rank 0). Multi-GPU runs are independent replicas (the
GEMM has no exchange step), launched one process per GPU.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["spense", "reference"], default="spense")
    ap.add_argument("--tokens", type=int, default=16, help="decode tokens M")
    ap.add_argument("--layers", type=int, default=8, help="weight sets rotated between steps")
    ap.add_argument("--dense-frac", type=float, default=0.25)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["gemm", "quantize", "score", "glu"], default="gemm",
                    help="gemm: the hybrid GEMM (default, the headline); quantize: the per-token FP8 "
                         "quantisation with the SpenseGPT+ column order fused in; score: the SpenseGPT+ "
                         "dense-set scorer and top-Kd selection; glu: a 32B-class GLU MLP's three projections "
                         "under the pages' GLU policy (gate/up output-split, down input-split, permutation folded)")
    return ap.parse_args()


SHAPES = (("q_proj", 8192, 5120), ("k_proj", 1024, 5120), ("v_proj", 1024, 5120), ("o_proj", 5120, 8192))
# One step = one layer's attention projections: q, k and v read the same hidden
# state and run as one grouped launch; o_proj reads the attention output.
GROUPS = ((0, 1, 2), (3,))


L2_BYTES = 126 << 20


def l2_note(sets, total):
    rel = "larger" if total > L2_BYTES else "NOT larger"
    return f"{sets} weight sets rotated per step ({total / 1e6:.0f} MB, {rel} than the 126 MB L2)"


def workload_config(args):
    return {
        "workload": f"attn32b q/k/v/o projections, decode M={args.tokens}",
        "shapes": [f"{n}x{k}" for _, n, k in SHAPES],
        "launches_per_step": "q+k+v grouped (shared input), o_proj",
        "tokens": args.tokens,
        "dense_frac": args.dense_frac,
        "dense_columns": "tail (SpenseGPT)",
        "weights": "FP8 e4m3 N(0,0.02) per-channel absmax scales; X N(0,1) per-token scales; seed 1",
        "l2": l2_note(args.layers, args.layers * step_bytes(args)),
        "graph": f"one CUDA graph per {args.layers} steps (the rotated layers back to back)",
    }


def step_bytes(args, dense=False):
    from dense_fp8_gemm_b200 import workloads
    total = 0
    for grp in GROUPS:
        mem = [(SHAPES[i][1], SHAPES[i][2],
                SHAPES[i][2] if dense else workloads.dense_count(SHAPES[i][2], args.dense_frac)) for i in grp]
        total += workloads.group_algorithmic_bytes(mem, args.tokens)
    return total


KERNEL_SOURCES = ("gemm_sm100.cu", "sm100_ptx.cuh", "spense_internal.h")


def kernel_source_sha256():
    """sha256 over the sources that define spense_gemm_kernel, in a fixed order."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "dense_fp8_gemm_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def read_traffic():
    """DRAM bytes per launch of spense_gemm_kernel from the committed ncu summary,
    or None when the kernel sources have changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "spense_gemm_attn32b_m16_traffic.txt")
    try:
        with open(path) as f:
            rec = json.load(f)
        return rec["dram_bytes_per_launch_avg"] if rec["kernel_source_sha256"] == kernel_source_sha256() else None
    except Exception:
        return None


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs.

    Sampling starts before the warm-up; `mark(t0, t1)` records the wall-clock
    window of the timed region and only samples inside it are summarized (all
    samples if the window caught none, which `in_window` reports)."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 50):
        self.gpu = gpu_index
        self.interval = interval_ms
        self.proc = None
        self.window = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)  # let the first samples arrive before the work starts
        except Exception:
            self.proc = None
        return self

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(2 * self.interval / 1000)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        import datetime
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        samples = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                samples.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        inside = samples
        in_window = False
        if self.window is not None:
            w = [x for x in samples if self.window[0] - 0.06 <= x[0] <= self.window[1] + 0.06]
            if w:
                inside, in_window = w, True
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "in_window": False}
        reasons = sorted({n for x in inside for n, v in zip(names, x[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max(x[2] for x in inside),
                "reasons": reasons, "samples": len(inside), "in_window": in_window}


# ----------------------------------------------------------------------------- CPU oracle timing


def oracle_items(args, rows_per_shape: int):
    """The bounded sample the CPU oracle runs: `rows_per_shape` output rows of
    each projection, with the step's activations (q/k/v share one input)."""
    import oracle
    from dense_fp8_gemm_b200 import workloads
    wl = workloads.ATTN32B
    acts = {0: workloads.make_activations(wl, 0, args.tokens), 3: workloads.make_activations(wl, 3, args.tokens)}
    items, members = [], []
    for grp in GROUPS:
        X, s_x = acts[grp[0]]
        mem = []
        for i in grp:
            w = workloads.make_weight(wl, i, args.dense_frac)
            rows = np.linspace(0, w.N - 1, rows_per_shape).astype(np.int64)
            keep = oracle.pack(w.W[rows], Kd=w.Kd)["keep"]
            items.append((X, s_x, w.W[rows].copy(), w.s_w[rows].copy(), keep))
            mem.append((rows_per_shape, w.K, w.Kd))
        members.append(mem)
    byts = sum(workloads.group_algorithmic_bytes(m, args.tokens) for m in members)
    return items, byts


def oracle_pass(items, nthreads):
    import oracle
    for X, s_x, W, s_w, keep in items:
        oracle.gemm(X, s_x, W, s_w, keep=keep, nthreads=nthreads)


def oracle_sample_rate(args, rows_per_shape: int, budget_s: float, nthreads: int):
    """Times the CPU oracle (as it stands) on the bounded sample, repeating until
    `budget_s` elapses. Returns (GB/s, seconds, passes)."""
    items, byts = oracle_items(args, rows_per_shape)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_pass(items, nthreads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return byts * reps / el / 1e9, el, reps


# ----------------------------------------------------------------------------- reference arm


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = os.cpu_count() or 1
    rows = 32  # bounded sample per step: 32 output rows of each projection
    items, per_step = oracle_items(args, rows)
    for _ in range(args.warmup):
        oracle_pass(items, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(items, cores)
    el = time.perf_counter() - t0
    value = per_step * args.steps / el / 1e9
    sample = f"{rows} output rows of each of q/k/v/o per step (M={args.tokens}), all {cores} host threads"
    line = {
        "impl": "reference", "metric": "spense_fp8_weight_stream_GBps", "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / max(1, args.steps) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(args),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- Spense arm


def run_spense(args):
    import torch

    from dense_fp8_gemm_b200 import replicas, spense, workloads

    ranks = replicas.from_env()
    world, rank, local = ranks.world, ranks.rank, ranks.local
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init(ranks, "nccl", device=dev)

    M = args.tokens
    wl = workloads.ATTN32B
    # ---- weights: one synthetic layer, packed into `layers` distinct buffer sets
    host_w = [workloads.make_weight(wl, i, args.dense_frac) for i in range(len(SHAPES))]
    layers_sp, layers_dn = [], []
    for _ in range(args.layers):
        sp, dn = [], []
        for w in host_w:
            Wd = torch.from_numpy(w.W).to(dev)
            sd = torch.from_numpy(w.s_w).to(dev)
            sp.append(spense.pack(Wd, sd, Kd=w.Kd))
            dn.append(spense.pack(Wd, sd, Kd=w.K))
            del Wd
        layers_sp.append(sp)
        layers_dn.append(dn)
    # activations: q/k/v share the hidden state, o_proj reads the attention output
    host_x = {grp[0]: workloads.make_activations(wl, grp[0], M) for grp in GROUPS}
    dev_x = {k: (torch.from_numpy(v[0]).to(dev), torch.from_numpy(v[1]).to(dev)) for k, v in host_x.items()}
    Ys = [torch.empty((M, n), dtype=torch.bfloat16, device=dev) for _, n, _ in SHAPES]
    ws_bytes = max(spense.grouped_workspace_size([L[i] for i in grp], M)
                   for L in (layers_sp[0], layers_dn[0]) for grp in GROUPS)
    ws = spense.new_workspace(ws_bytes, dev)
    torch.cuda.synchronize()

    def launch_layer(packs, stream, events=None):
        for gi, grp in enumerate(GROUPS):
            X, sx = dev_x[grp[0]]
            if events is not None:
                events[gi][0].record(stream)
            spense.gemm_grouped([packs[i] for i in grp], X, sx, [Ys[i] for i in grp], ws, stream)
            if events is not None:
                events[gi][1].record(stream)

    def capture_chain(layer_list):
        """One graph over all layers in sequence (a decode step of the whole stack)."""
        for L in layer_list:
            launch_layer(L, torch.cuda.current_stream())
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for L in layer_list:
                launch_layer(L, torch.cuda.current_stream())
        torch.cuda.synchronize()
        return g

    def capture(layer_list, with_events=False):
        graphs, evs = [], []
        for L in layer_list:
            launch_layer(L, torch.cuda.current_stream())  # warm (attribute setup outside capture)
        torch.cuda.synchronize()
        for L in layer_list:
            g = torch.cuda.CUDAGraph()
            e = [(torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True)) for _ in GROUPS] if with_events else None
            with torch.cuda.graph(g):
                launch_layer(L, torch.cuda.current_stream(), e)
            graphs.append(g)
            evs.append(e)
        torch.cuda.synchronize()
        return graphs, evs

    def timed(graphs, chain, steps, warmup, clocks=None):
        # Steps run as whole-stack graphs (all rotated layers back to back, so
        # each launch overlaps the previous one's tail); a remainder of fewer
        # than `layers` steps uses the per-layer graphs.
        def run(n):
            for _ in range(n // len(graphs)):
                chain.replay()
            for i in range(n % len(graphs)):
                graphs[i].replay()
        run(warmup)
        torch.cuda.synchronize()
        replicas.barrier(ranks)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        w0 = time.time()
        e0.record()
        run(steps)
        e1.record()
        torch.cuda.synchronize()
        if clocks is not None:
            clocks.mark(w0, time.time())
        replicas.barrier(ranks)
        return e0.elapsed_time(e1) / 1e3  # seconds

    g_sp, _ = capture(layers_sp)
    g_dn, _ = capture(layers_dn)
    c_sp = capture_chain(layers_sp)
    c_dn = capture_chain(layers_dn)

    with ClockSampler(local) as clocks:
        t_sp = timed(g_sp, c_sp, args.steps, args.warmup, clocks)
    t_dn = timed(g_dn, c_dn, args.steps, args.warmup)

    t_sp, t_dn = replicas.max_over_ranks(ranks, [t_sp, t_dn], device=dev)

    per_step = step_bytes(args)
    value = replicas.job_rate(per_step * args.steps, world, t_sp) / 1e9
    launches = args.steps * len(GROUPS)

    # ---- dominant kernel: per-launch device time from events captured around each launch
    g_ev, evs = capture(layers_sp, with_events=True)
    dur = [[] for _ in GROUPS]
    reps = max(8, min(args.steps, 64))
    for i in range(reps):
        g_ev[i % len(g_ev)].replay()
        torch.cuda.synchronize()
        for gi, (a, b) in enumerate(evs[i % len(g_ev)]):
            dur[gi].append(a.elapsed_time(b) / 1e3)
    per_launch = [statistics.median(d) for d in dur]  # isolated: event nodes serialize the launches
    # The timed region holds only spense_gemm_kernel launches (tail dense set: no gather), so the
    # average launch duration over it is t_sp / launches and the bytes per launch average the
    # step's algorithmic bytes over its launches.
    avg_launch_s = t_sp / launches
    bytes_per_launch = per_step / len(GROUPS)
    achieved = bytes_per_launch / avg_launch_s / 1e9
    peak, peak_kind = read_peaks()
    del g_ev, evs

    # ---- e2e: host buffers in, host buffers out, copies inside the timed region.
    # Each group's X and x_scale sit in one pinned host buffer and one device
    # buffer (one host-to-device copy per group); all outputs of a step sit in
    # one device buffer (one device-to-host copy per step); the GEMM calls are
    # prepared once per layer (their arguments marshalled once).
    import torch as _t
    in_host, in_dev, in_views = {}, {}, {}
    for k, (xh, sxh) in host_x.items():
        nx = xh.size
        buf_h = _t.empty(nx + 4 * M, dtype=_t.uint8).pin_memory()
        buf_h[:nx] = _t.from_numpy(xh.reshape(-1))
        buf_h[nx:] = _t.from_numpy(sxh.view(np.uint8))
        buf_d = _t.empty_like(buf_h, device=dev)
        in_host[k], in_dev[k] = buf_h, buf_d
        in_views[k] = (buf_d[:nx].view(M, -1), buf_d[nx:].view(_t.float32))
    offs = np.cumsum([0] + [M * n for _, n, _ in SHAPES])
    out_dev = _t.empty(int(offs[-1]), dtype=_t.bfloat16, device=dev)
    out_host = _t.empty(int(offs[-1]), dtype=_t.bfloat16).pin_memory()
    y_views = [out_dev[int(offs[i]):int(offs[i + 1])].view(M, SHAPES[i][1]) for i in range(len(SHAPES))]
    calls = [[spense.PreparedGrouped([layer[i] for i in grp], in_views[grp[0]][0], in_views[grp[0]][1],
                                     [y_views[i] for i in grp], ws) for grp in GROUPS] for layer in layers_sp]
    stream = torch.cuda.current_stream()

    def e2e_step(layer_calls):
        for grp, call in zip(GROUPS, layer_calls):
            in_dev[grp[0]].copy_(in_host[grp[0]], non_blocking=True)
            call(stream)
        out_host.copy_(out_dev, non_blocking=True)
        stream.synchronize()

    e2e_steps = max(4, min(args.steps, 200))
    for i in range(min(args.warmup, 8)):
        e2e_step(calls[i % args.layers])
    replicas.barrier(ranks)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        e2e_step(calls[i % args.layers])
    e1.record()
    torch.cuda.synchronize()
    t_e2e = replicas.max_over_ranks(ranks, [e0.elapsed_time(e1) / 1e3], device=dev)[0]
    h2d = sum(M * SHAPES[g[0]][2] + 4 * M for g in GROUPS)
    d2h = sum(2 * M * n for _, n, _ in SHAPES)
    e2e_value = replicas.job_rate(per_step * e2e_steps, world, t_e2e) / 1e9

    status = spense.workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word {status:#x}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        gbs, el, reps_c = oracle_sample_rate(args, 256, args.cpu_seconds, cores)
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"256 output rows of each of q/k/v/o, M={args.tokens}, {reps_c} passes in {el:.1f} s"}

    if rank == 0:
        kd = [workloads.dense_count(k, args.dense_frac) for _, _, k in SHAPES]
        tflops = sum(workloads.useful_flops(n, k, kd[i], M) for i, (_, n, k) in enumerate(SHAPES)) \
            * args.steps * world / t_sp / 1e12
        line = {
            "metric": "spense_fp8_weight_stream_GBps", "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_sp / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3xe4m3->f32",
            "data": "synthetic", "config": workload_config(args),
            "speedup_vs_dense_fp8": t_dn / t_sp,
            "dense_fp8_GBps": step_bytes(args, dense=True) * args.steps * world / t_dn / 1e9,
            "tflops": tflops,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": read_traffic(), "peak_source": peak_kind,
                         "kernel": "spense_gemm_kernel", "avg_launch_us": avg_launch_s * 1e6,
                         "bytes_per_launch": bytes_per_launch,
                         "isolated_launch_us": {"qkv_grouped": per_launch[0] * 1e6, "o_proj": per_launch[1] * 1e6}},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)

    for L in layers_sp + layers_dn:
        for p in L:
            p.free()
    del g_sp, g_dn, c_sp, c_dn  # graphs are released before the process group goes away
    replicas.finalize(ranks)
    return 0


def graph_time(launch, copies, steps, warmup):
    """Seconds per launch: `copies` launches (rotating inputs) captured in one
    CUDA graph, replayed until `steps` launches ran, timed with CUDA events on
    the capturing stream after `warmup` launches."""
    import torch
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(copies):
            launch(i, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(copies):
            launch(i, stream)
    reps = max(1, -(-steps // copies))
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-warmup // copies))):
            g.replay()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        stream.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / (reps * copies)
    del g
    return t, reps * copies


def run_quantize(args):
    """spense_quantize on the SpenseGPT+ workload's activations (down_proj input,
    K = 25600, dense_frac 0.25 scattered): bf16 [M][K] -> e4m3 + per-token
    scales, with the packed column order fused in; the plain (no gather) variant
    is timed beside it. HBM roofline: 3 bytes per element + 4 per token."""
    import torch
    from dense_fp8_gemm_b200 import spense, synth, workloads
    import oracle
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M, K = args.tokens, 25600
    Kd = workloads.dense_count(K, args.dense_frac)
    W, s_w = synth.quantize_rows(synth.normal(3, 1, (128, K), 0.02))
    dense_idx = synth.scored_dense_idx(3, 2, K, Kd)
    pw = spense.pack(torch.from_numpy(W).to(dev), torch.from_numpy(s_w).to(dev), Kd=Kd, dense_idx=dense_idx)
    xb = synth.normal(3, 3, (M, K), 1.0)
    x_bits = torch.from_numpy(xb).to(torch.bfloat16)
    per = M * K * 2
    copies = max(2, -(-(256 << 20) // per))  # inputs larger than L2 across one graph
    Xs = [x_bits.to(dev) for _ in range(copies)]
    Xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
    sx = torch.empty((M,), dtype=torch.float32, device=dev)
    bytes_per = M * K * 3 + 4 * M
    steps = max(args.steps // 100, copies)
    with ClockSampler(0) as clocks:
        t0w = time.time()
        t_fused, n = graph_time(lambda i, st: spense.quantize(Xs[i], order=pw, Xq=Xq, x_scale=sx, stream=st),
                                copies, steps, args.warmup)
        t_plain, _ = graph_time(lambda i, st: spense.quantize(Xs[i], Xq=Xq, x_scale=sx, stream=st),
                                copies, steps, args.warmup)
        clocks.mark(t0w, time.time())
    peak, peak_kind = read_peaks()
    # end to end: host bf16 in, host e4m3 + scales out, copies and a sync each step
    hx = x_bits.pin_memory()
    hq = torch.empty((M, K), dtype=torch.uint8).pin_memory()
    hs = torch.empty((M,), dtype=torch.float32).pin_memory()
    e2e_steps = 50
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        Xs[0].copy_(hx, non_blocking=True)
        spense.quantize(Xs[0], order=pw, Xq=Xq, x_scale=sx, stream=stream)
        hq.copy_(Xq, non_blocking=True)
        hs.copy_(sx, non_blocking=True)
        stream.synchronize()
    e1.record()
    torch.cuda.synchronize()
    t_e2e = e0.elapsed_time(e1) / 1e3 / e2e_steps
    cpu = None
    if not args.no_cpu_baseline:
        rows = min(M, 4)
        bits = x_bits[:rows].view(torch.int16).numpy().view(np.uint16)
        c0, done = time.time(), 0
        while time.time() - c0 < min(args.cpu_seconds, 5.0) or done == 0:
            oracle.quantize(bits, dense_idx=dense_idx)
            done += 1
        el = time.time() - c0
        cpu = {"value": done * rows * (K * 3 + 4) / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{rows} token rows x {K} columns with the packed order, {done} passes in {el:.1f} s"}
    line = {
        "metric": "spense_quantize_GBps", "value": bytes_per / t_fused / 1e9, "unit": "GB/s", "n_gpus": 1,
        "steps": n, "warmup": args.warmup, "ms_per_step": t_fused * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3", "data": "synthetic",
        "config": {"workload": f"SpenseGPT+ down_proj input, bf16 [{M}x{K}] -> e4m3, dense_frac "
                               f"{args.dense_frac} scattered (fused column order)",
                   "l2": f"{copies} input copies rotated in one graph (larger than L2)"},
        "plain_GBps": bytes_per / t_plain / 1e9,
        "roofline": {"bound": "hbm", "achieved": bytes_per / t_fused / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": bytes_per / t_fused / 1e9 / peak, "traffic": None, "peak_source": peak_kind,
                     "kernel": "quantize_kernel<true>", "bytes_per_launch": bytes_per,
                     "avg_launch_us": t_fused * 1e6},
        "cpu_baseline": cpu,
        "e2e": {"value": bytes_per / t_e2e / 1e9, "unit": "GB/s", "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * K + 4 * M},
        "gpu_launches": n * 2,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    pw.free()
    return 0


def run_score(args):
    """SpenseGPT+ dense-set selection on the 32B-class FFN shapes: scores of the
    I = 25600 intermediate indices from gate, up [I][5120] and down [5120][I]
    (FP8 + row scales, synthetic Hessian diagonals), then the top Kd = 0.25 I.
    One step = score + select. HBM roofline over the algorithmic bytes (the
    three weight matrices, their scales, the Hessian diagonals, the scores)."""
    import torch
    from dense_fp8_gemm_b200 import spense, synth
    import oracle
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    I, H = 25600, 5120
    Kd = int(round(args.dense_frac * I))
    g = np.random.default_rng(2)
    sets = []
    copies = 2  # 2 x 393 MB of weights, larger than L2
    for c in range(copies):
        gq, gs = synth.quantize_rows(synth.normal(2, 10 + c, (I, H), 0.02))
        uq, us = synth.quantize_rows(synth.normal(2, 20 + c, (I, H), 0.02))
        dq, ds = synth.quantize_rows(synth.normal(2, 30 + c, (H, I), 0.02))
        sets.append({k: torch.from_numpy(v).to(dev) for k, v in
                     dict(gate=gq, s_gate=gs, up=uq, s_up=us, down=dq, s_down=ds).items()})
    h_in = torch.from_numpy((g.standard_normal((8, H)).astype(np.float32) ** 2).sum(0)).to(dev)
    h_mid = torch.from_numpy((g.standard_normal((8, I)).astype(np.float32) ** 2).sum(0)).to(dev)
    score = torch.empty((I,), dtype=torch.float32, device=dev)
    idx = torch.empty((Kd,), dtype=torch.int32, device=dev)
    ws = spense.new_workspace(max(256, int(spense.lib().spense_score_workspace_size(I, H))), dev)
    bytes_per = 3 * I * H + 4 * (2 * I + H) + 4 * (H + I) + 4 * I + 4 * Kd

    def launch(i, st):
        w = sets[i]
        spense.score_glu(w["down"], w["s_down"], h_in, h_mid, gate=w["gate"], s_gate=w["s_gate"], up=w["up"],
                         s_up=w["s_up"], score=score, workspace=ws, stream=st)
        spense.select_dense(score, Kd, out=idx, stream=st)

    steps = max(20, min(args.steps // 100, 200))
    with ClockSampler(0) as clocks:
        t0w = time.time()
        t_step, n = graph_time(launch, copies, steps, args.warmup // 20)
        clocks.mark(t0w, time.time())
    peak, peak_kind = read_peaks()
    cpu = None
    if not args.no_cpu_baseline:
        w = {k: v.cpu().numpy() for k, v in sets[0].items()}
        cols = 512  # a bounded sample: the scores of 512 intermediate indices
        sub = dict(gate=w["gate"][:cols], s_gate=w["s_gate"][:cols], up=w["up"][:cols], s_up=w["s_up"][:cols],
                   down=np.ascontiguousarray(w["down"][:, :cols]), s_down=w["s_down"])
        hi, hm = h_in.cpu().numpy(), h_mid.cpu().numpy()[:cols]
        c0, done = time.time(), 0
        while time.time() - c0 < min(args.cpu_seconds, 5.0) or done == 0:
            oracle.score_glu(sub["down"], sub["s_down"], hi, hm, gate=sub["gate"], s_gate=sub["s_gate"],
                             up=sub["up"], s_up=sub["s_up"])
            done += 1
        el = time.time() - c0
        cpu = {"value": done * 3 * cols * H / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"scores of {cols} of {I} intermediate indices (weight bytes only), {done} passes in "
                         f"{el:.1f} s"}
    line = {
        "metric": "spense_score_select_GBps", "value": bytes_per / t_step / 1e9, "unit": "GB/s", "n_gpus": 1,
        "steps": n, "warmup": args.warmup // 20, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3->f32", "data": "synthetic",
        "config": {"workload": f"SpenseGPT+ dense-set selection, 32B FFN: gate/up {I}x{H}, down {H}x{I}, "
                               f"Kd = {Kd}", "l2": f"{copies} weight sets rotated (786 MB, larger than L2)"},
        "roofline": {"bound": "hbm", "achieved": bytes_per / t_step / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": bytes_per / t_step / 1e9 / peak, "traffic": None, "peak_source": peak_kind,
                     "kernel": "score_rows + score_cols + score_finish + select_top", "bytes_per_step": bytes_per},
        "cpu_baseline": cpu,
        "e2e": None,
        "gpu_launches": n * 4,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_glu(args):
    """The GEMMs of one 32B-class GLU MLP at decode (hidden 5120, intermediate
    25600) under the pages' GLU policy: gate and up output-split (their dense
    rows are the SpenseGPT+ dense set, folded to the end of the intermediate
    order), four members in one launch; down input-split with the same dense
    set, reading the already-permuted activations without a gather. One step =
    those two launches (the activation between them is outside this library;
    a fixed quantised input stands in for it). Timed beside it: the all
    input-split layout (gate+up as one K-split matrix, down with a tail set)."""
    import torch
    from dense_fp8_gemm_b200 import spense, synth, workloads
    import oracle
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    H, I, M = 5120, 25600, args.tokens
    Nd = int(round(args.dense_frac * I / 128)) * 128
    Ns = I - Nd
    layers = 2
    D = synth.scored_dense_idx(2, 5, I, Nd)
    pi = oracle.glu_order(I, D)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    sets, base = [], []
    for L in range(layers):
        gq, gs = synth.quantize_rows(synth.normal(2, 40 + L, (I, H), 0.02))
        uq, us = synth.quantize_rows(synth.normal(2, 50 + L, (I, H), 0.02))
        dq, ds = synth.quantize_rows(synth.normal(2, 60 + L, (H, I), 0.02))
        gu = [spense.pack(t(gq), t(gs), Kd=0, rows=pi[:Ns]), spense.pack(t(gq), t(gs), Kd=H, rows=pi[Ns:]),
              spense.pack(t(uq), t(us), Kd=0, rows=pi[:Ns]), spense.pack(t(uq), t(us), Kd=H, rows=pi[Ns:])]
        dn = spense.pack(t(dq), t(ds), Kd=Nd, dense_idx=D)
        sets.append((gu, dn))
        both = np.concatenate([gq, uq])
        both_s = np.concatenate([gs, us])
        base.append((spense.pack(t(both), t(both_s), Kd=workloads.dense_count(H, args.dense_frac)),
                     spense.pack(t(dq), t(ds), Kd=workloads.dense_count(I, args.dense_frac))))
        del gq, uq, dq, both
    x, sx = synth.quantize_rows(synth.normal(2, 70, (M, H), 1.0))
    h, sh = synth.quantize_rows(synth.normal(2, 71, (M, I), 1.0))
    X, SX, Hq, SH = t(x), t(sx), t(h), t(sh)
    G = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    U = torch.empty((M, I), dtype=torch.bfloat16, device=dev)
    GU = torch.empty((M, 2 * I), dtype=torch.bfloat16, device=dev)
    Y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    ws = spense.new_workspace(max(spense.grouped_workspace_size(sets[0][0], M), spense.workspace_size(sets[0][1], M),
                                  spense.workspace_size(base[0][0], M), spense.workspace_size(base[0][1], M)), dev)
    Ys_gu = [G[:, :Ns], G[:, Ns:], U[:, :Ns], U[:, Ns:]]

    def step_policy(i, st):
        gu, dn = sets[i % layers]
        spense.gemm_grouped(gu, X, SX, Ys=Ys_gu, workspace=ws, stream=st)
        spense.gemm_grouped([dn], Hq, SH, Ys=[Y], workspace=ws, stream=st, flags=spense.GEMM_X_PACKED_ORDER)

    def step_base(i, st):
        gu, dn = base[i % layers]
        spense.gemm_grouped([gu], X, SX, Ys=[GU], workspace=ws, stream=st)
        spense.gemm_grouped([dn], Hq, SH, Ys=[Y], workspace=ws, stream=st)

    mem_gu = [(Ns, H, 0), (Nd, H, H), (Ns, H, 0), (Nd, H, H)]
    bytes_policy = workloads.group_algorithmic_bytes(mem_gu, M) + workloads.algorithmic_bytes(H, I, Nd, M)
    kd_h, kd_i = workloads.dense_count(H, args.dense_frac), workloads.dense_count(I, args.dense_frac)
    bytes_base = workloads.algorithmic_bytes(2 * I, H, kd_h, M) + workloads.algorithmic_bytes(H, I, kd_i, M)
    steps = max(40, min(args.steps // 20, 1000))
    with ClockSampler(0) as clocks:
        t0w = time.time()
        t_pol, n = graph_time(step_policy, layers, steps, args.warmup // 10)
        t_base, _ = graph_time(step_base, layers, steps, args.warmup // 10)
        clocks.mark(t0w, time.time())
    assert spense.workspace_status(ws) == 0
    peak, peak_kind = read_peaks()
    line = {
        "metric": "spense_glu_mlp_GBps", "value": bytes_policy / t_pol / 1e9, "unit": "GB/s", "n_gpus": 1,
        "steps": n, "warmup": args.warmup // 10, "ms_per_step": t_pol * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3xe4m3->f32", "data": "synthetic",
        "config": {"workload": f"32B GLU MLP decode M={M}: gate/up {I}x{H} output-split ({Nd} dense rows, "
                               f"SpenseGPT+ set folded to the end), down {H}x{I} input-split with the same set, "
                               f"no gather", "l2": f"{layers} layers rotated (larger than L2)",
                   "launches_per_step": 2},
        "input_split_layout": {"GBps": bytes_base / t_base / 1e9, "ms_per_step": t_base * 1e3,
                               "bytes_per_step": bytes_base},
        "roofline": {"bound": "hbm", "achieved": bytes_policy / t_pol / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": bytes_policy / t_pol / 1e9 / peak, "traffic": None, "peak_source": peak_kind,
                     "kernel": "spense_gemm_kernel", "bytes_per_step": bytes_policy},
        "cpu_baseline": None,
        "e2e": None,
        "gpu_launches": 2 * n,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    for gu, dn in sets:
        for pw in gu + [dn]:
            pw.free()
    for a, b in base:
        a.free()
        b.free()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "quantize":
        return run_quantize(args)
    if args.op == "score":
        return run_score(args)
    if args.op == "glu":
        return run_glu(args)
    return run_spense(args)


if __name__ == "__main__":
    sys.exit(main())
