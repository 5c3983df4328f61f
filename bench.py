"""Benchmark of the gated local-global graph-attention forward on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--forwards-per-step R]
                  [--impl mine|reference] [--workload arxiv] [--no-cpu-baseline]

One step is R forwards of the layer (projection GEMM, global statistics, local branch,
readout with the gate blend) over the arxiv-shaped synthetic graph, with the graph already
bound (glga_create, timed separately as create_ms) and inputs resident in HBM.  Every
forward replays a CUDA graph of glga_forward captured once on the same buffers
(Layer.capture: the same kernels, without host work between them) and is timed with its
own pair of CUDA events on the launching stream; L2 is flushed (256 MiB write) before
every forward, outside the timed spans, so the K steps' timed region lasts seconds and the
clock sampler sees it.  The library's stage events, recorded inside the captured graph,
give the local kernel's launch time over the timed region for the roofline.
Metric: edge*heads/s = E * H / seconds per forward, E counting self-loops.

Multi-GPU (torchrun, one rank per GPU): the row-sharded forward (sharded.ShardedForward:
each rank owns a block of target rows with about equal CSR entries; one NCCL all-gather of
the K/V row blocks and one of the partial statistics per forward; strong scaling), or
with --replicas every rank runs the whole forward on its own copy (weak scaling).  Time is
the maximum over ranks.  `--impl reference` times the float64 CPU oracle on the host
instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GLGA fwd edge·heads/s (1 B200, bf16 arxiv-shaped); local-branch HBM GB/s % of peak"
UNIT = "edge*heads/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_NOTE = "flushed before every timed forward (256 MiB write, outside the timed spans)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks_dist(x, world, device):
    """The largest value of x over all ranks (every rank gets it); x itself at world 1."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world, units_per_rank, slowest_total_ms, steps):
    """Whole-job units per second when every rank runs `steps` steps of `units_per_rank`
    units and the slowest rank took `slowest_total_ms` for them."""
    return world * units_per_rank * steps / (slowest_total_ms * 1e-3)


def local_kernel_bytes(N, E, D, s):
    """Algorithmic bytes of one launch of the local-branch kernel: CSR (row_ptr, col_idx),
    one k_j and v_j row gather per edge, q_i read and L_i written once per row."""
    return 4 * (N + 1) + 4 * E + 2 * D * s * E + D * s * N + D * s * N


def branch_bytes_model(N, E, D, H, r, s):
    """Algorithmic bytes of the local branch with the readout and gate (steps a3-a5 taken
    together, as if fused): CSR, the k_j / v_j gathers, q_i and Y_i once per row, the gate
    logit, and S, z."""
    return (4 * (N + 1) + 4 * E + 2 * D * s * E + D * s * N + D * s * N + 4 * N
            + 4 * H * r * (r + 1))


def branch_compulsory_bytes(N, E, D, H, r, s):
    """Lower bound on the DRAM traffic of steps a3-a5: every Q, K, V row read once, Y
    written once, plus CSR, gate logits and S, z."""
    return 4 * (N + 1) + 4 * E + 3 * D * s * N + D * s * N + 4 * N + 4 * H * r * (r + 1)


def kernel_source_hash():
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "sparse_graph_attention_tcgen05_b200", "csrc", "local.cu"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def profiled_counters(workload):
    """ncu counters of the local kernel from the structured summary
    profiles/local_kernel_<workload>.json, if it was taken on the current kernel source:
    DRAM bytes per launch (scaled to the full workload) and warp instructions per edge."""
    path = os.path.join(ROOT, "profiles", f"local_kernel_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("local_cu_sha256_16") != kernel_source_hash():
        return {"stale": True, "file": os.path.relpath(path, ROOT)}
    d["file"] = os.path.relpath(path, ROOT)
    return d


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1])); smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def cpu_baseline(w, csr, min_seconds=10.0, max_seconds=30.0):
    import oracle
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(w.N, w.d, w.H, w.r, w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps,
                       csr[0], csr[1])
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or el * (reps + 1) / reps > max_seconds:
            break
    return {"value": w.E * w.H * reps / el, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"the full {w.name} workload (N={w.N}, E={w.E}), {reps} float64 forward(s) "
                      f"in {el:.1f} s on {oracle.num_threads()} OpenMP threads"}


def run_mode(args, world):
    """'sharded' (the default for more than one rank, or --sharded), 'replicas'
    (--replicas with more than one rank) or 'single'."""
    if args.sharded or (world > 1 and not args.replicas):
        return "sharded"
    return "replicas" if world > 1 else "single"


def workload_config(args, w, world, mode, seg=None):
    """The `config` of the JSON line: the workload and how it is split; both arms of the
    bench (the library and the oracle) print the same one for the same command line."""
    par = {"single": "single process",
           "replicas": f"replicas x{world} (every rank the whole forward)",
           "sharded": f"row-sharded x{world} (NCCL all-gathers of the K/V row blocks and the partial S|z)"}[mode]
    return {"workload": args.workload if args.scale == 1.0 else f"{args.workload}@scale{args.scale}",
            "N": w.N, "E": w.E, "d": w.d, "H": w.H, "r": w.r, "io": w.io,
            "segments": 1 if seg is None else int(seg.shape[0] - 1), "parallelism": par, "l2": L2_NOTE}


def run_reference(args, rank, world):
    """The reference arm: the float64 oracle as it stands, on the host cores, rank 0 only;
    one step = one full oracle forward of the workload."""
    from sparse_graph_attention_tcgen05_b200.workloads import make_workload
    import oracle
    if rank != 0:
        return
    w = make_workload(args.workload, scale=args.scale)
    csr = oracle.csr_from_coo(w.N, w.src, w.dst)

    def step():
        oracle.forward(w.N, w.d, w.H, w.r, w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps,
                       csr[0], csr[1])
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter(); step(); times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = w.E * w.H / sec
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(args, w, world, run_mode(args, world)),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"one full float64 oracle forward of the {w.name} workload per step "
                                       f"(N={w.N}, E={w.E}) on {oracle.num_threads()} OpenMP threads, rank 0"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class TimedRegion:
    """K steps of R forwards: every forward is preceded by an L2 flush outside its span and
    bracketed by its own CUDA events on `stream`; one host synchronisation per step.
    `after_step` (optional) is called after each step's synchronisation."""

    def __init__(self, stream, flush, R):
        import torch
        self.stream, self.flush, self.R = stream, flush, R
        self.evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(R)]

    def step(self, run_fwd, run_last=None):
        for i, (a, b) in enumerate(self.evs):
            self.flush.zero_()
            a.record(self.stream)
            (run_last if run_last is not None and i == self.R - 1 else run_fwd)()
            b.record(self.stream)
        self.evs[-1][1].synchronize()
        self.last_ms = self.evs[-1][0].elapsed_time(self.evs[-1][1])   # the step's last forward
        return sum(a.elapsed_time(b) for a, b in self.evs)

    def run(self, run_fwd, K, gpu_index, barrier=None, after_step=None, run_last=None):
        import torch
        if barrier:
            barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(gpu_index)
        wall0 = time.perf_counter()
        step_ms = []
        for _ in range(K):
            step_ms.append(self.step(run_fwd, run_last))
            if after_step:
                after_step()
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        clocks = sampler.stop()
        if barrier:
            barrier()
        return step_ms, clocks, wall


def gpu_index_of(local_rank):
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in visible.split(",") if v.strip()]
    return ids[local_rank] if local_rank < len(ids) else local_rank


def roofline_local(w, t_local_ms, peaks, peak_kind, counters, source):
    """Roofline object of the dominant kernel (the local softmax branch): algorithmic bytes
    per launch over its average launch time, against the measured HBM copy rate; with the
    ncu DRAM bytes per launch (when taken on the current source) the DRAM-level fraction."""
    s_io = 4 if w.io == "f32" else 2
    B_kern = local_kernel_bytes(w.N, w.E, w.D, s_io)
    achieved = B_kern / (t_local_ms * 1e-3) / 1e9
    ro = {"bound": "hbm", "kernel": "local_kernel (local softmax branch; writes L)",
          "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
          "frac": achieved / peaks["hbm_gbs"], "traffic": None,
          "algorithmic_bytes_per_launch": B_kern, "avg_launch_ms": t_local_ms, "launch_time_source": source,
          "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
          else "fallback 6.65 TB/s (no MEASURED_PEAKS.json)",
          "frac_note": "frac counts every k_j/v_j gather as HBM bytes; on this graph most gathers hit "
                       "L2, so dram_frac (ncu DRAM bytes over the same launch time) is the HBM-level "
                       "figure"}
    if counters and not counters.get("stale"):
        dram = float(counters["dram_bytes_per_launch"])
        ro["traffic"] = dram
        ro["dram_gbs"] = dram / (t_local_ms * 1e-3) / 1e9
        ro["dram_frac"] = ro["dram_gbs"] / peaks["hbm_gbs"]
        ro["warp_instructions_per_edge"] = counters.get("warp_instructions_per_edge")
        ro["counters_from"] = counters["file"]
    elif counters:
        ro["counters_from"] = counters["file"] + " (stale: taken on another local.cu)"
    return ro


def time_block(layer, w, X, Y, dt, dev, flush, stream, steps, peaks):
    """The block around the layer alone, Z = LayerNorm(X + Y Wo): CUDA events per call,
    L2 flushed between calls; FLOPs 2*N*(H*r)*d, bytes Y + X + Z + Wo."""
    import torch
    rng = np.random.default_rng(3)
    Wo = torch.from_numpy((rng.standard_normal((w.D, w.d)) / np.sqrt(w.D)).astype(np.float32)).to(dt).to(dev)
    g = torch.ones(w.d, dtype=dt, device=dev)
    b = torch.zeros(w.d, dtype=dt, device=dev)
    Z = torch.empty(w.N, w.d, dtype=dt, device=dev)
    for _ in range(3):
        layer.block_output(Y, X, Wo, g, b, 1e-5, Z)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for _ in range(steps):
        flush.zero_()
        ev0.record(stream)
        layer.block_output(Y, X, Wo, g, b, 1e-5, Z)
        ev1.record(stream)
        ev1.synchronize()
        ms.append(ev0.elapsed_time(ev1))
    assert layer.last_device_error() == 0
    t = float(np.mean(ms)) * 1e-3
    s = 4 if w.io == "f32" else 2
    flops = 2.0 * w.N * w.D * w.d
    nbytes = s * (w.N * w.D + 2 * w.N * w.d + w.D * w.d)
    return {"ms": t * 1e3, "tflops": flops / t / 1e12,
            "frac_of_tensor_peak": flops / t / (peaks["bf16_tflops"] * 1e12),
            "gbs": nbytes / t / 1e9, "frac_of_hbm": nbytes / t / 1e9 / peaks["hbm_gbs"],
            "arith_intensity_flop_per_byte": flops / nbytes}


def time_backward(layer, w, X, WQ, WK, WV, wg, dt, dev, flush, stream, steps):
    """glga_backward alone (after one forward with the same inputs): CUDA events per call,
    L2 flushed between calls."""
    import torch
    rng = np.random.default_rng(4)
    dY = torch.from_numpy(rng.standard_normal((w.N, w.D)).astype(np.float32)).to(dt).to(dev)
    layer.forward(X, WQ, WK, WV, wg, b_g=w.b_g, eps=w.eps)
    for _ in range(2):
        layer.backward(X, WQ, WK, WV, wg, w.b_g, w.eps, dY)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ms = []
    for _ in range(steps):
        flush.zero_()
        ev0.record(stream)
        layer.backward(X, WQ, WK, WV, wg, w.b_g, w.eps, dY)
        ev1.record(stream)
        ev1.synchronize()
        ms.append(ev0.elapsed_time(ev1))
    assert layer.last_device_error() == 0
    t = float(np.mean(ms))
    graph, _ = layer.capture_backward(X, WQ, WK, WV, wg, w.b_g, w.eps, dY)
    gms = []
    for _ in range(steps):
        flush.zero_()
        ev0.record(stream)
        graph.replay()
        ev1.record(stream)
        ev1.synchronize()
        gms.append(ev0.elapsed_time(ev1))
    del graph
    tg = float(np.mean(gms))
    return {"ms": t, "edge_heads_per_s": w.E * w.H / (t * 1e-3), "steps": steps,
            "graph_ms": tg, "graph_edge_heads_per_s": w.E * w.H / (tg * 1e-3),
            "kernels": (("gathers on the CUDA cores with bf16 rows kept packed (fma.rn.f32.bf16, f32 "
                         "accumulation); readout backward, dS | dz, the source side's global terms and "
                         "dX | dW in one pass over dZ on the tcgen05 tensor cores (H*r = 128, d = 128)")
                        if w.io == "bf16" else
                        "gathers, reductions and the dW / dX GEMMs on the CUDA cores (fp32 arithmetic)")}


def median_event_ms(fn, steps, warmup, flush):
    """Median over `steps` calls of fn, each timed with CUDA events on the current stream
    with L2 flushed before it (outside the timed span), after `warmup` untimed calls."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    times = []
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(steps):
        flush.zero_()
        ev0.record(stream)
        fn()
        ev1.record(stream)
        ev1.synchronize()
        times.append(ev0.elapsed_time(ev1))
    return float(np.median(times))


def sweep_points(exponents, k=8, steps=30, warmup=5, seed=0, d=32, H=1, r=16, io="f32", dense=None):
    """Forward time against N at fixed in-degree: by default the tiny config's shape
    (d=32, H=1, r=16, fp32, k distinct uniform in-neighbours + self-loop; the method page's
    cost-proxy setting |E|/N = 8, r = 16) at N = 2^e for each e.  Median of `steps`
    forwards, each timed with CUDA events on the launching stream, L2 flushed between
    them.  Returns [(N, E, ms)], or [(N, E, ms, dense)] with dense(w, args, flush) called
    on each point when given."""
    import torch
    from sparse_graph_attention_tcgen05_b200 import glga
    from sparse_graph_attention_tcgen05_b200.workloads import make_custom, uniform_in_neighbours
    dev = torch.device("cuda")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    dt = glga.torch_dtype(io)
    out = []
    for e in exponents:
        N = 1 << e
        src, dst = uniform_in_neighbours(N, k, seed)
        w = make_custom(N, d, H, r, src, dst, io=io, seed=seed + 1)
        row_ptr, col_idx = glga.csr_from_coo(N, torch.from_numpy(src).to(dev), torch.from_numpy(dst).to(dev))
        layer = glga.Layer(N, w.d, w.H, w.r, w.io, row_ptr, col_idx)
        args = [torch.from_numpy(a).to(dev).to(dt) for a in (w.X, w.W_Q, w.W_K, w.W_V, w.w_g)]
        Y = torch.empty(N, w.D, dtype=dt, device=dev)
        ms = median_event_ms(lambda: layer.forward(*args, b_g=w.b_g, eps=w.eps, Y=Y), steps, warmup, flush)
        if dense is None:
            out.append((N, w.E, ms))
        else:
            extra = dense(w, args, flush)
            graph, _ = layer.capture(*args, w.b_g, w.eps, Y=Y)
            extra["glga_graph_ms"] = median_event_ms(graph.replay, steps, warmup, flush)
            del graph
            out.append((N, w.E, ms, extra))
        assert layer.last_device_error() == 0
        layer.close()
    return out


def dense_attention_ms(w, args, flush, steps=20, warmup=3, masked_max_n=8192):
    """The dense baseline of the method page's cost comparison at the layer's width: the
    Q, K, V projections (torch matmul) and softmax attention of every node over all N nodes
    (torch scaled_dot_product_attention, a library kernel), timed like the layer; also the
    adjacency-masked form (each node over its CSR row only, as a boolean mask) up to
    masked_max_n nodes.  Not the product path: a comparison only."""
    import torch
    import torch.nn.functional as F
    X, WQ, WK, WV = args[:4]
    N, H, r = w.N, w.H, w.r

    def heads(t):
        return t.view(1, N, H, r).transpose(1, 2)

    def run(mask):
        q, k, v = heads(X @ WQ), heads(X @ WK), heads(X @ WV)
        return F.scaled_dot_product_attention(q, k, v, attn_mask=mask)

    res = {"dense_ms": median_event_ms(lambda: run(None), steps, warmup, flush), "masked_ms": None}
    if N <= masked_max_n:
        mask = torch.zeros(N, N, dtype=torch.bool, device=X.device)
        mask[torch.from_numpy(w.dst.astype(np.int64)).to(X.device),
             torch.from_numpy(w.src.astype(np.int64)).to(X.device)] = True
        res["masked_ms"] = median_event_ms(lambda: run(mask), steps, warmup, flush)
        del mask
    return res


def run_dense_sweep():
    """Dense-vs-hybrid latency at matched width (the arxiv width: d=128, H=4, r=32, bf16):
    N = 2^10 .. 2^16 at in-degree 8 (+ self-loop), then in-degree 4 .. 128 at N = 2^14."""
    rows = []
    for k, exps in ((8, range(10, 17)), (4, [14]), (16, [14]), (32, [14]), (64, [14]), (128, [14])):
        for N, E, ms, dn in sweep_points(exps, k=k, steps=20, warmup=3, d=128, H=4, r=32, io="bf16",
                                         dense=dense_attention_ms):
            rows.append({"N": N, "in_degree": k, "E": E, "glga_ms": ms, **dn,
                         "dense_over_glga_graph": dn["dense_ms"] / dn["glga_graph_ms"],
                         "dense_over_glga": dn["dense_ms"] / ms,
                         "masked_over_glga": None if dn["masked_ms"] is None else dn["masked_ms"] / ms})
    n_pts = [p for p in rows if p["in_degree"] == 8]
    print(json.dumps({"dense_sweep": "layer forward (glga) vs dense softmax attention (projections + "
                                     "torch SDPA over all N; masked: over the CSR row) at d=128, H=4, "
                                     "r=32, bf16; median of 20, L2 flushed",
                      "points": rows,
                      "glga_loglog_slope_N": loglog_slope([(p["N"], p["E"], p["glga_ms"]) for p in n_pts
                                                           if p["N"] >= (1 << 13)]),
                      "dense_loglog_slope_N": loglog_slope([(p["N"], p["E"], p["dense_ms"]) for p in n_pts
                                                            if p["N"] >= (1 << 13)])}))


def loglog_slope(points):
    """Least-squares slope of log(ms) against log(N)."""
    x = np.log([p[0] for p in points])
    y = np.log([p[2] for p in points])
    return float(np.polyfit(x, y, 1)[0])


def run_sweep():
    pts = sweep_points(range(12, 22))
    upper = [p for p in pts if p[0] >= (1 << 17)]
    print(json.dumps({"sweep": "forward ms vs N at fixed in-degree 8 (+ self-loop), d=32, H=1, "
                               "r=16, fp32; median of 30, L2 flushed",
                      "points": [{"N": n, "E": e, "ms": ms} for n, e, ms in pts],
                      "slope_loglog_all": loglog_slope(pts),
                      "slope_loglog_N_ge_2^17": loglog_slope(upper)}), flush=True)


def e2e_pipelined(layer, w, host, dt, dev, steps, warmup=3, graphs=False):
    """End-to-end throughput through the public API: every step copies its inputs (X and
    the weights) from pinned host memory, runs the forward and copies Y back to pinned host
    memory.  The inputs sit in one glga.HostInputs slab, so they cross PCIe as one copy per
    step.  Copies run on their own streams with two slots, so step i's host->device copy
    and step i-1's device->host copy overlap step i's forward (PCIe is full duplex); events
    order every buffer reuse.  With `graphs` each slot's forward is a Layer.capture graph
    replayed per step, as in the device-timed value.  Device time from the first copy's
    start to the last copy's end."""
    import torch
    from sparse_graph_attention_tcgen05_b200 import glga
    stage = glga.HostInputs(w.N, w.d, w.D, dt, dev, slots=2)
    for k in stage.NAMES:
        stage.host[k].copy_(host[k])
    Yd = [torch.empty(w.N, w.D, dtype=dt, device=dev) for _ in range(2)]
    Yh = [torch.empty(w.N, w.D, dtype=dt).pin_memory() for _ in range(2)]
    comp = torch.cuda.current_stream()
    replays = None
    if graphs:
        replays = [layer.capture(*stage.device_inputs[b], w.b_g, w.eps, Y=Yd[b])[0] for b in range(2)]
        torch.cuda.synchronize()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i % 2
        if used[b]:
            s_in.wait_event(ev_fwd[b])              # the forward that read slot b is done
        ins = stage.upload(b, s_in)
        ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        if used[b]:
            comp.wait_event(ev_out[b])              # Y buffer b has been copied out
        if replays is not None:
            replays[b].replay()
        else:
            layer.forward(*ins, b_g=w.b_g, eps=w.eps, Y=Yd[b], stream=comp)
        ev_fwd[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_fwd[b])
            Yh[b].copy_(Yd[b], non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        step(warmup + i)
    t1.record(s_out)
    t1.synchronize()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    del replays
    return ms, stage.nbytes, Yh[0].numel() * Yh[0].element_size()


def run_sharded(args, rank, world, local_rank):
    """Row-sharded forward (sharded.ShardedForward): every rank owns a contiguous block of
    target rows with about equal CSR entries, projects them, exchanges K/V row blocks and
    partial statistics over NCCL (two all-gathers) and finishes its rows.  Total work is
    fixed as ranks are added (strong scaling); value = E*H per forward over the slowest
    rank's time."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from sparse_graph_attention_tcgen05_b200 import glga
    from sparse_graph_attention_tcgen05_b200.sharded import LibraryShard, ShardedForward, ShardPlan
    from sparse_graph_attention_tcgen05_b200.workloads import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if not dist.is_initialized():
        if world > 1:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        else:
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=300))
    w = make_workload(args.workload, scale=args.scale)
    dt = glga.torch_dtype(w.io)
    row_ptr, col_idx = glga.csr_from_coo(w.N, torch.from_numpy(w.src).to(dev), torch.from_numpy(w.dst).to(dev))
    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    plan = ShardPlan(rp, ci, world, rank)
    shard = LibraryShard(plan.n_kv, w.d, w.H, w.r, w.io, plan.row_ptr, plan.col_idx, plan.kv0, plan.kv1,
                         device=dev)
    fwd = ShardedForward(shard, rank, world)
    names = ("X", "W_Q", "W_K", "W_V", "w_g")
    host = {"X": torch.from_numpy(np.ascontiguousarray(w.X[plan.b0:plan.b1])).to(dt).pin_memory()}
    for k, a in zip(names[1:], (w.W_Q, w.W_K, w.W_V, w.w_g)):
        host[k] = torch.from_numpy(a).to(dt).pin_memory()
    X, WQ, WK, WV, wg = (host[k].to(dev) for k in names)
    Y = torch.empty(plan.b1 - plan.b0, w.D, dtype=dt, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def run_fwd():
        fwd(X, WQ, WK, WV, wg, w.b_g, w.eps, Y)

    for _ in range(args.warmup):
        run_fwd()
    torch.cuda.synchronize()
    assert shard.last_device_error() == 0
    parity = None
    if not args.no_parity and plan.b1 > plan.b0:
        import oracle
        rng = np.random.default_rng(rank)
        rows = np.unique(rng.integers(plan.b0, plan.b1, min(256, plan.b1 - plan.b0)))
        ref = oracle.forward(w.N, w.d, w.H, w.r, w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps,
                             rp, ci, rows=rows)
        got = Y.float().cpu().numpy()[rows - plan.b0].astype(np.float64)
        parity = float(np.abs(got - ref["Y"]).max() / np.abs(ref["Y"]).max())
    stream = torch.cuda.current_stream()
    # the local kernel's launch time: stage events of the last forward of every step
    shard.set_timing(True)
    local_ms = []
    launches0 = shard.kernel_launches()
    tr = TimedRegion(stream, flush, args.forwards_per_step)
    step_ms, clocks, wall = tr.run(run_fwd, args.steps, gpu_index_of(local_rank), barrier=dist.barrier,
                                   after_step=lambda: local_ms.append(shard.stage_times()["local"]))
    launches = shard.kernel_launches() - launches0
    shard.set_timing(False)
    assert shard.last_device_error() == 0
    total = max_over_ranks_dist(sum(step_ms), world, dev)
    n_fwd = args.steps * args.forwards_per_step
    # end to end: the rank's X rows and the weights in, its Y rows out, per forward
    Yh = torch.empty_like(Y, device="cpu").pin_memory()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = []
    for i in range(args.e2e_steps + 3):
        ev0.record(stream)
        for t, k in zip((X, WQ, WK, WV, wg), names):
            t.copy_(host[k], non_blocking=True)
        run_fwd()
        Yh.copy_(Y, non_blocking=True)
        ev1.record(stream)
        ev1.synchronize()
        if i >= 3:
            e2e_ms.append(ev0.elapsed_time(ev1))
    e2e_total = max_over_ranks_dist(sum(e2e_ms), world, dev)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    peaks, peak_kind = load_peaks()
    t_local = float(np.mean(local_ms)) if local_ms else float("nan")
    line = {"metric": METRIC, "value": w.E * w.H * n_fwd / (total * 1e-3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps, "forwards_per_step": args.forwards_per_step,
            "ms_per_forward": total / n_fwd, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": w.io, "data": "synthetic",
            "config": workload_config(args, w, world, "sharded"),
            "rows_per_rank_0": plan.b1 - plan.b0, "kv_rows_padded": plan.n_kv,
            "roofline": roofline_local(w, t_local, peaks, peak_kind, None,
                                       "stage events of rank 0's local kernel (its own rows), timed region"),
            "gpu_launches": int(launches),
            "e2e": {"value": w.E * w.H * len(e2e_ms) / (e2e_total * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": Yh.numel() * Yh.element_size(),
                    "ms_per_step": e2e_total / len(e2e_ms), "note": "per rank: its X rows and the weights "
                    "in, its Y rows out, serial on one stream; bytes are rank 0's"},
            "clocks": clocks, "wall_s_timed_region": wall, "parity_max_rel_err": parity}
    # the roofline above uses rank 0's rows only: scale its algorithmic bytes to them
    if plan.b1 > plan.b0:
        frac_rows = (plan.b1 - plan.b0) / w.N
        line["roofline"]["note"] = (f"algorithmic bytes of the whole graph; rank 0 holds {frac_rows:.3f} "
                                    "of the rows and about 1/P of the entries")
    if rank == 0:
        print(json.dumps(line), flush=True)
    shard.close()
    dist.barrier()
    dist.destroy_process_group()


def run_single(args, rank, world, local_rank, mode):
    """One process per GPU, each running the whole forward (one GPU, or replicas)."""
    import torch
    import torch.distributed as dist
    from sparse_graph_attention_tcgen05_b200 import glga
    from sparse_graph_attention_tcgen05_b200.workloads import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return max_over_ranks_dist(x, world, dev)

    w = make_workload(args.workload, scale=args.scale)
    dt = glga.torch_dtype(w.io)
    s_io = 4 if w.io == "f32" else 2

    # ---- bind the graph (CSR build + create), timed separately ----
    src = torch.from_numpy(w.src).to(dev)
    dst = torch.from_numpy(w.dst).to(dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    row_ptr, col_idx = glga.csr_from_coo(w.N, src, dst)
    t1 = time.perf_counter()
    seg = None
    if args.segment_len > 0:
        seg = np.unique(np.concatenate([np.arange(0, w.N, args.segment_len), [w.N]])).astype(np.int64)
    opts = glga.default_options()
    opts.backward = 1 if args.backward else 0
    layer = glga.Layer(w.N, w.d, w.H, w.r, w.io, row_ptr, col_idx, opts, segments=seg)
    torch.cuda.synchronize()
    t2 = time.perf_counter()
    create = {"csr_from_coo_ms": (t1 - t0) * 1e3, "glga_create_ms": (t2 - t1) * 1e3,
              "buckets": layer.bucket_counts(), "workspace_bytes": layer.workspace_bytes()}

    host = {k: torch.from_numpy(np.ascontiguousarray(a)).to(dt).pin_memory()
            for k, a in (("X", w.X), ("W_Q", w.W_Q), ("W_K", w.W_K), ("W_V", w.W_V), ("w_g", w.w_g))}
    X, WQ, WK, WV, wg = (host[k].to(dev) for k in ("X", "W_Q", "W_K", "W_V", "w_g"))
    Y = torch.empty(w.N, w.D, dtype=dt, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def fwd():
        layer.forward(X, WQ, WK, WV, wg, b_g=w.b_g, eps=w.eps, Y=Y)

    # ---- warm-up ----
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    assert layer.last_device_error() == 0

    # ---- parity spot check of what is being timed (sampled rows vs the oracle) ----
    parity = None
    if rank == 0 and not args.no_parity:
        import oracle
        csr = (row_ptr.cpu().numpy(), col_idx.cpu().numpy())
        rng = np.random.default_rng(0)
        rows = np.unique(np.concatenate([rng.choice(w.N, min(256, w.N), replace=False),
                                         np.argsort(np.diff(csr[0]))[-8:]]))
        ref = oracle.forward(w.N, w.d, w.H, w.r, w.X, w.W_Q, w.W_K, w.W_V, w.w_g, w.b_g, w.eps,
                             csr[0], csr[1], rows=rows, seg_ptr=seg)
        Yg = Y.float().cpu().numpy()[rows].astype(np.float64)
        parity = float(np.abs(Yg - ref["Y"]).max() / np.abs(ref["Y"]).max())

    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    # ---- eager forwards with the library's stage events: per-stage times, launch count ----
    n_eager = 100
    layer.set_timing(True)
    launches0 = layer.kernel_launches()
    stage_sum = {k: 0.0 for k in glga.STAGES}
    eager_ms = []
    for _ in range(n_eager):
        flush.zero_()
        ev0.record(stream)
        fwd()
        ev1.record(stream)
        ev1.synchronize()
        eager_ms.append(ev0.elapsed_time(ev1))
        for k, v in layer.stage_times().items():
            stage_sum[k] += v
    launches_per_forward = (layer.kernel_launches() - launches0) / n_eager
    stages = {k: v / n_eager for k, v in stage_sum.items()}
    eager_total = max_over_ranks(sum(eager_ms))
    eager = {"value": replica_throughput(world, w.E * w.H, eager_total, n_eager), "unit": UNIT,
             "ms_per_step": eager_total / n_eager, "steps": n_eager,
             "note": "glga_forward called per forward, stage events on"}

    # ---- timed region: K steps of R forwards, each a replay of a CUDA graph of
    # glga_forward (the same kernels on the same buffers, no host work between them); the
    # last forward of every step replays a second graph that also records the library's
    # stage events (event record nodes), for the local kernel's launch time; eager calls
    # if the capture is refused ----
    graph, graph_t = None, None
    layer.set_timing(False)
    try:
        graph, _ = layer.capture(X, WQ, WK, WV, wg, w.b_g, w.eps, Y=Y)
    except RuntimeError as exc:
        eager["capture_refused"] = str(exc).splitlines()[0][:200]
    if graph is not None:
        layer.set_timing(True)
        try:
            graph_t, _ = layer.capture(X, WQ, WK, WV, wg, w.b_g, w.eps, Y=Y)
            graph_t.replay()
            torch.cuda.synchronize()
            layer.stage_times()
        except (RuntimeError, glga.GLGAError) as exc:
            eager["capture_with_stage_events"] = str(exc).splitlines()[0][:200]
            graph_t = None
            layer.set_timing(False)
    run_step = graph.replay if graph is not None else fwd
    for _ in range(args.warmup):
        run_step()
    local_ms, fwd_check = [], []
    tr = TimedRegion(stream, flush, args.forwards_per_step)

    def after():
        st = layer.stage_times()
        local_ms.append(st["local"])
        fwd_check.append(st["forward"] / tr.last_ms)
    step_ms, clocks, wall = tr.run(run_step, args.steps, gpu_index_of(local_rank),
                                   barrier=barrier if world > 1 else None,
                                   after_step=after if graph_t is not None else None,
                                   run_last=graph_t.replay if graph_t is not None else None)
    layer.set_timing(False)
    # the graph's stage events must span the same forward as the outer events
    if fwd_check and not 0.8 <= float(np.median(fwd_check)) <= 1.05:
        eager["graph_stage_events"] = f"rejected (forward span / outer events = {float(np.median(fwd_check)):.3f})"
        local_ms = []
    graph_ok = graph is not None
    del graph, graph_t
    assert layer.last_device_error() == 0
    n_fwd = args.steps * args.forwards_per_step
    launches = int(round(launches_per_forward * n_fwd))
    total_ms = max_over_ranks(sum(step_ms))
    value = replica_throughput(world, w.E * w.H, total_ms, n_fwd)

    # ---- end to end through the public API: pinned host -> device, forward, Y -> host ----
    e2e_ms, h2d, d2h = e2e_pipelined(layer, w, host, dt, dev, args.e2e_steps)
    e2e_total = max_over_ranks(e2e_ms)
    e2e = {"value": replica_throughput(world, w.E * w.H, e2e_total, args.e2e_steps), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_total / args.e2e_steps,
           "note": "Layer.forward per step with its inputs copied in (one glga.HostInputs slab: X and "
                   "the weights, pinned) and Y copied out to pinned host memory; copies on their own "
                   "streams, two slots, overlapping the forwards"}

    peaks, peak_kind = load_peaks()
    if local_ms:
        t_local, src_t = float(np.mean(local_ms)), ("stage events recorded inside the replayed graph of the "
                                                    "last forward of every timed step")
    else:
        t_local, src_t = stages["local"], "stage events of the eager forwards"
    roofline = roofline_local(w, t_local, peaks, peak_kind, profiled_counters(args.workload), src_t)
    # steps a3-a5 (local branch, readout, gate) against the fused-branch byte model
    B_loc = branch_bytes_model(w.N, w.E, w.D, w.H, w.r, s_io)
    t_branch = (stages["local"] + stages["readout"]) * 1e-3
    branch = {"bytes": B_loc, "ms": t_branch * 1e3, "gbs": B_loc / t_branch / 1e9,
              "frac": B_loc / t_branch / 1e9 / peaks["hbm_gbs"],
              "compulsory_bytes": branch_compulsory_bytes(w.N, w.E, w.D, w.H, w.r, s_io)}
    gemm_flops = 2.0 * w.N * w.d * (3 * w.D + 1)
    gemm_bytes = w.N * w.d * s_io + w.N * 3 * w.D * s_io + 4 * w.N
    t_gemm = stages["gemm"] * 1e-3
    tpeak = peaks["bf16_tflops"]
    attainable = min(tpeak * 1e12, gemm_flops / gemm_bytes * peaks["hbm_gbs"] * 1e9)
    projection = {"tflops": gemm_flops / t_gemm / 1e12, "frac_of_tensor_peak": gemm_flops / t_gemm / (tpeak * 1e12),
                  "frac_of_attainable": gemm_flops / t_gemm / attainable,
                  "arith_intensity_flop_per_byte": gemm_flops / gemm_bytes,
                  "hbm_gbs": gemm_bytes / t_gemm / 1e9}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "forwards_per_step": args.forwards_per_step, "ms_per_forward": total_ms / n_fwd,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.io,
            "data": "synthetic", "config": workload_config(args, w, world, mode, seg),
            "roofline": roofline, "local_branch_a3_a5": branch, "projection": projection,
            "stages_ms": stages, "create": create, "gpu_launches": launches,
            "e2e": e2e, "eager": eager, "timed_region": ("CUDA graph replays of glga_forward" if graph_ok
                                                         else "eager glga_forward"),
            "clocks": clocks, "parity_max_rel_err": parity, "wall_s_timed_region": wall}
    if args.block:
        line["block"] = time_block(layer, w, X, Y, dt, dev, flush, stream, 200, peaks)
    if args.backward:
        line["backward"] = time_backward(layer, w, X, WQ, WK, WV, wg, dt, dev, flush, stream, args.backward_steps)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, (row_ptr.cpu().numpy(), col_idx.cpu().numpy()))
    if rank == 0:
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--forwards-per-step", type=int, default=300,
                    help="forwards per timed step (each with its own L2 flush and events)")
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default="arxiv")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink the workload (small profiling captures only; reported lines use 1.0)")
    ap.add_argument("--no-parity", action="store_true", help="skip the sampled-row oracle check")
    ap.add_argument("--segment-len", type=int, default=0,
                    help="segments of this many nodes, each with its own global statistics "
                         "(a batch of graphs; 0 = one segment over all nodes)")
    ap.add_argument("--backward-steps", type=int, default=50,
                    help="timed glga_backward calls (and as many graph replays) with --backward")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward pass (glga_backward) of the same forward")
    ap.add_argument("--block", action="store_true",
                    help="also time the block around the layer, Z = LayerNorm(X + Y Wo)")
    ap.add_argument("--sharded", action="store_true",
                    help="the row-sharded forward also on one rank (the default for more than one)")
    ap.add_argument("--replicas", action="store_true",
                    help="with more than one rank, every rank runs the whole forward (weak scaling)")
    ap.add_argument("--dense-sweep", action="store_true",
                    help="layer forward against dense softmax attention over N and in-degree")
    ap.add_argument("--sweep", action="store_true",
                    help="time the forward against N at fixed degree instead (one JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.forwards_per_step = max(args.forwards_per_step, 1)
    if args.sweep:
        run_sweep()
        return
    if args.dense_sweep:
        run_dense_sweep()
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    mode = run_mode(args, world)
    if mode == "sharded":
        run_sharded(args, rank, world, local_rank)
    else:
        run_single(args, rank, world, local_rank, mode)


if __name__ == "__main__":
    main()
