"""Benchmark of the quantized-matmul hot path on B200.

Headline (``metric``): weight GB/s of the 4-bit G=64 QMV kernel at M=1 on the
decode workload: one "step" is a decode pass through three Llama-3-8B-shaped
linears, (K, N) = (4096, 4096), (4096, 14336), (14336, 4096), each a
``aq_matmul`` of one bf16 activation row against affine 4-bit G=64 weights.
value = packed weight + scale + bias bytes of a step / step time, summed over
ranks (weak scaling: every rank runs its own copy of the workload).

Also measured in the same run (``sections``): QMM prefill TFLOP/s (M = 8192,
K = 4096, N = 14336, the tensor-core kernel), the M = 1..8 QMV curve, and the
quantize / dequantize kernels.  Inputs are synthetic (seeded; shapes of the
models the pages measure on), resident in HBM before timing; weight sets are
rotated so every timed launch reads HBM (working set > 126 MB L2).

``--impl reference`` times the CPU oracle (the plain C statement of the method)
on the host cores for the same metric: see ``oracle/``.
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

import synth  # noqa: E402

L2_BYTES = 126 * 2 ** 20
DECODE_SHAPES = [(4096, 4096), (4096, 14336), (14336, 4096)]  # (K, N)
G, BITS = 64, 4
METRIC = "4-bit G64 QMV weight GB/s (% of HBM peak) at M=1; QMM prefill TFLOP/s"
WORKLOAD = ("decode step: QMV M=1 over Llama-3-8B linears (K,N) = (4096,4096), (4096,14336), (14336,4096); "
            "affine 4-bit G=64; W ~ N(0,0.02) with 0.1% x10 outliers; x ~ N(0,1) bf16")


def weight_bytes(K, N, g=G, bits=BITS):
    return N * K * bits // 8 + 4 * N * K // g


STEP_BYTES = sum(weight_bytes(K, N) for K, N in DECODE_SHAPES)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(files=None):
    """Hash of CUDA sources of the library (all of them, or the named files of
    csrc/): a recorded ncu figure is only reported while the kernel it was taken
    on is unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_group_b200", "csrc")
    names = sorted(files) if files else sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for f in names:
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(name):
    """DRAM bytes per unit for a kernel from a committed ncu summary, if the sources
    that kernel is built from have not changed since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "counters.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(name)
    if not e or e.get("source_hash") != kernel_source_hash(e.get("sources")):
        return None
    return e.get("dram_bytes_per_unit")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.index = str(device_index)
        try:  # the GPU's UUID identifies it for nvidia-smi regardless of CUDA_VISIBLE_DEVICES
            import torch
            self.index = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            pass
        self.proc = None
        self.path = os.path.join("/tmp", f"aq_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- ranks (host plumbing only)

def _dist():
    try:
        import torch.distributed as dist
    except ImportError:
        return None
    return dist if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1 else None


def rank_barrier(device=None):
    dist = _dist()
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_max(v, device=None):
    """Max of a per-rank scalar over all ranks (identity on one rank)."""
    dist = _dist()
    if dist is None:
        return v
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(bytes_per_step, steps_per_rank, world, ms_max):
    """Whole-job throughput: the bytes all ranks processed over the slowest rank's time."""
    return bytes_per_step * steps_per_rank * world / (ms_max * 1e-3) / 1e9


# ----------------------------------------------------------------------------- our implementation

def run_sharded(args, rank, world, local_rank):
    """The decode step with W split along N over the ranks (weight_only_group_b200.shard):
    each rank streams its rows of the three linears and one NCCL all-gather per step
    assembles the three y.  The job processes STEP_BYTES per step whatever the
    number of ranks (strong scaling)."""
    import torch
    import torch.distributed as dist

    import weight_only_group_b200 as aq
    from weight_only_group_b200 import shard
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = read_peaks()
    layer = []
    for si, (K, N) in enumerate(DECODE_SHAPES):
        seed = 1000 + 100 * 2 + si
        w = torch.from_numpy(synth.weights(N, K, seed)).to(dev)
        p, s, b = aq.aq_quantize(w, G, BITS)
        del w
        pl, sl, bl, n0, n1 = shard.shard_rows(p, s, b, world, rank)
        layer.append((pl.contiguous(), sl.contiguous(), bl.contiguous(), synth.activations(1, K, seed + 1).to(dev), N))

    def step():
        ys = [aq.aq_matmul(x, p, s, b, G, BITS, overlap_previous=True) for (p, s, b, x, N) in layer]
        return [shard.all_gather_columns(y, N) for y, (_, _, _, _, N) in zip(ys, layer)]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rank_barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    rank_barrier(dev)
    ms_max = reduce_max(e0.elapsed_time(e1), dev)
    value = STEP_BYTES * args.steps / (ms_max * 1e-3) / 1e9
    return {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 6), "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic (seeded; shapes of Llama-3-8B linears; no checkpoints)",
            "config": {"workload": WORKLOAD, "M": 1, "bits": BITS, "G": G, "shapes_KN": DECODE_SHAPES,
                       "parallelism": f"W split along N over {world} ranks; one NCCL all-gather of y per linear",
                       "l2": "each rank's slice is read once per step (no rotation)"},
            "gpu_launches": args.steps * len(DECODE_SHAPES),
            "roofline": {"bound": "hbm", "achieved": round(value / world, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(value / world / peaks["hbm_gbs"], 4), "traffic": None}}, {}


def run_ours(args, rank, world, local_rank):
    import torch
    import weight_only_group_b200 as aq

    if args.shard and world > 1:
        return run_sharded(args, rank, world, local_rank)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    def barrier():
        rank_barrier(dev)

    def max_over_ranks(v):
        return reduce_max(v, dev)

    peaks = read_peaks()
    stream = torch.cuda.Stream(dev)

    # -- resident inputs: weight sets rotated so the working set exceeds L2
    copies = max(2, -(-2 * L2_BYTES // STEP_BYTES) + 1)
    sets = []
    for ci in range(copies):
        layer = []
        for si, (K, N) in enumerate(DECODE_SHAPES):
            seed = 1000 + 100 * 2 + si
            if ci == 0:
                w = torch.from_numpy(synth.weights(N, K, seed)).to(dev)
                p, s, b = aq.aq_quantize(w, G, BITS)
                del w
            else:
                p, s, b = (t.clone() for t in sets[0][si][:3])
            x = synth.activations(1, K, seed + 1).to(dev)
            y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
            layer.append((p, s, b, x, y))
        sets.append(layer)
    torch.cuda.synchronize()

    # Each launch may start while the previous one finishes (programmatic dependent
    # launch): it reads its activations only after the previous kernel has
    # completed, and the weights, which nothing writes during the step, before.
    def step(layer):
        for (p, s, b, x, y) in layer:
            aq.aq_matmul(x, p, s, b, G, BITS, out=y, overlap_previous=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            for layer in sets:
                step(layer)
    torch.cuda.synchronize()
    # One graph holds whole rotations over the weight sets, about 20 steps (fewer
    # graph boundaries inside the timed region); the timed steps are whole graphs.
    per_graph = copies * max(1, min(-(-20 // copies), -(-args.steps // copies)))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(per_graph):
            step(sets[i % copies])
    reps_w = max(1, -(-args.warmup // per_graph))
    reps = max(1, -(-args.steps // per_graph))
    steps = reps * per_graph
    for _ in range(reps_w):
        graph.replay()
    torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        with torch.cuda.stream(stream):
            # an untimed replay ahead of the start event keeps the GPU busy while
            # the host submits the timed replays (else the first submission's host
            # time would count as step time)
            graph.replay()
            e0.record(stream)
            for _ in range(reps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms)
    clocks = clk.summary()
    value = aggregate_gbs(STEP_BYTES, steps, world, ms_max)
    ms_per_step = ms_max / steps
    achieved = STEP_BYTES / (ms / steps * 1e-3) / 1e9  # this rank's kernel-only GB/s (the step is 3 QMV launches)
    traffic = recorded_traffic("qmv_decode_step")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "traffic_unit": "DRAM bytes read + written per decode step (3 launches), from ncu",
                "peak_source": peaks["source"], "frac_of_8TBs_nominal": round(achieved / 8000.0, 4),
                "kernel": ("qmv_tc_kernel<bits=4,G=64,MP=1> (mma.sync m16n8k32: u8 codes x both signed-byte digit planes of "
                           "16-bit fixed-point activations in one MMA, int32 accumulate, fp32 fold; 3 launches per step)"),
                "algorithmic_bytes_per_step": STEP_BYTES}
    del graph

    # -- end to end through the public API with host buffers (pinned), per step:
    #    one H2D copy of the three linears' x (one pinned buffer), three aq_matmul
    #    calls, one D2H copy of the three y, read on the host
    e2e_steps = min(steps, args.e2e_steps)
    kx = [K for K, N in DECODE_SHAPES]
    ny = [N for K, N in DECODE_SHAPES]
    hx = torch.cat([synth.activations(1, K, 7) for K in kx], dim=1).pin_memory()
    hy = torch.empty((1, sum(ny)), dtype=torch.bfloat16).pin_memory()
    dx = torch.empty_like(hx, device=dev)
    dy = torch.empty((1, sum(ny)), dtype=torch.bfloat16, device=dev)
    xs_e2e = [dx[:, a:a + K] for a, K in zip([sum(kx[:i]) for i in range(len(kx))], kx)]
    ys_e2e = [dy[:, a:a + N] for a, N in zip([sum(ny[:i]) for i in range(len(ny))], ny)]
    h2d = hx.numel() * 2
    d2h = hy.numel() * 2

    def e2e_step(layer):
        dx.copy_(hx, non_blocking=True)
        for (p, s, b, _, _), x, y in zip(layer, xs_e2e, ys_e2e):
            aq.aq_matmul(x, p, s, b, G, BITS, out=y, overlap_previous=True)
        hy.copy_(dy, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        return float(hy[0, -1])

    with torch.cuda.stream(stream):
        for i in range(20):
            e2e_step(sets[i % copies])
        barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(e2e_steps):
            e2e_step(sets[i % copies])
        f1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1))
    e2e = {"value": round(STEP_BYTES * e2e_steps * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "ms_per_step": round(e2e_ms / e2e_steps, 5)}
    del sets
    torch.cuda.empty_cache()

    sections = {}
    if args.sections != "none":
        sections = measure_sections(args, aq, torch, dev, stream, peaks)

    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": (reps_w + 1) * per_graph, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic (seeded; shapes of Llama-3-8B linears; no checkpoints)",
            "config": {"workload": WORKLOAD, "M": 1, "bits": BITS, "G": G, "shapes_KN": DECODE_SHAPES,
                       "parallelism": f"replicas x{world} (no data-path collective)",
                       "l2": f"rotating {copies} resident weight sets ({copies * STEP_BYTES / 2**20:.0f} MiB > "
                             f"126 MiB L2); step replayed from a CUDA graph"},
            "pct_of_hbm_peak": round(value / world / peaks["hbm_gbs"] * 100, 2),
            "roofline": roofline, "e2e": e2e, "gpu_launches": steps * len(DECODE_SHAPES),
            "clocks": clocks}
    line.update(compact_sections(sections))
    return line, sections


def compact_sections(sec):
    """The headline figures of every workload, small enough for the final line:
    per-shape decode GB/s, the M = 1..8 curve, the bits x G sweep (GB/s) and the
    prefill QMM points (TFLOP/s and fraction of the burst bf16 peak)."""
    out = {}
    if "decode_shapes" in sec:
        out["decode_shapes_GBps"] = {k: v["weight_GBps"] for k, v in sec["decode_shapes"].items()}
    if "qmv_small_m" in sec:
        out["small_m_GBps"] = {k: v["weight_GBps"] for k, v in sec["qmv_small_m"]["curve"].items()}
    if "qmv_small_m_long_k" in sec:
        out["small_m_long_k_GBps"] = {k: v["weight_GBps"] for k, v in sec["qmv_small_m_long_k"]["curve"].items()}
    if "qmv_bits_group_sweep" in sec:
        out["sweep_GBps"] = {k: v["weight_GBps"] for k, v in sec["qmv_bits_group_sweep"]["points"].items()}
    if "decode_sequence" in sec:
        out["decode_sequence_GBps"] = {k: v["weight_GBps"] for k, v in sec["decode_sequence"].items()}
    if "qmm_prefill" in sec:
        out["qmm_prefill"] = {k: [v["TFLOP/s"], v["frac_of_burst"]] for k, v in sec["qmm_prefill"]["points"].items()}
        out["qmm_prefill_unit"] = "[TFLOP/s, fraction of the measured burst bf16 peak]"
    return out


def timed_graph(torch, stream, fn, reps_inner, reps_outer):
    """Capture reps_inner calls of fn into a graph; time reps_outer replays; ms per call."""
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn(0)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps_inner):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps_outer):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / (reps_inner * reps_outer)


def measure_sections(args, aq, torch, dev, stream, peaks):
    out = {}
    want = set(args.sections.split(",")) if args.sections != "all" else {"shapes", "seq", "qmm", "curve", "sweep",
                                                                         "quant", "embed", "gather", "mxfp4"}
    if "shapes" in want:
        out.update(section_decode_shapes(args, aq, torch, dev, stream, peaks))
    if "seq" in want:
        out.update(section_decode_sequence(args, aq, torch, dev, stream, peaks))
    if "qmm" in want:
        out.update(section_qmm(args, aq, torch, dev, stream, peaks))
    if "curve" in want:
        out.update(section_curve(args, aq, torch, dev, stream, peaks))
    if "sweep" in want or "quant" in want:
        out.update(section_sweep_quant(args, aq, torch, dev, stream, peaks, want))
    if "embed" in want:
        out.update(section_embedding(args, aq, torch, dev, stream, peaks))
    if "gather" in want:
        out.update(section_gather(args, aq, torch, dev, stream, peaks))
    if "mxfp4" in want:
        out.update(section_mxfp4(args, aq, torch, dev, stream, peaks))
    return out


def section_gather(args, aq, torch, dev, stream, peaks):
    """MoE gather matmul: eight experts of a 14336 x 4096 projection (4-bit G64, a
    Mixtral-8x7B-size w1), tokens routed top-2; weight GB/s of the expert rows
    read.  Consecutive calls route to different experts (the stack, 264 MB, is
    larger than L2), as consecutive tokens of a decode would."""
    E, N, K = 8, 14336, 4096
    w = torch.randn((E * N, K), device=dev, dtype=torch.float32, generator=torch.Generator(device=dev).manual_seed(7)) * 0.02
    p, s, b = aq.aq_quantize(w, G, BITS)
    del w
    torch.cuda.empty_cache()
    gp, gs, gb = p.view(E, N, -1), s.view(E, N, -1), b.view(E, N, -1)
    res = {}
    for tokens in (1, 4):
        T = 2 * tokens
        routes = [torch.tensor([(2 * r + j) % E for j in range(T)], dtype=torch.int32, device=dev) for r in range(4)]
        x = synth.activations(T, K, 17).to(dev)
        y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_gather_matmul(x, routes[i % 4], gp, gs, gb, G, BITS, out=y), 16, 20)
        wb = T * weight_bytes(K, N)
        gbs = wb / (ms * 1e-3) / 1e9
        res[f"tokens{tokens}_top2"] = {"rows": T, "us": round(ms * 1e3, 2), "weight_GBps": round(gbs, 1),
                                       "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    # prefill form: 4096 routed rows (2048 tokens, top-2) grouped by expert, one matmul per expert.
    # The call reads the per-expert counts on the host, so it is timed per call, not from a graph.
    T = 4096
    ex = torch.randint(0, E, (T,), dtype=torch.int32, device=dev, generator=torch.Generator(device=dev).manual_seed(8))
    x = synth.activations(T, K, 18).to(dev)
    y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(2):
            aq.aq_gather_matmul(x, ex, gp, gs, gb, G, BITS, out=y, grouped=True)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            aq.aq_gather_matmul(x, ex, gp, gs, gb, G, BITS, out=y, grouped=True)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 5
    tf = 2.0 * T * N * K / (ms * 1e-3) / 1e12
    res["prefill_grouped_4096_rows"] = {"rows": T, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                                        "frac_bf16_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                                        "note": "includes routing and the gather/scatter copies; one matmul launch over all experts, no host read"}
    return {"gather_qmv": {"E": E, "N": N, "K": K, "bits": BITS, "G": G, "points": res}}


def section_mxfp4(args, aq, torch, dev, stream, peaks):
    """mxfp4 decode (M = 1) on the integer tensor cores: weight GB/s (codes + E8M0
    scales, N*K/2 + N*K/32 bytes) over rotating resident copies, and the quantizer."""
    out = {}
    x_cache = {}
    for (K, N) in ((4096, 14336), (14336, 4096), (8192, 28672)):
        w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 6 + K % 7)).to(dev)
        base = aq.aq_mxfp4_quantize(w)
        if (K, N) == (8192, 28672):
            ms_q = timed_graph(torch, stream, lambda i: aq.aq_mxfp4_quantize(w), 1, 10)
            out["mxfp4_quantize"] = {"K": K, "N": N, "ms": round(ms_q, 4),
                                     "GBps": round((N * K * 4 + N * K // 2 + N * K // 32) / (ms_q * 1e-3) / 1e9, 1)}
        del w
        wb = N * K // 2 + N * K // 32
        copies = max(2, -(-2 * L2_BYTES // wb) + 1)
        qs = [base] + [tuple(t.clone() for t in base) for _ in range(copies - 1)]
        x = x_cache.setdefault(K, synth.activations(1, K, 17).to(dev))
        y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_mxfp4_matmul(x, *qs[i % copies], out=y, overlap_previous=True),
                         copies * 4, 20)
        gbs = wb / (ms * 1e-3) / 1e9
        out[f"mxfp4_qmv_K{K}_N{N}"] = {"us": round(ms * 1e3, 3), "weight_GBps": round(gbs, 1),
                                       "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                       "kernel": "qmv_tc_kernel<4,32,1,mxfp4> (mma.sync m16n8k32, codes split by sign)"}
        del qs, base
        torch.cuda.empty_cache()
    # mxfp8: E4M3 codes + E8M0 per 32 (bytes N*K + N*K/32), f16 MMAs
    for (K, N) in ((4096, 14336), (8192, 28672)):
        w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 6 + 5 + K % 7)).to(dev)
        base = aq.aq_mxfp8_quantize(w)
        del w
        wb = N * K + N * K // 32
        copies = max(2, -(-2 * L2_BYTES // wb) + 1)
        qs = [base] + [tuple(t.clone() for t in base) for _ in range(copies - 1)]
        x = x_cache.setdefault(K, synth.activations(1, K, 17).to(dev))
        y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_mxfp8_matmul(x, *qs[i % copies], out=y, overlap_previous=True),
                         copies * 4, 20)
        gbs = wb / (ms * 1e-3) / 1e9
        out[f"mxfp8_qmv_K{K}_N{N}"] = {"us": round(ms * 1e3, 3), "weight_GBps": round(gbs, 1),
                                       "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                       "kernel": "qmv_tc_kernel<8,32,1,mxfp8> (mma.sync m16n8k16 f16, E4M3 widened)"}
        del qs, base
        torch.cuda.empty_cache()
    # nvfp4: E4M3 scale per 16 + tensor scale (bytes N*K/2 + N*K/16)
    for (K, N) in ((4096, 14336), (8192, 28672)):
        w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 6 + 3 + K % 7)).to(dev)
        base = aq.aq_nvfp4_quantize(w)
        del w
        wb = N * K // 2 + N * K // 16
        copies = max(2, -(-2 * L2_BYTES // wb) + 1)
        qs = [base] + [tuple(t.clone() for t in base) for _ in range(copies - 1)]
        x = x_cache.setdefault(K, synth.activations(1, K, 17).to(dev))
        y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_nvfp4_matmul(x, *qs[i % copies], out=y, overlap_previous=True),
                         copies * 4, 20)
        gbs = wb / (ms * 1e-3) / 1e9
        out[f"nvfp4_qmv_K{K}_N{N}"] = {"us": round(ms * 1e3, 3), "weight_GBps": round(gbs, 1),
                                       "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                       "kernel": "qmv_tc_kernel<4,32,1,nvfp4> (two 16-groups per MMA K step)"}
        del qs, base
        torch.cuda.empty_cache()
    # prefill (M = 2048, K = 4096, N = 14336) of the three formats on the tcgen05 matmul
    M, K, N = 2048, 4096, 14336
    w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 6 + 9)).to(dev)
    x = synth.activations(M, K, 19).to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    for name, quant, call in (("mxfp4", aq.aq_mxfp4_quantize, aq.aq_mxfp4_matmul),
                              ("nvfp4", aq.aq_nvfp4_quantize, aq.aq_nvfp4_matmul),
                              ("mxfp8", aq.aq_mxfp8_quantize, aq.aq_mxfp8_matmul)):
        q = quant(w)
        ms = timed_graph(torch, stream, lambda i: call(x, *q, out=y), 2, 10)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[f"{name}_qmm_M{M}_K{K}_N{N}"] = {"us": round(ms * 1e3, 2), "TFLOP/s": round(tf, 1),
                                             "frac_of_burst": round(tf / peaks["bf16_tflops"], 4),
                                             "kernel": "qmm_pair_kernel (CTA pairs, tcgen05 kind::f16, codes dequantized to fp16)"}
        del q
    del w, x, y
    torch.cuda.empty_cache()
    return out


def section_embedding(args, aq, torch, dev, stream, peaks):
    """Quantized embedding lookup: 4096 random ids into a Llama-3-size table
    (V = 128256, D = 4096), 4-bit G = 32; bytes = rows read + bf16 rows written."""
    V, D, g, bits, T = 128256, 4096, 32, 4, 4096
    w = torch.randn((V, D), device=dev, dtype=torch.float32, generator=torch.Generator(device=dev).manual_seed(5)) * 0.02
    p, s, b = aq.aq_quantize(w, g, bits)
    del w
    torch.cuda.empty_cache()
    ids = torch.randint(0, V, (T,), device=dev, dtype=torch.int32, generator=torch.Generator(device=dev).manual_seed(6))
    o = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    ms = timed_graph(torch, stream, lambda i: aq.aq_embedding(ids, p, s, b, D, g, bits, out=o), 1, 20)
    nbytes = T * (D * bits // 8 + 4 * D // g) + T * D * 2
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"embedding": {"V": V, "D": D, "T": T, "bits": bits, "G": g, "us": round(ms * 1e3, 2),
                          "GBps": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}}


QMM_POINTS = [(M, K, N) for (K, N) in ((4096, 14336), (14336, 4096)) for M in (512, 2048, 8192)]


def section_qmm(args, aq, torch, dev, stream, peaks):
    """Prefill QMM (the tensor-core kernel) at every M x (K, N) point of the
    prefill workload: TFLOP/s (2*M*N*K per call) against the measured bf16
    dense peak (burst: the kernel is timed on its own, back to back)."""
    out = {}
    wcache = {}
    points = QMM_POINTS
    if args.qmm_points:
        want = {tuple(int(v) for v in t.split("x")) for t in args.qmm_points.split(",")}
        points = [pt for pt in QMM_POINTS if pt in want]
    for (M, K, N) in points:
        if (K, N) not in wcache:
            wcache.clear()
            torch.cuda.empty_cache()
            w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 5 + (0 if K == 4096 else 1))).to(dev)
            wcache[(K, N)] = aq.aq_quantize(w, G, BITS)
            del w
        p, s, b = wcache[(K, N)]
        x = synth.activations(M, K, 7).to(dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        reps = max(2, args.qmm_reps * 8192 // (4 * M))
        ms = timed_graph(torch, stream, lambda i: aq.aq_matmul(x, p, s, b, G, BITS, out=y), 2, reps)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        # the K split runs exactly when the workspace holds more than the activations' part
        act_bytes = -(-M * K * 2 // 256) * 256 + -(-M * 4 // 256) * 256
        out[f"M{M}_K{K}_N{N}"] = {"TFLOP/s": round(tf, 1), "us": round(ms * 1e3, 2),
                                  "frac_of_burst": round(tf / peaks["bf16_tflops"], 4),
                                  "frac_of_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                                  "k_split": aq.aq_matmul_workspace_bytes(M, N, K, G, BITS) > act_bytes}
        del x, y
    wcache.clear()
    torch.cuda.empty_cache()
    return {"qmm_prefill": {"bits": BITS, "G": G, "peak_burst": peaks["bf16_tflops"],
                            "peak_sustained": peaks["bf16_tflops_sustained"], "points": out,
                            "traffic": recorded_traffic("qmm_prefill")}}


def section_decode_shapes(args, aq, torch, dev, stream, peaks):
    """Each decode linear on its own (M = 1, 4-bit G64): back-to-back launches of
    that shape over rotating resident weight copies (larger than L2), each
    launched as a programmatic dependent of the one before, as in the step."""
    out = {}
    for si, (K, N) in enumerate(DECODE_SHAPES):
        w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 2 + si)).to(dev)
        base = aq.aq_quantize(w, G, BITS)
        del w
        wb = weight_bytes(K, N)
        copies = max(2, -(-2 * L2_BYTES // wb) + 1)
        ws = [base] + [tuple(t.clone() for t in base) for _ in range(copies - 1)]
        x = synth.activations(1, K, 1000 + 100 * 2 + si + 1).to(dev)
        y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_matmul(x, *ws[i % copies], G, BITS, out=y,
                                                               overlap_previous=True), copies * 8, 20)
        gbs = wb / (ms * 1e-3) / 1e9
        out[f"K{K}_N{N}"] = {"us": round(ms * 1e3, 3), "weight_GBps": round(gbs, 1),
                             "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
        del ws, base
        torch.cuda.empty_cache()
    return {"decode_shapes": out}


def section_decode_sequence(args, aq, torch, dev, stream, peaks):
    """The decode step's three linears as one aq_matmul_sequence launch (the
    weights of each linear stream while the one before finishes; a grid barrier
    before each linear's activations), against three launches, over rotating
    resident weight sets larger than L2."""
    base = []
    for si, (K, N) in enumerate(DECODE_SHAPES):
        w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 2 + si)).to(dev)
        base.append(aq.aq_quantize(w, G, BITS))
        del w
    copies = max(2, -(-2 * L2_BYTES // STEP_BYTES) + 1)
    out = {}
    for M in (1, 2, 4):
        sets = []
        for c in range(copies):
            sets.append([(tuple(t.clone() for t in base[si]) if c else base[si]) +
                         (synth.activations(M, K, 7 + si).to(dev), torch.empty((M, N), dtype=torch.bfloat16, device=dev))
                         for si, (K, N) in enumerate(DECODE_SHAPES)])

        def three(i):
            for (p, s, b, x, y) in sets[i % copies]:
                aq.aq_matmul(x, p, s, b, G, BITS, out=y, overlap_previous=True)

        def seq(i):
            aq.aq_matmul_sequence([(x, p, s, b, y) for (p, s, b, x, y) in sets[i % copies]], G, BITS,
                                  overlap_previous=True)
        for name, fn in (("three_launches", three), ("sequence", seq)):
            ms = timed_graph(torch, stream, fn, copies * 4, 10)
            out[f"M{M}_{name}"] = {"us": round(ms * 1e3, 2), "weight_GBps": round(STEP_BYTES / (ms * 1e-3) / 1e9, 1)}
        del sets
        torch.cuda.empty_cache()
    return {"decode_sequence": out}


def section_curve(args, aq, torch, dev, stream, peaks):
    out = {}
    # ---- QMV small-M curve on K=4096, N=14336 (rotating weight copies)
    K, N = 4096, 14336
    w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 3)).to(dev)
    base = aq.aq_quantize(w, G, BITS)
    del w
    wb = weight_bytes(K, N)
    copies = max(2, -(-2 * L2_BYTES // wb) + 1)
    ws = [base] + [tuple(t.clone() for t in base) for _ in range(copies - 1)]
    curve = {}
    for M in (1, 2, 3, 4, 5, 6, 8):
        x = synth.activations(M, K, 11).to(dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_matmul(x, *ws[i % copies], G, BITS, out=y,
                                                               overlap_previous=True), copies * 8, 50)
        curve[str(M)] = {"us": round(ms * 1e3, 3), "weight_GBps": round(wb / (ms * 1e-3) / 1e9, 1),
                         "frac_hbm": round(wb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                         "kernel": ["qmv", "qmm"][aq.aq_dispatch(M, N, K, G, BITS) - 1]}
    out["qmv_small_m"] = {"K": K, "N": N, "bits": BITS, "G": G, "curve": curve}
    del ws, base
    torch.cuda.empty_cache()
    # ---- the same curve at a long K (K=14336, N=4096: M > 4 runs as token chunks of one launch each)
    K, N = 14336, 4096
    w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 3 + 1)).to(dev)
    base = aq.aq_quantize(w, G, BITS)
    del w
    wb = weight_bytes(K, N)
    copies = max(2, -(-2 * L2_BYTES // wb) + 1)
    ws = [base] + [tuple(t.clone() for t in base) for _ in range(copies - 1)]
    curve = {}
    for M in (1, 2, 3, 4, 5, 6, 8):
        x = synth.activations(M, K, 12).to(dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ms = timed_graph(torch, stream, lambda i: aq.aq_matmul(x, *ws[i % copies], G, BITS, out=y,
                                                               overlap_previous=True), copies * 8, 20)
        curve[str(M)] = {"us": round(ms * 1e3, 3), "weight_GBps": round(wb / (ms * 1e-3) / 1e9, 1),
                         "frac_hbm": round(wb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    out["qmv_small_m_long_k"] = {"K": K, "N": N, "bits": BITS, "G": G, "curve": curve}
    del ws, base
    torch.cuda.empty_cache()
    return out


def section_sweep_quant(args, aq, torch, dev, stream, peaks, want):
    out = {}
    # ---- bits x group sweep at M=1 on K=8192, N=28672 (one point per bits, G=64 and the 4-bit G sweep)
    K, N = 8192, 28672
    w = torch.from_numpy(synth.weights(N, K, 1000 + 100 * 4)).to(dev)
    sweep = {}
    x = synth.activations(1, K, 13).to(dev)
    y = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
    for bits in ((2, 3, 4, 8) if "sweep" in want else ()):
        for g in (32, 64, 128):
            q = aq.aq_quantize(w, g, bits)
            wb = weight_bytes(K, N, g, bits)
            copies = max(2, -(-2 * L2_BYTES // wb) + 1)
            qs = [q] + [tuple(t.clone() for t in q) for _ in range(copies - 1)]
            ms = timed_graph(torch, stream, lambda i: aq.aq_matmul(x, *qs[i % copies], g, bits, out=y), copies * 4,
                             20)
            sweep[f"b{bits}_G{g}"] = {"us": round(ms * 1e3, 2), "weight_GBps": round(wb / (ms * 1e-3) / 1e9, 1),
                                      "frac_hbm": round(wb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
            del qs, q
            torch.cuda.empty_cache()
    if sweep:
        out["qmv_bits_group_sweep"] = {"K": K, "N": N, "M": 1, "points": sweep}
    if "quant" not in want:
        return out

    # ---- quantize and dequantize (bytes: read W fp32 + write packed/scales/biases; read packed + write bf16)
    p, s, b = aq.aq_quantize(w, G, BITS)
    ms_q = timed_graph(torch, stream, lambda i: aq.aq_quantize(w, G, BITS), 1, 10)
    qbytes = N * K * 4 + weight_bytes(K, N)
    dq = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    ms_d = timed_graph(torch, stream, lambda i: aq.aq_dequantize(p, s, b, K, G, BITS, out=dq), 1, 10)
    dbytes = weight_bytes(K, N) + N * K * 2
    out["quantize"] = {"K": K, "N": N, "bits": BITS, "G": G, "ms": round(ms_q, 4),
                       "GBps": round(qbytes / (ms_q * 1e-3) / 1e9, 1),
                       "frac_hbm": round(qbytes / (ms_q * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    out["dequantize_bf16"] = {"K": K, "N": N, "bits": BITS, "G": G, "ms": round(ms_d, 4),
                              "GBps": round(dbytes / (ms_d * 1e-3) / 1e9, 1),
                              "frac_hbm": round(dbytes / (ms_d * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    # ---- range-search quantize (32 candidate grids per group; ALU-bound, one-off)
    ms_m = timed_graph(torch, stream, lambda i: aq.aq_quantize_mse(w, G, BITS), 1, 3)
    out["quantize_mse"] = {"K": K, "N": N, "bits": BITS, "G": G, "candidates": 32, "ms": round(ms_m, 3),
                           "Gweights_per_s": round(N * K / (ms_m * 1e-3) / 1e9, 2),
                           "x_plain_quantize_time": round(ms_m / ms_q, 2)}
    return out


# ----------------------------------------------------------------------------- CPU oracle (baseline / reference arm)

def oracle_decode_inputs():
    import oracle
    ins = []
    for si, (K, N) in enumerate(DECODE_SHAPES):
        seed = 1000 + 100 * 2 + si
        p, s, b = oracle.quantize(synth.weights(N, K, seed), G, BITS)
        ins.append((synth.bf16_bits(synth.activations(1, K, seed + 1)), p, s, b))
    return ins


def time_oracle(ins, steps, budget_s):
    """Time decode steps of the oracle (plain C, fp64) on the host cores: at
    most `steps` steps and about budget_s seconds.  Returns (GB/s, steps, s)."""
    import oracle
    t0 = time.perf_counter()
    done = 0
    while done < steps:
        for (xb, p, s, b) in ins:
            oracle.matmul(xb, p, s, b, G, BITS)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return STEP_BYTES * done / dt / 1e9, done, dt


def cpu_baseline(budget_s):
    import oracle
    ins = oracle_decode_inputs()
    time_oracle(ins, 1, 0)  # warm
    gbs, done, dt = time_oracle(ins, 10 ** 6, budget_s)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done} full decode steps (all three linears at M=1) in {dt:.1f} s"}


def run_reference(args, rank, world):
    """The oracle arm: exactly --warmup then --steps timed steps on the host cores,
    each step a bounded sample of the decode workload: R consecutive output rows
    (rotating) of each of the three linears, computed by the oracle's sampled
    matmul over the real quantized weights.  R is sized from a calibration call so
    that all the steps fit in about --ref-budget seconds; the metric is weight
    bytes of the sampled rows per second."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    ins = oracle_decode_inputs()
    row_bytes = [K * BITS // 8 + 4 * K // G for K, N in DECODE_SHAPES]
    n_min = min(N for K, N in DECODE_SHAPES)

    def step(r0, R):
        for (xb, p, s, b), (K, N) in zip(ins, DECODE_SHAPES):
            oracle.matmul_sampled(xb, p, s, b, G, BITS, [0], (r0 + np.arange(R)) % N)

    step(0, 64)  # warm the caches and threads
    t0 = time.perf_counter()
    step(64, 64)
    per_row = (time.perf_counter() - t0) / 64
    total = args.warmup + args.steps
    R = int(max(1, min(n_min, args.ref_budget / max(total, 1) / per_row)))
    for i in range(args.warmup):
        step(i * R, R)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step((args.warmup + i) * R, R)
    dt = time.perf_counter() - t0
    step_bytes = R * sum(row_bytes)
    gbs = step_bytes * args.steps / dt / 1e9
    cores = min(oracle.num_threads(), R)
    sample = (f"{R} consecutive output rows (rotating) of each of the three linears per step, "
              f"{step_bytes} weight bytes per step; {args.steps} steps in {dt:.1f} s")
    return {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; shapes of Llama-3-8B linears; no checkpoints)",
            "config": {"workload": WORKLOAD, "M": 1, "bits": BITS, "G": G, "shapes_KN": DECODE_SHAPES,
                       "parallelism": "host cores (OpenMP over sampled rows)"},
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--qmm-reps", type=int, default=20)
    ap.add_argument("--qmm-points", default="",
                    help="comma list of MxKxN prefill points to run (default: every point of the prefill workload)")
    ap.add_argument("--sections", default="all",
                    help="all | none | comma list of shapes,seq,qmm,curve,sweep,quant,embed,gather,mxfp4 (secondary measurements)")
    ap.add_argument("--no-sections", dest="sections", action="store_const", const="none")
    ap.add_argument("--shard", action="store_true",
                    help="with N > 1 ranks: split W along N (one all-gather of y per step) instead of replicas")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="seconds of oracle work the reference arm's warm-up and timed steps aim at")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    pg = False
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        pg = True
    try:
        line, sections = run_ours(args, rank, world, local_rank)
        if rank == 0:
            line["cpu_baseline"] = cpu_baseline(args.cpu_budget)
            if sections:  # the detail, on a line of its own before the result line
                print(json.dumps({"sections": sections}), flush=True)
            print(json.dumps(line), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
