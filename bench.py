#!/usr/bin/env python
"""Benchmark of the MoE-layer hot path on B200.

Default workload: the 35B-A3B-class decode stack (hidden 2048, 256 routed
experts top-8 plus 1 shared expert, intermediate 512, 40 layers, MXFP4 weights
resident in HBM, batch 1), routed by seeded Zipf(1.1) traces with 0.6
adjacent-token reuse.  One step = one token through all 40 MoE layers
(the routing kernel and the persistent decode kernel: gate/up + SwiGLU,
down, combine for every layer), replayed as one CUDA graph.  Each step reads ~600 MB of distinct expert weights, far more than
the 126 MB L2, so no L2 flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line.  Multi-GPU runs are independent replicas (the path does
not shard): one process per GPU, timing = max over ranks, value = all tokens /
that time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE decode tok/s + HBM GB/s vs roofline; prefill FP4 TFLOP/s; miss H2D GB/s"
SEED = 1002


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--tokens", type=int, default=1, help="decode batch (1 to 16; the extras use 1 and 4)")
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary measurements")
    ap.add_argument("--case", default="decode",
                    choices=["decode", "prefill", "miss", "glm", "gemm", "router", "nvfp4", "dsv4"],
                    help="decode: the 35B-class decode stack (default line); prefill / miss / glm: only that "
                         "measurement; nvfp4: the NVFP4 prefill layer alone; dsv4: the DSV4-class decode stack "
                         "alone; gemm / router: the prefill GEMMs or router GEMV alone on a small case (the ncu "
                         "captures' workloads)")
    ap.add_argument("--layers", type=int, default=40, help="layers of the decode stack (40 = the full stack)")
    ap.add_argument("--layerwise", action="store_true",
                    help="decode with two kernels per layer instead of a persistent stack kernel")
    ap.add_argument("--format", default="mxfp4", choices=["mxfp4", "nvfp4", "bf16"],
                    help="expert weight format of the decode stack (and of --case gemm)")
    ap.add_argument("--counters", action="store_true",
                    help="decode with the counter-synchronised persistent kernel instead of the dataflow kernel")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# peaks, clocks
# ---------------------------------------------------------------------------
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, src="fallback")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every 10 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            pr = torch.cuda.get_device_properties(index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)
# ---------------------------------------------------------------------------
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The largest of the ranks' values (a device time): the job ends when the
    slowest replica does."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank_step, steps, ms_max, world):
    """Whole-job throughput of `world` independent replicas: every rank's
    units over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# 35B-class decode stack
# ---------------------------------------------------------------------------
H, I, E, K_TOP, S_SHARED, L = 2048, 512, 256, 8, 1, 40
TRACE_LEN = 512
# DRAM bytes (read + write) of the dataflow kernel k_dec_flow per algorithmic
# byte, from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum) of a
# 4-layer launch of this workload: 60,285,440 B read + 1,479,168 B written
# against 60,162,048 B.  The full 40-layer launch is too large to capture; its
# traffic grows with the layers.
STACK_TRAFFIC_PER_BYTE = (60285440 + 1479168) / 60162048


# The arithmetic of the decode GEMVs: MXFP4 and NVFP4 weights decode exactly
# to f16 and meet f16-encoded activations (x exact, h to 11 bits) in fused
# multiply-adds that accumulate in fp32; BF16 weights widen exactly to fp32
# and meet fp32 activations.
DECODE_DTYPE = {"mxfp4": "f16*f16+f32", "nvfp4": "f16*f16+f32", "bf16": "f32"}


def decode_routing(T):
    """Per token position p < TRACE_LEN: sets [L][T][k] of T independent sequences."""
    import numpy as np
    import synth
    sets = np.empty((TRACE_LEN, L, T, K_TOP), np.int32)
    for layer in range(L):
        for t in range(T):
            sets[:, layer, t] = synth.zipf_trace(SEED, layer, TRACE_LEN, E, K_TOP, 1.1, 0.6, stream=t)
    return sets


def decode_logits(sets):
    import numpy as np
    import synth
    P, Lx, T, _ = sets.shape
    out = np.empty((P, Lx, T, E), np.float32)
    for p in range(P):
        for layer in range(Lx):
            out[p, layer] = synth.logits_for_sets(SEED, p * 1000 + layer, sets[p, layer], E)
    return out


def run_ours(args, world, rank):
    import numpy as np
    import torch

    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu

    T = args.tokens
    fmt = getattr(args, "format", "mxfp4")
    fcode = {"mxfp4": ft.FT_FMT_MXFP4, "nvfp4": ft.FT_FMT_NVFP4, "bf16": ft.FT_FMT_BF16}[fmt]
    lay = ft.ft_blob_layout_format(H, I, fcode)
    used = lay["used"]
    gu_bytes = (lay["wd"] - lay["wg"]) + (lay["wd_sf"] - lay["wg_sf"])   # Wg + Wu codes and scales
    d_bytes = used - gu_bytes                                            # Wd codes, scales (and matrix scales)
    pools = [synth.gpu.layer_pool(H, I, E + S_SHARED, SEED, layer, fmt=fmt) for layer in range(L)]
    torch.cuda.synchronize()
    ctx = ft.ft_create(ft.make_desc(H, I, E, K_TOP, L, S_SHARED, 0, T, weight_format=fcode), None, pools)
    sets = decode_routing(T)
    logits_all = torch.from_numpy(decode_logits(sets)).cuda()        # [P][L][T][E]
    logits_buf = torch.empty_like(logits_all[0])
    xb = synth.activations_bf16(SEED, 7, T, H)
    x0 = torch.from_numpy(xb.view(np.int16).copy()).cuda().view(torch.bfloat16)
    # algorithmic bytes per step position: distinct routed experts + shared, whole blobs
    uniq = np.array([[len(np.unique(sets[p, layer])) for layer in range(L)] for p in range(TRACE_LEN)])
    bytes_pos = (uniq + S_SHARED).sum(axis=1) * used                 # [P]
    stream = torch.cuda.Stream()
    out_buf = torch.empty_like(x0)

    flags = ft.FT_ROUTE_RENORM | (ft.FT_STACK_LAYERWISE if args.layerwise else 0) | \
        (ft.FT_STACK_COUNTERS if getattr(args, "counters", False) else 0)

    def one_pass(src):
        ft.ft_moe_stack_forward(ctx, 0, L, src, T, logits_buf, out_buf, flags, stream.cuda_stream)
        return out_buf

    with torch.cuda.stream(stream):
        logits_buf.copy_(logits_all[0])
        one_pass(x0)
        stream.synchronize()
        ft.ft_sync_status(ctx, stream.cuda_stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            final = one_pass(x0)
    launches_per_step = stack_launches(T, args.layerwise, getattr(args, "counters", False), args.format)

    def step(p):
        logits_buf.copy_(logits_all[p % TRACE_LEN], non_blocking=True)
        g.replay()

    with torch.cuda.stream(stream):
        for w in range(args.warmup):
            step(w)
        stream.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as clk:
            e0.record(stream)
            for s in range(args.steps):
                step(args.warmup + s)
            e1.record(stream)
            e1.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        ms = e0.elapsed_time(e1)
    ft.ft_sync_status(ctx, stream.cuda_stream)
    ms_max = max_over_ranks(ms, world)
    positions = [(args.warmup + s) % TRACE_LEN for s in range(args.steps)]
    step_bytes = float(np.mean(bytes_pos[positions]))
    res = dict(ms=ms_max, tok_s=replica_throughput(T, args.steps, ms_max, world), hbm_gbs=step_bytes * args.steps / (ms / 1e3) / 1e9,
               step_bytes=step_bytes, launches=launches_per_step * args.steps, clocks=clk.summary())

    # per-kernel device time over the same positions: a graph of the same pass
    # with every kernel bracketed by events, replayed and read step by step
    ft.ft_kernel_timing_enable(ctx, True)
    nk = min(args.steps, 200)
    with torch.cuda.stream(stream):
        gt = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gt, stream=stream):
            one_pass(x0)
        stream.synchronize()
        for s in range(nk):
            logits_buf.copy_(logits_all[positions[s]], non_blocking=True)
            gt.replay()
            kt = ft.ft_kernel_timing_read(ctx)
    del gt
    ft.ft_kernel_timing_enable(ctx, False)
    pos = positions[:nk]
    gu_launch_bytes = float(np.mean([(uniq[p] + S_SHARED).mean() for p in pos])) * gu_bytes
    dn_launch_bytes = float(np.mean([(uniq[p] + S_SHARED).mean() for p in pos])) * d_bytes
    res["kernels"] = {k: {"ms_total": v[0], "launches": v[1], "us_avg": 1e3 * v[0] / v[1]} for k, v in kt.items() if v[1]}
    res["kernel_steps"] = nk
    res["gate_up_bytes"] = gu_launch_bytes
    res["down_bytes"] = dn_launch_bytes
    res["stack_bytes"] = float(np.mean(bytes_pos[pos]))  # every layer's routed + shared blobs

    # end to end through the C ABI with host buffers: H2D of the step's inputs
    # (x and the 40 layers' logits) from pinned memory, the pass, D2H of the output
    host_x = x0.cpu().pin_memory()
    host_lg = logits_all.cpu().pin_memory()
    host_out = torch.empty_like(host_x).pin_memory()
    xin = torch.empty_like(x0)
    with torch.cuda.stream(stream):
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            final2 = one_pass(xin)
        stream.synchronize()
        barrier(world)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for s in range(args.steps):
            p = positions[s]
            xin.copy_(host_x, non_blocking=True)
            logits_buf.copy_(host_lg[p], non_blocking=True)
            g2.replay()
            host_out.copy_(final2, non_blocking=True)
        a1.record(stream)
        a1.synchronize()
        barrier(world)
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), world)
    res["e2e"] = {"value": replica_throughput(T, args.steps, e2e_ms, world), "unit": "tok/s",
                  "h2d_bytes_per_step": int(host_x.numel() * 2 + host_lg[0].numel() * 4),
                  "d2h_bytes_per_step": int(host_out.numel() * 2)}
    del g, g2, final, final2
    ft.ft_destroy(ctx)
    del pools
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
def oracle_layer_times(T, n_layers, warm, budget_s, threads, distinct=4):
    """Time the C++ oracle (oracle/ft_oracle.cpp) on one token position of the
    40-layer stack, one layer per step, on `threads` OpenMP threads: the
    synthetic inputs (selected experts' blobs, logits) of `distinct` layers are
    generated first, outside any timed region; then `warm` untimed layers and
    up to `n_layers` timed layers cycle through them, stopping early once
    `budget_s` seconds of timed oracle work are done.  Returns (seconds per
    timed layer, threads used)."""
    import numpy as np
    import synth
    from oracle import cpp
    xb = synth.activations_bf16(SEED, 7, T, H)
    inputs = []
    for layer in range(distinct):
        sets = np.stack([synth.zipf_trace(SEED, layer, 4, E, K_TOP, 1.1, 0.6, stream=t)[-1] for t in range(T)])
        lg = synth.logits_for_sets(SEED, layer, sets, E)
        blobs = {int(e): synth.expert_blob(SEED, layer, int(e), H, I) for e in np.unique(sets)}
        blobs[E] = synth.expert_blob(SEED, layer, E, H, I)
        inputs.append((lg, blobs))
    times = []
    for i in range(warm + n_layers):
        lg, blobs = inputs[i % distinct]
        t0 = time.perf_counter()
        cpp.moe_layer(xb, blobs.__getitem__, H, I, E, K_TOP, logits=lg, shared_blob=blobs[E], threads=threads)
        dt = time.perf_counter() - t0
        if i >= warm:
            times.append(dt)
            if sum(times) > budget_s:
                break
    return times, threads


def oracle_tok_s(T, threads, budget_s=8.0, max_layers=12):
    """CPU baseline: tok/s of the C++ oracle over the 40-layer stack, from the
    mean of its timed layers (one warm-up layer); returns (tok/s, layers)."""
    times, _ = oracle_layer_times(T, max_layers, 1, budget_s, threads)
    return T / (statistics.mean(times) * L), len(times)


def host_cores():
    """Cores this process may run on (the OpenMP threads the oracle is given)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# secondary measurements: prefill FP4 GEMM throughput with double-buffered
# prefetch, expert-cache miss fetch bandwidth
# ---------------------------------------------------------------------------
FP4_DENSE_TFLOPS_NOMINAL = 9000.0   # B200 dense FP4 tensor peak, spec figure (quoted beside the measured one)
EV_HIT, EV_MISS = 0, 1               # cache event kinds of the C ABI


def miss_phases(events, per_token, phases):
    """Miss rate of each named token range [a, b) of a decode run, from the
    cache's event trace: the HIT/MISS lookups in order, per_token of them per
    token (batch 1: one per selected expert and layer).  Returns None when the
    trace does not hold exactly that many lookups."""
    look = [e[0] for e in events if e[0] in (EV_HIT, EV_MISS)]
    n_tok = max((b for _, (a, b) in phases), default=0)
    if len(look) != n_tok * per_token:
        return None
    out = {}
    for name, (a, b) in phases:
        seg = look[a * per_token:b * per_token]
        out[name] = sum(1 for k in seg if k == EV_MISS) / len(seg) if seg else None
    return out


def prefill_roofline(flops, weight_bytes, hbm_gbs, tflops, fp4_peak=FP4_DENSE_TFLOPS_NOMINAL):
    """The prefill GEMM against its own roofline: min(FP4 dense peak, HBM
    bandwidth x arithmetic intensity over the weight bytes it must read)."""
    ai = flops / weight_bytes
    roof = min(fp4_peak, hbm_gbs * ai / 1e3)
    return {"flop_per_weight_byte": ai, "roofline_tflops": roof, "frac_of_roofline": tflops / roof,
            "frac_of_fp4_peak": tflops / fp4_peak, "frac_of_fp4_nominal": tflops / FP4_DENSE_TFLOPS_NOMINAL,
            "bound": "hbm" if roof < fp4_peak else "tensor"}


def measure_fp4_peak(iters=16384, reps=7):
    """Dense FP4 tensor peak of this GPU: the library's tcgen05 kind::mxf4
    probe (one CTA per SM, operands in shared memory, M = N = 128, K = 64),
    timed by CUDA events per launch after two warm-up launches; the median
    launch, with the SM clocks sampled meanwhile."""
    import torch
    import expert_offloaded_serving_b200 as ft
    sink = torch.zeros(1024, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(2):
        grid = ft.ft_fp4_mma_probe(iters, sink, status, stream.cuda_stream)
    ms = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            grid = ft.ft_fp4_mma_probe(iters, sink, status, stream.cuda_stream)
            b.record(stream)
            b.synchronize()
            ms.append(a.elapsed_time(b))
    if int(status.item()) != 0:
        raise RuntimeError("FP4 probe: the wait for the tensor pipe gave up")
    flops = grid * iters * 4 * 2 * 128 * 128 * 64
    t = statistics.median(ms)
    return {"tflops": flops / (t * 1e-3) / 1e12, "ms": t, "ctas": grid, "iters": iters,
            "instruction": "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32, M = N = 128, K = 64",
            "clocks": clk.summary()}


def overlap_fraction(copy_ms, compute_ms, total_ms, hideable_ms):
    """Share of the hideable compute time that ran under the copies, when
    copies totalling copy_ms and computes totalling compute_ms took total_ms
    together (1: all hideable compute hidden, 0: serialised), clamped to
    [0, 1].  In a double-buffered run over n layers the first copy and the
    last layer's compute have nothing to overlap with, so hideable_ms is the
    compute of n - 1 layers."""
    if hideable_ms <= 0:
        return None
    return max(0.0, min(1.0, (copy_ms + compute_ms - total_ms) / hideable_ms))


def pinned_h2d_gbs(nbytes=1 << 30, reps=10):
    """Best-of-reps pinned host -> device copy bandwidth (GB/s)."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    best = 1e9
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        d.copy_(h, non_blocking=True)
        b.record()
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    del h, d
    return nbytes / (best / 1e3) / 1e9


def host_layer_pools(H, I, n_blobs, seed, layers):
    """Pinned host pools of `layers` layers, filled on the GPU and copied down."""
    import torch
    import synth.gpu
    stride = synth.blob_stride(H, I)
    pools = []
    for layer in range(layers):
        h = torch.empty(n_blobs * stride, dtype=torch.uint8).pin_memory()
        d = synth.gpu.layer_pool(H, I, n_blobs, seed, layer)
        h.copy_(d)
        del d
        pools.append(h)
    torch.cuda.synchronize()
    return pools


def measure_prefill(reps=3, layers=3):
    """DeepSeek-V4-Flash-class prefill: hidden 4096, 256 experts top-6,
    intermediate 2048, one 4096-token chunk, near-uniform routing through the
    router GEMV.  (a) GEMM throughput on a resident layer (kernel timers);
    (b) layers served from pinned host pools with double-buffered prefetch."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu
    H2, I2, E2, k2, T2, seed = 4096, 2048, 256, 6, 4096, 1004
    flops = 2.0 * T2 * k2 * 3 * H2 * I2
    pool = synth.gpu.layer_pool(H2, I2, E2, seed, 0)
    ctx = ft.ft_create(ft.make_desc(H2, I2, E2, k2, 1, 0, 0, T2), None, [pool])
    x = torch.from_numpy(synth.activations_bf16(seed, 1, T2, H2).view(np.int16).copy()).cuda().view(torch.bfloat16)
    wr = torch.from_numpy(synth.router_weights(seed, 0, E2, H2)).cuda()
    out = torch.empty_like(x)
    flags = ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM
    for _ in range(2):
        ft.ft_moe_layer_forward(ctx, 0, x, T2, wr, None, out, flags)
    torch.cuda.synchronize()
    ft.ft_kernel_timing_enable(ctx, True)
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, x, T2, wr, None, out, flags)
    kt = ft.ft_kernel_timing_read(ctx)
    ft.ft_kernel_timing_enable(ctx, False)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, x, T2, wr, None, out, flags)
    b.record()
    b.synchronize()
    layer_ms = a.elapsed_time(b) / reps
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    del pool
    torch.cuda.empty_cache()
    gemm_ms = (kt["gemm_gate_up"][0] + kt["gemm_down"][0]) / reps
    res = {"workload": "DSV4-class prefill layer: hidden 4096, 256 experts top-6, intermediate 2048, 4096 tokens",
           "flop_per_layer": flops, "gemm_ms": gemm_ms, "gemm_tflops": flops / (gemm_ms * 1e-3) / 1e12,
           "gate_up_ms": kt["gemm_gate_up"][0] / reps, "down_ms": kt["gemm_down"][0] / reps,
           "layer_ms_resident": layer_ms,
           "kernels_ms": {k: v[0] / reps for k, v in kt.items() if v[1]}}
    wbytes = E2 * ft.ft_blob_layout(H2, I2)["used"]
    res["gemm_weight_gbs"] = wbytes / (gemm_ms * 1e-3) / 1e9
    pk = peaks()
    fp4 = measure_fp4_peak()
    res["fp4_peak"] = fp4
    res["gemm_roofline"] = {**prefill_roofline(flops, wbytes, pk["hbm"], res["gemm_tflops"], fp4["tflops"]),
                            "hbm_peak_gbs": pk["hbm"], "hbm_peak_source": pk["src"],
                            "fp4_peak_tflops": fp4["tflops"], "fp4_peak_source": "measured (tcgen05 mxf4 probe)",
                            "fp4_nominal_tflops": FP4_DENSE_TFLOPS_NOMINAL}
    res["calibration"] = measure_prefill_calibration(fp4["tflops"])
    res["nvfp4"] = measure_prefill_nvfp4(fp4["tflops"], pk)
    # (b) pinned host pools, double-buffered prefetch
    hp = host_layer_pools(H2, I2, E2, seed, layers)
    ctx = ft.ft_create(ft.make_desc(H2, I2, E2, k2, layers, 0, 0, T2), hp, None)
    torch.cuda.synchronize()
    a.record()
    ft.ft_prefetch_layer(ctx, 0)
    for l in range(layers):
        if l + 1 < layers:
            ft.ft_prefetch_layer(ctx, l + 1)
        ft.ft_moe_layer_forward(ctx, l, x, T2, wr, None, out, flags)
    b.record()
    b.synchronize()
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    pack = E2 * ft.ft_blob_stride(H2, I2)
    res["prefetch_layers"] = layers
    res["layer_ms_prefetched"] = a.elapsed_time(b) / layers
    res["prefetch_h2d_gbs"] = pack * layers / (a.elapsed_time(b) * 1e-3) / 1e9
    del hp
    # overlap: each layer's copy alone at the measured pinned H2D rate and the
    # resident layer's compute, against the prefetched run's time
    h2d = pinned_h2d_gbs()
    copy_ms = pack / (h2d * 1e9) * 1e3
    res["pinned_h2d_gbs"] = h2d
    res["copy_ms_per_layer_at_pinned"] = copy_ms
    res["compute_hidden_frac"] = overlap_fraction(layers * copy_ms, layers * layer_ms, a.elapsed_time(b),
                                                  (layers - 1) * layer_ms)
    return res


def host_pools_pageable(H, I, n_blobs, seed, layers):
    """Host pools of `layers` layers in ordinary (pageable) host memory, filled
    on the GPU by the seeded filler and copied down; ft_create pins them
    (cudaHostRegister) without copying.  Pageable numpy buffers avoid the
    power-of-two rounding of torch's pinned allocator at these sizes."""
    import numpy as np
    import torch
    import synth.gpu
    stride = synth.blob_stride(H, I)
    pools = []
    for layer in range(layers):
        h = np.empty(n_blobs * stride, np.uint8)
        d = synth.gpu.layer_pool(H, I, n_blobs, seed, layer)
        torch.from_numpy(h).copy_(d)
        del d
        pools.append(h)
    torch.cuda.synchronize()
    return pools


def available_host_bytes():
    try:
        import psutil
        return psutil.virtual_memory().available
    except Exception:
        return os.sysconf("SC_AVPHYS_PAGES") * os.sysconf("SC_PAGE_SIZE")


def measure_prefill_nvfp4(fp4_peak, pk, reps=3):
    """The DSV4-class prefill layer with NVFP4 experts (E4M3 scales per 16,
    fp32 matrix scales) through FT_ACT_NVFP4: x and h quantised to NVFP4,
    tcgen05 kind::mxf4nvf4 grouped GEMMs; 4096 tokens through the router
    GEMV.  GEMM TFLOP/s from the kernel timers against the layer's roofline
    (its NVFP4 weight bytes at the HBM rate; the tensor peak is the measured
    kind::mxf4 one, the same nominal rate)."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu
    H2, I2, E2, k2, T2, seed = 4096, 2048, 256, 6, 4096, 1006
    flops = 2.0 * T2 * k2 * 3 * H2 * I2
    pool = synth.gpu.layer_pool(H2, I2, E2, seed, 0, fmt="nvfp4")
    ctx = ft.ft_create(ft.make_desc(H2, I2, E2, k2, 1, 0, 0, T2, weight_format=ft.FT_FMT_NVFP4), None, [pool])
    x = torch.from_numpy(synth.activations_bf16(seed, 1, T2, H2).view(np.int16).copy()).cuda().view(torch.bfloat16)
    wr = torch.from_numpy(synth.router_weights(seed, 0, E2, H2)).cuda()
    out = torch.empty_like(x)
    flags = ft.FT_ACT_NVFP4 | ft.FT_ROUTE_RENORM
    for _ in range(2):
        ft.ft_moe_layer_forward(ctx, 0, x, T2, wr, None, out, flags)
    torch.cuda.synchronize()
    ft.ft_kernel_timing_enable(ctx, True)
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, x, T2, wr, None, out, flags)
    kt = ft.ft_kernel_timing_read(ctx)
    ft.ft_kernel_timing_enable(ctx, False)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, x, T2, wr, None, out, flags)
    b.record()
    b.synchronize()
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    del pool
    torch.cuda.empty_cache()
    gemm_ms = (kt["gemm_gate_up"][0] + kt["gemm_down"][0]) / reps
    tflops = flops / (gemm_ms * 1e-3) / 1e12
    wbytes = E2 * ft.ft_blob_layout_format(H2, I2, ft.FT_FMT_NVFP4)["used"]
    return {"workload": "DSV4-class prefill layer with NVFP4 experts: hidden 4096, 256 experts top-6, "
                        "intermediate 2048, 4096 tokens",
            "gemm_ms": gemm_ms, "gemm_tflops": tflops, "gate_up_ms": kt["gemm_gate_up"][0] / reps,
            "down_ms": kt["gemm_down"][0] / reps, "layer_ms_resident": a.elapsed_time(b) / reps,
            "kernels_ms": {k: v[0] / reps for k, v in kt.items() if v[1]},
            "gemm_weight_gbs": wbytes / (gemm_ms * 1e-3) / 1e9,
            "gemm_roofline": {**prefill_roofline(flops, wbytes, pk["hbm"], tflops, fp4_peak),
                              "hbm_peak_gbs": pk["hbm"], "hbm_peak_source": pk["src"]}}


def measure_prefill_calibration(fp4_peak, T=65536, reps=2):
    """The compute-bound calibration shape of the prefill GEMMs: the
    DSV4-class layer (hidden 4096, 256 experts top-6, intermediate 2048) on a
    65,536-token chunk, 1,536 tokens per expert on average (arithmetic
    intensity ~5.8k FLOP per weight byte, above the HBM / FP4 ridge), through
    the same path; GEMM TFLOP/s from the kernel timers against the measured
    FP4 peak.  Not a workload of its own: it shows the GEMM where the tensor
    pipe, not HBM, bounds it."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu
    H2, I2, E2, k2, seed = 4096, 2048, 256, 6, 1005
    flops = 2.0 * T * k2 * 3 * H2 * I2
    pool = synth.gpu.layer_pool(H2, I2, E2, seed, 0)
    ctx = ft.ft_create(ft.make_desc(H2, I2, E2, k2, 1, 0, 0, T), None, [pool])
    x = torch.from_numpy(synth.activations_bf16(seed, 1, T, H2).view(np.int16).copy()).cuda().view(torch.bfloat16)
    lg = torch.from_numpy(synth.logits_for_sets(seed, 3, synth.near_uniform_sets(seed, 0, T, E2, k2), E2)).cuda()
    out = torch.empty_like(x)
    flags = ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM
    ft.ft_moe_layer_forward(ctx, 0, x, T, None, lg, out, flags)
    torch.cuda.synchronize()
    ft.ft_kernel_timing_enable(ctx, True)
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, x, T, None, lg, out, flags)
    kt = ft.ft_kernel_timing_read(ctx)
    ft.ft_kernel_timing_enable(ctx, False)
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    del pool, x, out, lg
    torch.cuda.empty_cache()
    gemm_ms = (kt["gemm_gate_up"][0] + kt["gemm_down"][0]) / reps
    tf = flops / (gemm_ms * 1e-3) / 1e12
    return {"workload": f"DSV4-class prefill GEMMs, {T} tokens top-{k2} over {E2} experts ({T * k2 // E2} tokens "
                        "per expert on average)",
            "flop": flops, "gemm_ms": gemm_ms, "gemm_tflops": tf, "frac_of_fp4_peak": tf / fp4_peak,
            "gate_up_ms": kt["gemm_gate_up"][0] / reps, "down_ms": kt["gemm_down"][0] / reps}


def measure_gemm_small(reps=2, T=16384, E2=64, fmt="mxfp4"):
    """The prefill GEMMs at the calibration case's 1,536 tokens per expert on
    a small pool: the DSV4-class expert shape (hidden 4096, intermediate
    2048, top-6) with 64 experts and 16,384 tokens (0.8 GB of experts), one
    warm forward and `reps` timed ones through the MXFP4-activation path
    (fmt "nvfp4": NVFP4 experts through the NVFP4-activation path).  The
    workload of the GEMMs' ncu captures (a few GB on the device)."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu
    H2, I2, k2, seed = 4096, 2048, 6, 1005
    if fmt not in ("mxfp4", "nvfp4"):
        raise SystemExit("--case gemm takes --format mxfp4 or nvfp4 (the prefill path has no BF16 experts)")
    nv = fmt == "nvfp4"
    pool = synth.gpu.layer_pool(H2, I2, E2, seed, 0, fmt=fmt)
    ctx = ft.ft_create(ft.make_desc(H2, I2, E2, k2, 1, 0, 0, T,
                                    weight_format=ft.FT_FMT_NVFP4 if nv else ft.FT_FMT_MXFP4), None, [pool])
    x = torch.from_numpy(synth.activations_bf16(seed, 1, T, H2).view(np.int16).copy()).cuda().view(torch.bfloat16)
    lg = torch.from_numpy(synth.logits_for_sets(seed, 3, synth.near_uniform_sets(seed, 0, T, E2, k2), E2)).cuda()
    out = torch.empty_like(x)
    flags = (ft.FT_ACT_NVFP4 if nv else ft.FT_ACT_MXFP4) | ft.FT_ROUTE_RENORM
    ft.ft_moe_layer_forward(ctx, 0, x, T, None, lg, out, flags)
    torch.cuda.synchronize()
    ft.ft_kernel_timing_enable(ctx, True)
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, x, T, None, lg, out, flags)
    kt = ft.ft_kernel_timing_read(ctx)
    ft.ft_kernel_timing_enable(ctx, False)
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    gemm_ms = (kt["gemm_gate_up"][0] + kt["gemm_down"][0]) / reps
    flops = 2.0 * T * k2 * 3 * H2 * I2
    return {"workload": f"DSV4-shape prefill GEMMs, {E2} {fmt.upper()} experts, {T} tokens top-{k2} "
                        f"({T * k2 // E2} per expert)",
            "gemm_ms": gemm_ms, "gemm_tflops": flops / (gemm_ms * 1e-3) / 1e12,
            "gate_up_ms": kt["gemm_gate_up"][0] / reps, "down_ms": kt["gemm_down"][0] / reps}


def measure_router(reps=5, T=4096, H2=4096, E2=256):
    """The router GEMV of the DSV4-class prefill layer alone (4096 tokens x
    256 experts x hidden 4096, fp64 fixed order), through ft_router_logits:
    one warm call and `reps` timed ones.  The workload of its ncu capture."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    ctx = ft.ft_create(ft.make_desc(H2, 2048, E2, 6, 1, 0, 0, T))
    x = torch.from_numpy(synth.activations_bf16(1, 1, T, H2).view(np.int16).copy()).cuda().view(torch.bfloat16)
    wr = torch.from_numpy(synth.router_weights(1, 0, E2, H2)).cuda()
    lg = torch.empty((T, E2), dtype=torch.float32, device="cuda")
    ft.ft_router_logits(ctx, x, T, H2, wr, E2, lg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        ft.ft_router_logits(ctx, x, T, H2, wr, E2, lg)
    e1.record()
    torch.cuda.synchronize()
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    ms = e0.elapsed_time(e1) / reps
    return {"workload": f"router logits, {T} tokens x {E2} experts x hidden {H2}, fp64 fixed order",
            "ms": ms, "fp64_fma_per_s": T * E2 * H2 / (ms * 1e-3)}


def measure_misses(tokens=512, layers=43, resize_at=(170, 340)):
    """DeepSeek-V4-Flash-class decode over a GPU LRU expert cache (hidden
    4096, 256 experts top-6, intermediate 2048): `layers` layers (43 = the
    model) with their full pools in host memory pinned by the context, a
    32 GiB cache budget (2570 slots) halved at token 170 and restored at token
    340, batch 1 over a 512-token Zipf(1.0) trace with 0.5 adjacent reuse.
    The run goes twice on fresh contexts with the same trace (the same LRU
    events and copies): the default order, where the resident experts run
    while the misses' copies are in flight and each missed expert after its
    own copy, and FT_CACHE_SERIAL, where every copy lands first.  When the
    host cannot hold the full pool, the largest layer count that fits runs
    and the budget keeps its 32 GiB share of those layers (stated in the
    workload); tok/s is measured, never extrapolated."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    H3, I3, E3, k3, seed = 4096, 2048, 256, 6, 1003
    stride = ft.ft_blob_stride(H3, I3)
    pool_bytes = E3 * stride
    fit = int((available_host_bytes() - 24e9) // pool_bytes)
    L3 = max(1, min(layers, fit))
    budget = int(32 * 2 ** 30 * L3 / layers) // stride * stride
    hp = host_pools_pageable(H3, I3, E3, seed, L3)
    h2d_peak = pinned_h2d_gbs()
    sets = np.stack([synth.zipf_trace(seed, l, tokens, E3, k3, 1.0, 0.5) for l in range(L3)], axis=1)
    lg = torch.from_numpy(np.stack([[synth.logits_for_sets(seed, p * 100 + l, sets[p, l][None], E3)[0]
                                     for l in range(L3)] for p in range(tokens)])).cuda()
    x = torch.from_numpy(synth.activations_bf16(seed, 1, 1, H3).view(np.int16).copy()).cuda().view(torch.bfloat16)
    bufs = [torch.empty_like(x), torch.empty_like(x)]

    # one context (pinning the pool once); the second run starts from a cold
    # cache again: a resize to 0 evicts every expert, the next restores the budget
    ctx = ft.ft_create(ft.make_desc(H3, I3, E3, k3, L3, 0, budget, 1), hp, None)

    def run(flags, prefetch=0):
        ft.ft_expert_cache_resize(ctx, 0)
        ft.ft_expert_cache_resize(ctx, budget)
        ft.ft_cache_prefetch(ctx, prefetch)
        ft.ft_cache_trace(ctx, cap=1 << 22)
        ft.ft_cache_stats_get(ctx, reset=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        cur = x
        for p in range(tokens):
            if p == resize_at[0]:
                ft.ft_expert_cache_resize(ctx, budget // 2 // stride * stride)
            if p == resize_at[1]:
                ft.ft_expert_cache_resize(ctx, budget)
            for l in range(L3):
                nxt = bufs[(p * L3 + l) % 2]
                ft.ft_moe_layer_forward(ctx, l, cur, 1, None, lg[p, l], nxt, flags)
                cur = nxt
        b.record()
        b.synchronize()
        st = ft.ft_cache_stats_get(ctx)
        ev = ft.ft_cache_trace(ctx, cap=1 << 22)
        ft.ft_sync_status(ctx)
        return a.elapsed_time(b), st, ev

    total_ms, st, ev = run(ft.FT_ROUTE_RENORM)
    serial_ms, st_s, _ = run(ft.FT_ROUTE_RENORM | ft.FT_CACHE_SERIAL)
    pf = {n: run(ft.FT_ROUTE_RENORM, prefetch=n)[:2] for n in (1, 2)}
    ft.ft_destroy(ctx)
    del hp
    lookups = st["hits"] + st["misses"]
    miss_gbs = st["h2d_bytes"] / (st["h2d_ms"] * 1e-3) / 1e9 if st["h2d_ms"] > 0 else None
    phases = miss_phases(ev, L3 * k3, [("cold_first_token", (0, 1)), ("warm_full_budget", (1, resize_at[0])),
                                       ("half_budget", resize_at), ("restored_budget", (resize_at[1], tokens))])
    return {"workload": f"DSV4-class decode with expert cache: {L3} of {layers} layers, "
                        f"{L3 * pool_bytes / 1e9:.1f} GB pool in pinned host memory, budget "
                        f"{budget / 2 ** 30:.2f} GiB ({budget // stride} slots) halved at token {resize_at[0]} and "
                        f"restored at token {resize_at[1]}, batch 1, {tokens} tokens",
            "layers": L3, "tokens": tokens, "host_bytes_available": available_host_bytes(),
            "tok_s": tokens / (total_ms * 1e-3), "ms": total_ms,
            "miss_rate": st["misses"] / max(lookups, 1), "miss_rate_by_phase": phases,
            "hits": st["hits"], "misses": st["misses"], "evictions": st["evictions"], "moves": st["moves"],
            "miss_h2d_gbs": miss_gbs, "pinned_h2d_gbs": h2d_peak,
            "miss_h2d_frac": (miss_gbs / h2d_peak) if miss_gbs else None,
            "copy_busy_share": st["h2d_ms"] / total_ms if total_ms > 0 else None,
            # the resident experts' kernels of steps with misses, and the part of
            # them that ran while those steps' copies were in flight
            "overlap": {"resident_expert_ms": st["hit_ms"], "under_copies_ms": st["overlap_ms"],
                        "frac_of_resident_compute_hidden": st["overlap_ms"] / st["hit_ms"] if st["hit_ms"] else None,
                        "serial_order_tok_s": tokens / (serial_ms * 1e-3),
                        "saved_ms": serial_ms - total_ms},
            # the same trace with decode-time next-layer prefetch (1 and 2 per
            # layer step); the copies share the PCIe link with the misses
            "prefetch": [{"per_layer": n, "tok_s": tokens / (ms * 1e-3), "prefetches": sp["prefetches"],
                          "prefetch_hits": sp["prefetch_hits"],
                          "hit_rate": sp["prefetch_hits"] / sp["prefetches"] if sp["prefetches"] else None,
                          "miss_rate": sp["misses"] / max(sp["hits"] + sp["misses"], 1),
                          "h2d_bytes": sp["h2d_bytes"], "gain_vs_default": total_ms / ms - 1.0}
                         for n, (ms, sp) in pf.items()]}


def measure_decode_formats(args, pk, steps=300, warmup=20):
    """The same 35B-class decode stack at batch 1 with NVFP4 and with BF16
    experts (the pages' other formats of this model): tokens/s, the
    persistent kernel's bandwidth on the format's algorithmic bytes (whole
    blobs of the routed and shared experts) and its fraction of the HBM
    peak."""
    import copy
    out = {}
    for fmt in ("nvfp4", "bf16"):
        a = copy.copy(args)
        a.tokens, a.format, a.steps, a.warmup = 1, fmt, steps, warmup
        res = run_ours(a, 1, 0)
        o = {"workload": workload_config(1, fmt=fmt)["workload"], "tok_s": res["tok_s"], "ms_per_step": res["ms"] / steps,
             "e2e_tok_s": res["e2e"]["value"], "algorithmic_bytes_per_step": res["stack_bytes"], "clocks": res["clocks"]}
        st = res["kernels"].get("dec_stack")
        if st:
            gbs = res["stack_bytes"] / (st["us_avg"] * 1e-6) / 1e9
            o.update(kernel_us=st["us_avg"], kernel_gbs=gbs, kernel_frac=gbs / pk["hbm"])
        out[fmt] = o
    return out


def measure_glm(tokens=256, layers=8, prefill_tokens=2048, reps=3):
    """GLM-5.2-class slice (hidden 6144, 256 experts top-8, intermediate
    2048, 20 MB blobs): 8 of the 78 layers with their pools (41 GB) in pinned
    host memory, a 24 GiB cache (1285 slots), batch-1 decode over a 256-token
    Zipf(1.1) / 0.6-overlap trace through the cache path (tok/s, miss rate,
    miss H2D GB/s); and one 2048-token prefill chunk of a resident layer (GEMM
    TFLOP/s and layer time)."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu
    H5, I5, E5, k5, seed = 6144, 2048, 256, 8, 1006
    stride = ft.ft_blob_stride(H5, I5)
    budget = (24 * 2 ** 30) // stride * stride
    hp = host_pools_pageable(H5, I5, E5, seed, layers)
    sets = np.stack([synth.zipf_trace(seed, l, tokens, E5, k5, 1.1, 0.6) for l in range(layers)], axis=1)
    lg = torch.from_numpy(np.stack([[synth.logits_for_sets(seed, p * 100 + l, sets[p, l][None], E5)[0]
                                     for l in range(layers)] for p in range(tokens)])).cuda()
    x = torch.from_numpy(synth.activations_bf16(seed, 1, 1, H5).view(np.int16).copy()).cuda().view(torch.bfloat16)
    bufs = [torch.empty_like(x), torch.empty_like(x)]
    ctx = ft.ft_create(ft.make_desc(H5, I5, E5, k5, layers, 0, budget, 1), hp, None)
    ft.ft_cache_stats_get(ctx, reset=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    cur = x
    for p in range(tokens):
        for l in range(layers):
            nxt = bufs[(p * layers + l) % 2]
            ft.ft_moe_layer_forward(ctx, l, cur, 1, None, lg[p, l], nxt, ft.FT_ROUTE_RENORM)
            cur = nxt
    b.record()
    b.synchronize()
    st = ft.ft_cache_stats_get(ctx)
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    del hp
    ms = a.elapsed_time(b)
    lookups = st["hits"] + st["misses"]
    dec = {"workload": f"GLM-class decode: {layers} of 78 layers, {layers * E5 * stride / 1e9:.1f} GB pool in pinned "
                       f"host memory, 24 GiB cache ({budget // stride} slots), batch 1, {tokens} tokens",
           "tok_s_over_these_layers": tokens / (ms * 1e-3), "ms": ms, "miss_rate": st["misses"] / max(lookups, 1),
           "hits": st["hits"], "misses": st["misses"], "evictions": st["evictions"],
           "miss_h2d_gbs": st["h2d_bytes"] / (st["h2d_ms"] * 1e-3) / 1e9 if st["h2d_ms"] > 0 else None,
           "overlap": {"resident_expert_ms": st["hit_ms"], "under_copies_ms": st["overlap_ms"]}}
    # prefill: one resident layer, one 2048-token chunk through the router GEMV
    T = prefill_tokens
    pool = synth.gpu.layer_pool(H5, I5, E5, seed, 0)
    ctx = ft.ft_create(ft.make_desc(H5, I5, E5, k5, 1, 0, 0, T), None, [pool])
    xp = torch.from_numpy(synth.activations_bf16(seed, 2, T, H5).view(np.int16).copy()).cuda().view(torch.bfloat16)
    wr = torch.from_numpy(synth.router_weights(seed, 0, E5, H5)).cuda()
    out = torch.empty_like(xp)
    flags = ft.FT_ACT_MXFP4 | ft.FT_ROUTE_RENORM
    ft.ft_moe_layer_forward(ctx, 0, xp, T, wr, None, out, flags)
    torch.cuda.synchronize()
    ft.ft_kernel_timing_enable(ctx, True)
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, xp, T, wr, None, out, flags)
    kt = ft.ft_kernel_timing_read(ctx)
    ft.ft_kernel_timing_enable(ctx, False)
    a.record()
    for _ in range(reps):
        ft.ft_moe_layer_forward(ctx, 0, xp, T, wr, None, out, flags)
    b.record()
    b.synchronize()
    ft.ft_sync_status(ctx)
    ft.ft_destroy(ctx)
    del pool
    torch.cuda.empty_cache()
    flops = 2.0 * T * k5 * 3 * H5 * I5
    gemm_ms = (kt["gemm_gate_up"][0] + kt["gemm_down"][0]) / reps
    pre = {"workload": f"GLM-class prefill layer: {T} tokens, router GEMV, weights resident", "flop": flops,
           "gemm_ms": gemm_ms, "gemm_tflops": flops / (gemm_ms * 1e-3) / 1e12, "layer_ms": a.elapsed_time(b) / reps,
           "kernels_ms": {k_: v[0] / reps for k_, v in kt.items() if v[1]},
           "gemm_weight_gbs": E5 * ft.ft_blob_layout(H5, I5)["used"] / (gemm_ms * 1e-3) / 1e9}
    return {"decode": dec, "prefill": pre}


def measure_decode_dsv4(pk, n_layers=8, n_pos=64, reps=200):
    """The decode stack at another shape, through the dataflow kernel's build
    for any shape: DSV4-class layers (hidden 4096, 256 experts top-6,
    intermediate 2048, no shared expert), `n_layers` of them resident in HBM
    (27 GB at 8), batch 1, Zipf(1.1) / 0.6-reuse traces of `n_pos` positions.
    Time per token from events around `reps` stacked passes (not replayed as
    a graph); the persistent kernel's time from the kernel timers of a second
    run; HBM fraction of the distinct experts' blob bytes per token."""
    import numpy as np
    import torch
    import expert_offloaded_serving_b200 as ft
    import synth
    import synth.gpu
    H2, I2, E2, k2, seed = 4096, 2048, 256, 6, 1007
    pools = [synth.gpu.layer_pool(H2, I2, E2, seed, layer) for layer in range(n_layers)]
    ctx = ft.ft_create(ft.make_desc(H2, I2, E2, k2, n_layers, 0, 0, 1), None, pools)
    try:
        sets = np.stack([synth.zipf_trace(seed, layer, n_pos, E2, k2, 1.1, 0.6) for layer in range(n_layers)],
                        axis=1)                                                   # [P][L][k]
        lg = np.stack([np.stack([synth.logits_for_sets(seed, p * 1000 + layer, sets[p, layer][None], E2)
                                 for layer in range(n_layers)]) for p in range(n_pos)])   # [P][L][1][E]
        lgd = torch.from_numpy(lg).cuda()
        x = torch.from_numpy(synth.activations_bf16(seed, 1, 1, H2).view(np.int16).copy()).cuda().view(torch.bfloat16)
        out = torch.empty_like(x)
        used = ft.ft_blob_layout(H2, I2)["used"]
        step_bytes = np.array([sum(len(np.unique(sets[p, layer])) for layer in range(n_layers)) * used
                               for p in range(n_pos)], np.float64)
        flags = ft.FT_ROUTE_RENORM

        def run(n):
            for s in range(n):
                ft.ft_moe_stack_forward(ctx, 0, n_layers, x, 1, lgd[s % n_pos], out, flags)
        run(3)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as clk:
            a.record()
            run(reps)
            b.record()
            b.synchronize()
        ms = a.elapsed_time(b) / reps
        ft.ft_kernel_timing_enable(ctx, True)
        run(reps)
        kt = ft.ft_kernel_timing_read(ctx)
        ft.ft_kernel_timing_enable(ctx, False)
        ft.ft_sync_status(ctx)
    finally:
        ft.ft_destroy(ctx)
    del pools
    torch.cuda.empty_cache()
    kernel_us = 1e3 * kt["dec_stack"][0] / reps
    mean_bytes = float(step_bytes[np.arange(reps) % n_pos].mean())
    gbs = mean_bytes / (kernel_us * 1e-6) / 1e9
    return {"workload": f"DSV4-class decode stack: hidden {H2}, {E2} experts top-{k2}, intermediate {I2}, "
                        f"{n_layers} layers resident in HBM, batch 1, Zipf(1.1) routing traces with 0.6 "
                        f"adjacent-token reuse",
            "decode_kernels": decode_kernel_name_shape(H2, I2, E2, k2, 0, n_layers, 1),
            "ms_per_token_over_these_layers": ms, "us_per_layer": 1e3 * ms / n_layers,
            "kernel_us": kernel_us, "algorithmic_bytes_per_token": mean_bytes, "kernel_gbs": gbs,
            "kernel_frac": gbs / pk["hbm"], "clocks": clk.summary()}


def decode_kernel_name_shape(H2, I2, E2, k2, S2, L2, T):
    """The stacked-decode kernel for another shape (MXFP4, no flags)."""
    import expert_offloaded_serving_b200 as ft
    if ft.ft_flow_geometry(H2, I2, min(T, 2), k2, S2, E2, L2, ft.FT_FMT_MXFP4)["ok"] and T <= 4:
        return "persistent stack kernel, dataflow (tagged hand-overs), the build for any shape"
    return "persistent stack kernel, counter-synchronised"


def measure_decode_batch(args, T, pk):
    """The same 35B-class decode stack at batch T (the workload's other batch
    size): tokens/s, ms per step, end-to-end tokens/s and the persistent
    kernel's bandwidth on its algorithmic bytes (the union of the batch's
    experts and the shared one per layer)."""
    import copy
    a = copy.copy(args)
    a.tokens = T
    res = run_ours(a, 1, 0)
    out = {"workload": workload_config(T)["workload"], "tok_s": res["tok_s"], "ms_per_step": res["ms"] / a.steps,
           "e2e_tok_s": res["e2e"]["value"], "algorithmic_bytes_per_step": res["stack_bytes"],
           "clocks": res["clocks"]}
    st = res["kernels"].get("dec_stack")
    if st:
        # persistent-kernel time per step (a step runs one launch per wave)
        us = 1e3 * st["ms_total"] / res["kernel_steps"]
        gbs = res["stack_bytes"] / (us * 1e-6) / 1e9
        out.update(kernel_us=us, kernel_gbs=gbs, kernel_frac=gbs / pk["hbm"])
    return out


def _stack_path(T, layerwise=False, counters=False, fmt="mxfp4"):
    """The path ft_moe_stack_forward takes for a batch of T: ("flow", waves)
    when the dataflow kernel's geometry takes the stack (one launch for up to
    two tokens, waves of two for three or four), ("counters", 1) for the
    counter-synchronised kernel (MXFP4 only), else ("layerwise", 0)."""
    import expert_offloaded_serving_b200 as ft
    if layerwise:
        return "layerwise", 0
    code = {"mxfp4": ft.FT_FMT_MXFP4, "nvfp4": ft.FT_FMT_NVFP4, "bf16": ft.FT_FMT_BF16}[fmt]
    wave = T if T <= 2 else 2
    if not counters and T <= 4 and ft.ft_flow_geometry(H, I, wave, K_TOP, S_SHARED, E, L, code)["ok"]:
        return "flow", (T + wave - 1) // wave
    if code == ft.FT_FMT_MXFP4:
        return "counters", 1
    return "layerwise", 0


def stack_launches(T, layerwise=False, counters=False, fmt="mxfp4"):
    """Kernel launches of one stacked pass: a routing kernel and a persistent
    kernel per wave, or the routing kernel and two kernels per layer."""
    path, waves = _stack_path(T, layerwise, counters, fmt)
    return 1 + 2 * L if path == "layerwise" else 2 * waves


def decode_kernel_name(T, layerwise=False, counters=False, fmt="mxfp4"):
    """The kernels ft_moe_stack_forward runs for this batch."""
    path, waves = _stack_path(T, layerwise, counters, fmt)
    if path == "flow":
        return "persistent stack kernel, dataflow (tagged hand-overs)" + (
            f", {waves} waves of two tokens" if waves > 1 else "")
    if path == "counters":
        return "persistent stack kernel, counter-synchronised"
    return "two per layer"


FORMAT_NAMES = {"mxfp4": "MXFP4 (e2m1 + UE8M0/32)", "nvfp4": "NVFP4 (e2m1 + E4M3/16 + fp32 per matrix)",
                "bf16": "BF16"}


def workload_config(T, layerwise=False, counters=False, fmt="mxfp4"):
    return {"decode_kernels": decode_kernel_name(T, layerwise, counters, fmt),
            "workload": f"35B-A3B-class MoE decode stack: hidden {H}, {E} routed experts top-{K_TOP} + {S_SHARED} shared, "
                        f"intermediate {I}, {L} layers, {FORMAT_NAMES[fmt]} weights resident in HBM, "
                        f"batch {T}, Zipf(1.1) routing traces with 0.6 adjacent-token reuse",
            "global_batch": T, "layers": L, "l2": "inputs larger than L2 (~600 MB of distinct expert weights per step)"}


def main():
    global L
    args = parse()
    T = args.tokens
    L = args.layers
    if args.impl == "reference" and args.case == "decode":
        # the oracle runs on the host cores of rank 0 alone; other ranks exit
        # (no process group and no GPU needed)
        if int(os.environ.get("RANK", "0")) != 0:
            return
        world, rank = 1, 0
    else:
        world, rank, local = dist_setup(args)
    if args.case != "decode":
        if rank == 0:
            r = {"prefill": lambda: measure_prefill(reps=max(args.steps, 1)), "miss": measure_misses,
                 "glm": measure_glm, "gemm": lambda: measure_gemm_small(reps=max(args.steps, 1), fmt=args.format),
                 "router": lambda: measure_router(reps=max(args.steps, 1)),
                 "nvfp4": lambda: measure_prefill_nvfp4(measure_fp4_peak()["tflops"], peaks()),
                 "dsv4": lambda: measure_decode_dsv4(peaks())}[args.case]()
            print(json.dumps({"case": args.case, **r}))
        return
    if args.impl == "reference":
        # one step = one layer of the stack through the C++ oracle on every
        # host core: W warm-up and exactly K timed steps (about 0.1 s each on
        # 16 cores), so ms_per_step x steps is the timed region
        threads = host_cores()
        times, _ = oracle_layer_times(T, args.steps, args.warmup, float("inf"), threads)
        v = T * len(times) / (sum(times) * L)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": 1,
                "steps": len(times), "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": workload_config(T),
                "cpu_baseline": {"value": v, "unit": "tok/s", "cores": threads, "kind": "oracle",
                                 "sample": f"{len(times)} timed layers (after {args.warmup} warm-up) of one token "
                                           f"through the {L}-layer stack, one layer a step, cycling over the "
                                           f"inputs of 4 layers, mean extrapolated to {L} layers; C++ oracle on "
                                           f"{threads} OpenMP threads; inputs generated outside the timed region"},
                "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return
    res = run_ours(args, world, rank)
    if rank != 0:
        return
    pk = peaks()
    gu = res["kernels"].get("gate_up")
    dn = res["kernels"].get("down_combine")
    st = res["kernels"].get("dec_stack")
    print(f"# tok/s {res['tok_s']:.1f}  step HBM {res['hbm_gbs']:.0f} GB/s  kernels {res['kernels']}", file=sys.stderr)
    if st:  # the persistent kernel reads every layer's weights in one launch
        rk, rk_bytes, rk_us = "dec_stack", res["stack_bytes"], st["us_avg"]
        rk_traffic = STACK_TRAFFIC_PER_BYTE * rk_bytes if H == 2048 and I == 512 else None
    else:
        rk, rk_bytes, rk_us = "gate_up", res["gate_up_bytes"], gu["us_avg"] if gu else float("nan")
        rk_traffic = None
    rk_gbs = rk_bytes / (rk_us * 1e-6) / 1e9
    line = {"metric": METRIC, "value": res["tok_s"], "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DECODE_DTYPE[args.format], "data": "synthetic",
            "config": workload_config(T, args.layerwise, args.counters, args.format),
            "roofline": {"bound": "hbm", "kernel": rk, "achieved": rk_gbs, "peak": pk["hbm"],
                         "peak_source": pk["src"], "unit": "GB/s", "frac": rk_gbs / pk["hbm"], "traffic": rk_traffic,
                         "algorithmic_bytes_per_launch": rk_bytes},
            "hbm_gbs_step": res["hbm_gbs"], "hbm_frac_step": res["hbm_gbs"] / pk["hbm"],
            "gpu_launches": res["launches"], "clocks": res["clocks"], "e2e": res["e2e"],
            "kernels": res["kernels"]}
    if gu and dn:
        line["gate_up_gbs"] = res["gate_up_bytes"] / (gu["us_avg"] * 1e-6) / 1e9
        line["down_combine_gbs"] = res["down_bytes"] / (dn["us_avg"] * 1e-6) / 1e9
    if not args.no_extra and world == 1:
        try:
            line["prefill"] = measure_prefill()
        except Exception as ex:  # report, do not hide the main line
            line["prefill"] = {"error": repr(ex)}
        try:
            line["miss"] = measure_misses()
        except Exception as ex:
            line["miss"] = {"error": repr(ex)}
        if T == 1 and not args.layerwise:
            try:
                line["decode_batch4"] = measure_decode_batch(args, 4, pk)
            except Exception as ex:
                line["decode_batch4"] = {"error": repr(ex)}
            if args.format == "mxfp4":
                try:
                    line["decode_formats"] = measure_decode_formats(args, pk)
                except Exception as ex:
                    line["decode_formats"] = {"error": repr(ex)}
                try:
                    line["decode_dsv4"] = measure_decode_dsv4(pk)
                except Exception as ex:
                    line["decode_dsv4"] = {"error": repr(ex)}
        try:
            line["glm"] = measure_glm()
        except Exception as ex:
            line["glm"] = {"error": repr(ex)}
    if world == 1:
        cores = host_cores()
        v, done = oracle_tok_s(T, cores)
        v1, done1 = oracle_tok_s(T, 1)
        line["cpu_baseline"] = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle",
                                "sample": f"C++ oracle on {cores} OpenMP threads: 1 token through {done} layers of the "
                                          f"{L}-layer stack (after one warm-up layer), mean extrapolated to {L}; "
                                          f"inputs generated outside the timed region",
                                "single_thread": {"value": v1, "unit": "tok/s", "cores": 1, "layers": done1}}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
