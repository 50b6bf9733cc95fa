#!/usr/bin/env python
"""Benchmark: NVFP4 GEMM on the attention-projection M-sweep (N=768, K=6144).

One step = one pass of the hot path over the sweep M in {1,16,64,128,256,512}:
six NVFP4 GEMMs through the C ABI (row-major scales in, BF16 out), each on its
own buffers.  Steps rotate over enough distinct buffer sets that the working
set between two uses of a buffer is more than 4x the L2 cache, so every step
streams its operands from HBM.  Steps are replayed from CUDA graphs and timed
with CUDA events on the launching stream; the metric is algorithmic bytes /
time (GB/s) with bytes = M*K/2 + N*K/2 + (M+N)*K/16 + 2*M*N per GEMM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs the same per-GPU workload (weak scaling, no
collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from nvfp4_block_scaled_gemm_b200 import accounting, synth  # noqa: E402
from nvfp4_block_scaled_gemm_b200.dist_timing import max_over_ranks  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS & HBM GB/s vs B200 roofline, M-sweep on attn/MoE shapes"
SWEEP_M = synth.ATTN_SWEEP_M
N, K = synth.ATTN_N, synth.HIDDEN_K
SEED0 = 1100
WORKLOAD = "attention-projection NVFP4 GEMM sweep: M in {1,16,64,128,256,512}, N=768, K=6144, BF16 out"
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0


def step_bytes() -> int:
    return sum(accounting.gemm_bytes(m, N, K) for m in SWEEP_M)


def step_flops() -> int:
    return sum(accounting.gemm_flops(m, N, K) for m in SWEEP_M)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------- CPU oracle leg
def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_gemm_threaded(ca, sa, cb, sb, alpha, M, Nn, Kk, threads):
    """The whole GEMM through the oracle as it stands, its output split into
    `threads` blocks of rows (or of columns when M is small), one oracle call
    per block on its own host thread (the C oracle runs without the GIL).
    Returns the wall seconds."""
    import oracle  # test infrastructure: only the CPU-baseline legs use it
    from concurrent.futures import ThreadPoolExecutor

    by_rows = M >= threads or M >= Nn
    n = M if by_rows else Nn
    cuts = np.linspace(0, n, min(threads, n) + 1).astype(int)

    def block(i):
        a, b = cuts[i], cuts[i + 1]
        if by_rows:
            oracle.gemm(ca[a:b], sa[a:b], cb, sb, alpha, b - a, Nn, Kk)
        else:
            oracle.gemm(ca, sa, cb[a:b], sb[a:b], alpha, M, b - a, Kk)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(cuts) - 1) as ex:
        list(ex.map(block, range(len(cuts) - 1)))
    return time.perf_counter() - t0


def oracle_grouped_threaded(A, sA, B, sB, alpha, offsets, Nn, Kk, threads):
    """The whole grouped GEMM through the grouped oracle, its experts split
    into `threads` contiguous ranges of about equal row counts, one oracle
    call per range on its own host thread.  Returns the wall seconds."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    G = len(offsets) - 1
    total = int(offsets[-1])
    bounds = [0]
    for t in range(1, threads):
        bounds.append(int(np.searchsorted(offsets, total * t / threads, side="left")))
    bounds.append(G)
    bounds = sorted(set(min(max(b, 0), G) for b in bounds))

    def part(i):
        g0, g1 = bounds[i], bounds[i + 1]
        r0, r1 = int(offsets[g0]), int(offsets[g1])
        if r1 == r0:
            return
        off = (offsets[g0:g1 + 1] - r0).astype(np.int32)
        oracle.grouped_gemm(A[r0:r1], sA[r0:r1], B[g0:g1], sB[g0:g1], alpha[g0:g1], off, g1 - g0, r1 - r0, Nn, Kk)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(bounds) - 1) as ex:
        list(ex.map(part, range(len(bounds) - 1)))
    return time.perf_counter() - t0


def oracle_problem(name, M, Nn, Kk, kind, seed):
    import oracle
    A32, B32 = synth.source(kind, M, Nn, Kk, seed)
    ca, sa, ga = oracle.quantize(A32)
    cb, sb, gb = oracle.quantize(B32)
    return ca, sa, cb, sb, float(np.float32(ga) * np.float32(gb))


def oracle_sweep_problems():
    return [oracle_problem(*w) for w in synth.attention_sweep()]


def oracle_sweep_seconds(problems, threads) -> float:
    return sum(oracle_gemm_threaded(ca, sa, cb, sb, al, m, N, K, threads)
               for (ca, sa, cb, sb, al), m in zip(problems, SWEEP_M))


def cpu_baseline_record() -> dict:
    """The oracle on the host cores, whole GEMMs: the attention sweep (the
    line's own workload, its value), and one whole GEMM or more of every
    other configuration."""
    threads = host_threads()
    sweep = oracle_sweep_problems()
    secs = oracle_sweep_seconds(sweep, threads)
    per_config = {}
    # single 8 x 768 x 6144
    ca, sa, cb, sb, al = oracle_problem("single", 8, N, K, "normal", 1000)
    t = oracle_gemm_threaded(ca, sa, cb, sb, al, 8, N, K, threads)
    per_config["single_8x768x6144"] = {"s": round(t, 4), "GBps": round(accounting.gemm_bytes(8, N, K) / t / 1e9, 4)}
    # MoE sweep: one whole GEMM of each weight shape at M = 64
    for (name, M, Nn, Kk, kind, seed) in synth.moe_sweep():
        if M != 64:
            continue
        ca, sa, cb, sb, al = oracle_problem(name, M, Nn, Kk, kind, seed)
        t = oracle_gemm_threaded(ca, sa, cb, sb, al, M, Nn, Kk, threads)
        per_config[name] = {"s": round(t, 3), "GBps": round(accounting.gemm_bytes(M, Nn, Kk) / t / 1e9, 4),
                            "GFLOPs": round(accounting.gemm_flops(M, Nn, Kk) / t / 1e9, 2)}
    # saturation: the smallest shape, whole
    name, M, Nn, Kk, kind, seed = synth.saturation_sweep()[0]
    ca, sa, cb, sb, al = oracle_problem(name, M, Nn, Kk, kind, seed)
    t = oracle_gemm_threaded(ca, sa, cb, sb, al, M, Nn, Kk, threads)
    per_config[name] = {"s": round(t, 3), "GFLOPs": round(accounting.gemm_flops(M, Nn, Kk) / t / 1e9, 2)}
    # grouped MoE, whole (expert weights: random codes and scales of the right
    # shape -- the oracle's work does not depend on the values)
    r = synth.moe_routing()
    G, Nn, Kk = synth.MOE_EXPERTS, synth.MOE_N, synth.HIDDEN_K
    Mt = int(r.row_offsets[-1])
    A = synth.random_codes(Mt, Kk, 1)
    sA = synth.random_scales(Mt, Kk, 2)
    B = synth.random_codes(G * Nn, Kk, 3).reshape(G, Nn, Kk // 2)
    sB = synth.random_scales(G * Nn, Kk, 4).reshape(G, Nn, Kk // 16)
    alpha = np.full(G, 1e-3, np.float32)
    t = oracle_grouped_threaded(A, sA, B, sB, alpha, r.row_offsets, Nn, Kk, threads)
    counts = [int(c) for c in np.diff(r.row_offsets)]
    per_config["grouped_moe_256x2048x6144"] = {
        "s": round(t, 3), "GBps": round(accounting.grouped_bytes(counts, Nn, Kk) / t / 1e9, 4),
        "GFLOPs": round(accounting.grouped_flops(counts, Nn, Kk) / t / 1e9, 2)}
    return {
        "value": round(step_bytes() / secs / 1e9, 6), "unit": "GB/s", "cores": threads, "kind": "oracle",
        "sample": f"whole GEMMs, no extrapolation: the full attention sweep (six GEMMs, every output an exact "
                  f"integer dot product rounded once to BF16) in {secs:.2f} s on {threads} host threads; "
                  f"per_config: one or more whole GEMMs of every other configuration (grouped: random codes)",
        "per_config": per_config,
    }


# ---------------------------------------------------------------- clocks
class ClockSampler:
    REASONS = {
        0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x1: "gpu_idle",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.period, self.ok = [], period_s, False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self, t0: float, t1: float) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        self.t.join()
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        reasons = set()
        for _, _, rs in inside:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([s[1] for s in inside])) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------------- GPU arm
def graph_upload(g, stream) -> None:
    """Upload an instantiated CUDA graph to the device (cuGraphUpload), so
    that its first replay inside a timed region runs warm."""
    import ctypes
    h = g.raw_cuda_graph_exec()
    h = int(h) if not isinstance(h, int) else h
    lib = ctypes.CDLL("libcuda.so.1")
    lib.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.cuGraphUpload.restype = ctypes.c_int
    rc = lib.cuGraphUpload(ctypes.c_void_p(h), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cuGraphUpload failed with CUresult {rc}")


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_gemm_b200 as nv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    nv.lib()
    hbm_gbs, bf16_tf, peak_src = load_peaks()
    b_const = not args.no_b_constant

    # Inputs: seeded fp32 sources quantised on the GPU (not timed).
    base = []
    gen = torch.Generator(device=dev)
    for i, m in enumerate(SWEEP_M):
        gen.manual_seed(SEED0 + i + 1000 * rank)
        A32 = torch.randn((m, K), generator=gen, device=dev, dtype=torch.float32)
        B32 = torch.randn((N, K), generator=gen, device=dev, dtype=torch.float32)
        ca, sa, ga = nv.quantize(A32)
        cb, sb, gb = nv.quantize(B32)
        alpha = float(ga.item() * gb.item())
        base.append((m, ca, sa, cb, sb, alpha))
        del A32, B32
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    set_bytes = sum(accounting.gemm_bytes(m, N, K) for m in SWEEP_M)
    R = max(2, -(-4 * l2 // set_bytes))
    sets = []
    for r in range(R):
        sets.append([(m, ca.clone(), sa.clone(), cb.clone(), sb.clone(), al,
                      torch.empty((m, N), dtype=torch.bfloat16, device=dev)) for (m, ca, sa, cb, sb, al) in base])
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    def enqueue_step(r):
        for (m, ca, sa, cb, sb, al, D) in sets[r]:
            nv.gemm(ca, sa, cb, sb, al, out=D, stream=stream, b_constant=b_const)

    # One eager pass over every buffer set on the capture stream: allocates
    # the library's per-stream scratch once (before any capture), not counted
    # as a step.
    with torch.cuda.stream(stream):
        for r in range(R):
            enqueue_step(r)
    stream.synchronize()
    assert nv.get_device_error(stream) == 0

    # Graphs of consecutive steps (step i uses buffer set i % R): a full
    # rotation of R steps, and one graph each for the remainders of the
    # warm-up and of the timed region.
    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        l0 = nv.kernel_launches()
        with torch.cuda.graph(g, stream=stream):
            for r in range(nsteps):
                enqueue_step(r % R)
        return g, nv.kernel_launches() - l0

    g_full, launches_full = capture(R)
    rem = args.steps % R
    g_rem, launches_rem = capture(rem) if rem else (None, 0)
    wrem = args.warmup % R
    g_wrem, _ = capture(wrem) if wrem else (None, 0)

    # Exactly W untimed warm-up steps.
    with torch.cuda.stream(stream):
        for _ in range(args.warmup // R):
            g_full.replay()
        if g_wrem is not None:
            g_wrem.replay()
    # Every graph the timed region replays is on the device before it starts.
    graph_upload(g_full, stream)
    if g_rem is not None:
        graph_upload(g_rem, stream)
    stream.synchronize()

    clocks = ClockSampler(local_rank)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_wall0 = time.perf_counter()
    launches = 0
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps // R):
            g_full.replay()
            launches += launches_full
        if g_rem is not None:
            g_rem.replay()
            launches += launches_rem
        ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    clock_rec = clocks.stop(t_wall0, t_wall1)
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    status = nv.get_device_error(stream)
    if status != 0:
        raise RuntimeError(f"device error status {status}")

    total_bytes = step_bytes() * args.steps * world
    total_flops = step_flops() * args.steps * world
    gbs = total_bytes / (ms / 1e3) / 1e9
    tflops = total_flops / (ms / 1e3) / 1e12

    # Per-GEMM breakdown: each shape of the sweep alone, graph-replayed
    # back-to-back calls over rotating buffers (separate from the timed
    # region; a GEMM next to others of its own shape, not inside the sweep).
    sweep = []
    for i, m in enumerate(SWEEP_M):
        us = time_single_shape(nv, torch, dev, m, N, K, "normal", SEED0 + i, 400, stream, b_constant=b_const)
        b, f = accounting.gemm_bytes(m, N, K), accounting.gemm_flops(m, N, K)
        sweep.append({"M": m, "us": round(us, 3), "GBps": round(b / us / 1e3, 1), "TFLOPS": round(f / us / 1e6, 2),
                      "hbm_frac": round(b / us / 1e3 / hbm_gbs, 4)})

    # Roofline of the step's GEMM launches (one launch per GEMM: the CUDA-core
    # kernel for M = 1, the tensor-core kernels for the other five).
    # Average launch duration over the timed region.
    launches_per_rank = launches
    avg_launch_us = ms * 1e3 / max(1, launches_per_rank)
    bytes_per_launch = step_bytes() / len(SWEEP_M)
    achieved = bytes_per_launch / (avg_launch_us * 1e-6) / 1e9
    traffic = load_traffic()

    # End-to-end through the public API with host buffers.
    e2e = run_e2e(nv, torch, dev, base, min(args.steps, 20), stream)

    line = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": list(SWEEP_M), "N": N, "K": K, "parallelism": f"replicas{world}",
                   "l2": f"inputs larger than L2: {R} rotating buffer sets, {R * set_bytes / 2**20:.0f} MiB "
                         f"vs L2 {l2 / 2**20:.0f} MiB",
                   "launch": "CUDA graphs of back-to-back nvfp4_gemm calls (uploaded before the timed region)",
                   "weights": "constant: NVFP4_GEMM_B_CONSTANT" if b_const else "no constant-weight flag",
                   "inputs": "N(0,1) fp32 quantised to NVFP4 on the GPU (not timed)"},
        "tflops": round(tflops, 3),
        "sweep": sweep,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s",
                     "frac": round(achieved / hbm_gbs, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} hbm_gbs",
                     "kernel": "the GEMM launches of the step (one per GEMM: the CUDA-core kernel at M = 1, split-K kernel at M = 16, tiled kernel above)",
                     "per_launch": {"algorithmic_bytes": bytes_per_launch, "avg_us": round(avg_launch_us, 3)}},
        "e2e": e2e,
        "gpu_launches": launches_per_rank,
        "clocks": clock_rec,
        "accum": "f32", "out_dtype": "bf16",
    }
    if world == 1 and not args.no_configs:
        line["configs"] = run_configs(args, nv, torch, dev, stream, local_rank, b_const)
    return line


def run_configs(args, nv, torch, dev, stream, local_rank, b_const):
    """The other configurations, each shape timed alone (graph-replayed
    back-to-back calls over rotating buffers > 4x L2; the grouped GEMM as
    eager launches over 1.8 GB of weights), with the clocks sampled over the
    whole section."""
    hbm_gbs, bf16_tf, src = load_peaks()
    fp4_tf = 4.0 * bf16_tf
    clocks = ClockSampler(local_rank)
    clocks.start()
    t0 = time.perf_counter()
    calib = measure_fp4_peak(nv, torch, stream)

    def row(name, M, Nn, Kk, kind, seed, iters):
        us = time_single_shape(nv, torch, dev, M, Nn, Kk, kind, seed, iters, stream, b_constant=b_const)
        b, f = accounting.gemm_bytes(M, Nn, Kk), accounting.gemm_flops(M, Nn, Kk)
        t_hbm, t_fp4 = b / (hbm_gbs * 1e9), f / (fp4_tf * 1e12)
        return {"name": name, "M": M, "N": Nn, "K": Kk, "us": round(us, 2), "GBps": round(b / us / 1e3, 1),
                "TFLOPS": round(f / us / 1e6, 1), "bound": "hbm" if t_hbm >= t_fp4 else "tensor",
                "roofline_frac": round(max(t_hbm, t_fp4) / (us * 1e-6), 4),
                "frac_of_calibrated_fp4": round(f / us / 1e6 / max(calib.values()), 4)}

    out = {"single": [row("single_8x768x6144", 8, N, K, "normal", 1000, 400)],
           "moe_sweep": [row(*w, iters=400) for w in synth.moe_sweep()],
           "saturation": [row(*w, iters=60) for w in synth.saturation_sweep()]}
    out["grouped"] = run_grouped(argparse.Namespace(steps=50))
    clock_rec = clocks.stop(t0, time.perf_counter())
    out["peaks"] = {"hbm_gbs": hbm_gbs, "fp4_tflops": fp4_tf, "source": f"{src} (fp4 = 4 x bf16)",
                    "fp4_calibrated_tflops": calib}
    out["clocks"] = clock_rec
    return out


def load_traffic():
    """DRAM bytes per GEMM launch of the sweep from the committed ncu summary,
    or None when the kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "traffic_attn_sweep.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("source_hash") != source_hash():
            return None
        return rec["dram_bytes_per_launch"]
    except Exception:
        return None


def source_hash() -> str:
    from nvfp4_block_scaled_gemm_b200.build import source_hash as h
    return h()


def gpu_local_cpus(local_rank):
    """The host CPUs NVML reports as closest to this GPU (its NUMA node), or
    None.  Pinned host buffers allocated by a thread running there sit in that
    node's memory, which is what the PCIe copies read."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(local_rank)
        words = pynvml.nvmlDeviceGetCpuAffinity(h, 16)   # 16 x 64-bit masks
        cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (w >> b) & 1}
        pynvml.nvmlShutdown()
        cpus &= os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


def run_e2e(nv, torch, dev, base, steps, stream):
    """Same metric through nvfp4_gemm with pinned HOST buffers: every step copies
    all its inputs host->device (one pinned arena holding the six GEMMs' A, sA,
    B and sB, one copy) and all its outputs device->host (one arena, one copy)
    inside the timed region.  (Double-buffered device arenas with the input
    copy on a second stream measured slower: 26.8 against 45.5 GB/s.)"""
    def pad(n):
        return (n + 255) // 256 * 256

    # run (and allocate the pinned arenas) on the GPU's own NUMA node; restored below
    saved_cpus = os.sched_getaffinity(0)
    local = gpu_local_cpus(dev.index or 0)
    if local:
        os.sched_setaffinity(0, local)
    try:
        return _run_e2e(nv, torch, dev, base, steps, stream, pad, local)
    finally:
        os.sched_setaffinity(0, saved_cpus)


def _run_e2e(nv, torch, dev, base, steps, stream, pad, local):
    # input arena: per GEMM A, sA, B, sB as bytes, each on a 256-byte boundary
    layout, off = [], 0
    for (m, ca, sa, cb, sb, al) in base:
        ent = []
        for x in (ca, sa, cb, sb):
            ent.append((off, tuple(x.shape)))
            off += pad(x.numel())
        layout.append(ent)
    h_in = torch.zeros(off, dtype=torch.uint8).pin_memory()
    for (m, ca, sa, cb, sb, al), ent in zip(base, layout):
        for x, (o, shape) in zip((ca, sa, cb, sb), ent):
            h_in[o:o + x.numel()].copy_(x.reshape(-1).cpu())
    d_in = torch.empty(off, dtype=torch.uint8, device=dev)
    # output arena: per GEMM D (BF16), each on a 256-byte boundary
    out_off, o = [], 0
    for (m, *_rest) in base:
        out_off.append(o)
        o += pad(m * N * 2) // 2
    h_out = torch.empty(o, dtype=torch.bfloat16).pin_memory()
    d_out = torch.empty(o, dtype=torch.bfloat16, device=dev)
    gemms = []
    for (m, ca, sa, cb, sb, al), ent, oo in zip(base, layout, out_off):
        views = [d_in[o0:o0 + int(np.prod(shape))].view(shape) for (o0, shape) in ent]
        gemms.append((views, al, d_out[oo:oo + m * N].view(m, N)))
    h2d = sum(int(np.prod(shape)) for ent in layout for (_, shape) in ent)
    d2h = sum(m * N * 2 for (m, *_rest) in base)

    def one_step():
        d_in.copy_(h_in, non_blocking=True)
        for (dA, dsA, dB, dsB), al, dD in gemms:
            nv.gemm(dA, dsA, dB, dsB, al, out=dD, stream=stream)
        h_out.copy_(d_out, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            one_step()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            one_step()
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1)
    # the last step's results, read back through the host arena, are the GEMMs' results
    for ((dA, dsA, dB, dsB), al, dD), oo, (m, *_rest) in zip(gemms, out_off, base):
        assert torch.equal(h_out[oo:oo + m * N].view(m, N).view(torch.int16), dD.cpu().view(torch.int16))
    return {"value": round(step_bytes() * steps / (ms / 1e3) / 1e9, 3), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "copies_per_step": {"h2d": 1, "d2h": 1, "arena_bytes": int(off)},
            "host_cpus": f"the GPU's NUMA-local CPUs ({len(local)})" if local else "all (NVML affinity unavailable)"}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle, as it stands, on the host cores (all of them, one thread
    per block of outputs): each step is the whole attention sweep -- six
    whole GEMMs -- when the K + W steps fit a few minutes, otherwise the same
    fraction of every GEMM's output rows (columns for one token row)."""
    threads = host_threads()
    problems = oracle_sweep_problems()
    t_one = oracle_sweep_seconds(problems, threads)          # calibration (not a counted step)
    budget_s = 180.0
    frac = min(1.0, budget_s / max(1e-9, t_one * (args.steps + args.warmup)))

    def cut(ca, sa, cb, sb, m):
        if frac >= 1.0:
            return ca, sa, cb, sb, m, N
        if m >= 8:
            r = max(1, int(round(m * frac)))
            return ca[:r], sa[:r], cb, sb, r, N
        c = max(8, int(round(N * frac)))
        return ca, sa, cb[:c], sb[:c], m, c

    work = [cut(ca, sa, cb, sb, m) + (al,) for (ca, sa, cb, sb, al), m in zip(problems, SWEEP_M)]

    def one_step():
        return sum(oracle_gemm_threaded(ca, sa, cb, sb, al, m, n, K, threads) for (ca, sa, cb, sb, m, n, al) in work)

    for _ in range(args.warmup):
        one_step()
    total = sum(one_step() for _ in range(args.steps))
    done = sum(m * n for (_, _, _, _, m, n, _) in work) / sum(m * N for m in SWEEP_M)
    value = round(step_bytes() * done * args.steps / total / 1e9, 6)
    sample = (f"each step the whole sweep (six whole GEMMs) on {threads} host threads" if frac >= 1.0 else
              f"each step {done:.3f} of every GEMM's outputs on {threads} host threads; value = the sweep's "
              f"bytes x that fraction / time")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int64-exact/f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": list(SWEEP_M), "N": N, "K": K, "parallelism": f"cpu{threads}"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- other configurations
def time_single_shape(nv, torch, dev, M, Nn, Kk, kind, seed, iters, stream, b_constant=False):
    """Back-to-back GEMMs of one shape from a CUDA graph over rotating
    buffers (> 4x L2); returns microseconds per GEMM."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    if kind == "uniform":
        A32 = torch.rand((M, Kk), generator=gen, device=dev) * 2 - 1
        B32 = torch.rand((Nn, Kk), generator=gen, device=dev) * 2 - 1
    else:
        A32 = torch.randn((M, Kk), generator=gen, device=dev)
        B32 = torch.randn((Nn, Kk), generator=gen, device=dev) * (0.02 if kind == "moe" else 1.0)
        if kind == "moe":
            A32 = torch.where(torch.rand((M, Kk), generator=gen, device=dev) < 0.01, A32 * 20, A32)
    a, sa, ga = nv.quantize(A32)
    b, sb, gb = nv.quantize(B32)
    del A32, B32
    alpha = float(ga.item() * gb.item())
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nbytes = accounting.gemm_bytes(M, Nn, Kk)
    R = int(max(2, min(64, -(-4 * l2 // nbytes))))
    sets = [(a.clone(), sa.clone(), b.clone(), sb.clone(), torch.empty((M, Nn), dtype=torch.bfloat16, device=dev))
            for _ in range(R)]
    with torch.cuda.stream(stream):
        for x in sets:
            nv.gemm(x[0], x[1], x[2], x[3], alpha, out=x[4], stream=stream, b_constant=b_constant)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for x in sets:
            nv.gemm(x[0], x[1], x[2], x[3], alpha, out=x[4], stream=stream, b_constant=b_constant)
    reps = max(1, iters // R)
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    assert nv.get_device_error(stream) == 0
    return e0.elapsed_time(e1) * 1e3 / (reps * R)


def measure_fp4_peak(nv, torch, stream, steps=200000, reps=3):
    """Dense FP4 tensor-core rate from the library's calibration kernel
    (back-to-back block-scaled MMAs on resident operands): TFLOP/s for the
    1-CTA and the 2-CTA (CTA pair) instruction forms."""
    out = {}
    for pair in (False, True):
        with torch.cuda.stream(stream):
            nv.fp4_peak_probe(pair, steps // 10, stream)          # warm-up
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ctas = 0
            for _ in range(reps):
                ctas = nv.fp4_peak_probe(pair, steps, stream)
            e1.record(stream)
        stream.synchronize()
        assert nv.get_device_error(stream) == 0
        secs = e0.elapsed_time(e1) / 1e3 / reps
        out["cta_pair" if pair else "one_cta"] = round(steps * ctas * nv.FP4_PEAK_FLOPS_PER_STEP / secs / 1e12, 1)
    return out


def run_shapes(args, shapes, label):
    import torch
    import nvfp4_block_scaled_gemm_b200 as nv
    dev = torch.device("cuda", 0)
    nv.lib()
    hbm_gbs, bf16_tf, src = load_peaks()
    fp4_tf = 4.0 * bf16_tf      # dense FP4 = 4x dense BF16 (nominal 9 vs 2.25 PFLOP/s)
    stream = torch.cuda.Stream()
    calib = measure_fp4_peak(nv, torch, stream) if label in ("saturation", "pages") else None
    rows = []
    for (name, M, Nn, Kk, kind, seed) in shapes:
        us = time_single_shape(nv, torch, dev, M, Nn, Kk, kind, seed, args.steps, stream)
        b, f = accounting.gemm_bytes(M, Nn, Kk), accounting.gemm_flops(M, Nn, Kk)
        t_roof = max(b / (hbm_gbs * 1e9), f / (fp4_tf * 1e12))
        row = {"name": name, "M": M, "N": Nn, "K": Kk, "us": round(us, 2), "GBps": round(b / us / 1e3, 1),
               "TFLOPS": round(f / us / 1e6, 1), "roofline_frac": round(t_roof / (us * 1e-6), 4),
               "bound": "hbm" if b / (hbm_gbs * 1e9) >= f / (fp4_tf * 1e12) else "tensor"}
        if calib:
            row["frac_of_calibrated_fp4"] = round(f / us / 1e6 / max(calib.values()), 4)
            row["frac_of_nominal_9pf"] = round(f / us / 1e6 / 9000.0, 4)
        rows.append(row)
    peaks = {"hbm_gbs": hbm_gbs, "fp4_tflops": fp4_tf, "source": f"{src} (fp4 = 4 x bf16)"}
    if calib:
        peaks["fp4_calibrated_tflops"] = calib
        peaks["fp4_nominal_tflops"] = 9000.0
    return {"workload": label, "peaks": peaks, "shapes": rows}


def run_grouped(args):
    import torch
    import nvfp4_block_scaled_gemm_b200 as nv
    dev = torch.device("cuda", 0)
    nv.lib()
    hbm_gbs, bf16_tf, src = load_peaks()
    G, Nn, Kk = synth.MOE_EXPERTS, synth.MOE_N, synth.HIDDEN_K
    r = synth.moe_routing()
    Mt = int(r.row_offsets[-1])
    gen = torch.Generator(device=dev)
    gen.manual_seed(1400)
    X = torch.randn((synth.MOE_TOKENS, Kk), generator=gen, device=dev)
    X = torch.where(torch.rand(X.shape, generator=gen, device=dev) < 0.01, X * 20, X)
    ct, st_, ga = nv.quantize(X)
    tok = torch.from_numpy(r.token_of_row.astype(np.int64)).to(dev)
    A, sA = ct[tok].contiguous(), st_[tok].contiguous()
    B = torch.empty((G, Nn, Kk // 2), dtype=torch.uint8, device=dev)
    sB = torch.empty((G, Nn, Kk // 16), dtype=torch.uint8, device=dev)
    alpha = torch.empty((G,), dtype=torch.float32, device=dev)
    for g in range(G):
        W = torch.randn((Nn, Kk), generator=gen, device=dev) * 0.02
        cb, sb, gb = nv.quantize(W)
        B[g].copy_(cb)
        sB[g].copy_(sb)
        alpha[g] = ga[0] * gb[0]
    off = torch.from_numpy(r.row_offsets.astype(np.int32)).to(dev)
    D = torch.empty((Mt, Nn), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        nv.grouped_gemm(A, sA, B, sB, alpha, off, out=D)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    iters = max(3, min(args.steps, 50))
    e0.record()
    for _ in range(iters):
        nv.grouped_gemm(A, sA, B, sB, alpha, off, out=D)
    e1.record()
    torch.cuda.synchronize()
    assert nv.get_device_error() == 0
    us = e0.elapsed_time(e1) * 1e3 / iters
    counts = [int(c) for c in np.diff(r.row_offsets)]
    b, f = accounting.grouped_bytes(counts, Nn, Kk), accounting.grouped_flops(counts, Nn, Kk)
    return {"workload": "grouped MoE: 256 experts x [2048 x 6144], 512 tokens top-8 Zipf(1.1) -> 4096 rows",
            "active_experts": sum(1 for c in counts if c > 0), "max_rows": max(counts),
            "us": round(us, 2), "GBps": round(b / us / 1e3, 1), "TFLOPS": round(f / us / 1e6, 2),
            "hbm_frac": round(b / us / 1e3 / hbm_gbs, 4), "bytes": b, "peak_hbm_gbs": hbm_gbs,
            "note": "weights stream once per launch (1.8 GB >> L2); eager launches, events"}


def run_chain(args, layers=8):
    """A dependent layer sequence: attention-projection GEMMs alternating
    M x 768 x 6144 and M x 6144 x 768 (the tensor-parallel in/out projection
    shapes of one GPU), each layer's BF16 output quantized by
    nvfp4_quantize_scaled with a global scale fixed from one eager calibration
    pass, and fed to the next GEMM.  The whole chain is one CUDA graph; every
    launch in it uses programmatic dependent launch.  Reports the time per
    layer (quantize + GEMM) for each M."""
    import torch
    import nvfp4_block_scaled_gemm_b200 as nv
    dev = torch.device("cuda", 0)
    nv.lib()
    gen = torch.Generator(device=dev)
    gen.manual_seed(1500)
    dims = [(N, K), (K, N)]
    weights = []
    for li in range(layers):
        n_out, k_in = dims[li % 2]
        W = torch.randn((n_out, k_in), generator=gen, device=dev) * 0.02
        cb, sb, gb = nv.quantize(W)
        weights.append((cb, sb, float(gb.item())))
    stream = torch.cuda.Stream()
    out = []
    for m in (1, 16, 64, 256):
        X = torch.randn((m, K), generator=gen, device=dev).to(torch.bfloat16)
        # calibration: amax-scaled quantization of each layer's input, once
        g_act, cur = [], X
        for li in range(layers):
            cq, sq, gq = nv.quantize(cur.float())
            g = float(gq.item())
            g_act.append(g)
            cb, sb, gb = weights[li]
            cur = nv.gemm(cq, sq, cb, sb, g * gb)
        torch.cuda.synchronize()
        bufs = [torch.empty((m, dims[li % 2][0]), dtype=torch.bfloat16, device=dev) for li in range(layers)]

        def enqueue(fused):
            a = X
            for li in range(layers):
                cb, sb, gb = weights[li]
                if fused:   # the GEMM quantizes its activation tiles (one launch per layer where the shape allows)
                    nv.gemm_bf16a(a, g_act[li], cb, sb, g_act[li] * gb, out=bufs[li], stream=stream)
                else:
                    cq, sq = nv.quantize_scaled(a, g_act[li], stream=stream)
                    nv.gemm(cq, sq, cb, sb, g_act[li] * gb, out=bufs[li], stream=stream, b_constant=True)
                a = bufs[li]

        def time_chain(fused):
            with torch.cuda.stream(stream):
                enqueue(fused)
            stream.synchronize()
            g_chain = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_chain, stream=stream):
                enqueue(fused)
            reps = max(3, min(args.steps, 200))
            with torch.cuda.stream(stream):
                for _ in range(3):
                    g_chain.replay()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g_chain.replay()
                e1.record(stream)
            stream.synchronize()
            assert nv.get_device_error(stream) == 0
            return e0.elapsed_time(e1) * 1e3 / (reps * layers)

        us_two = time_chain(False)
        os.environ["NVFP4_GEMM_FUSE_QUANT"] = "1"
        try:
            us_fused = time_chain(True)
        finally:
            os.environ.pop("NVFP4_GEMM_FUSE_QUANT", None)
        b = sum(accounting.gemm_bytes(m, dims[li % 2][0], dims[li % 2][1]) for li in range(layers)) / layers
        out.append({"M": m, "us_per_layer": round(us_two, 2), "GBps": round(b / us_two / 1e3, 1),
                    "us_per_layer_fused": round(us_fused, 2)})
    return {"workload": f"dependent chain of {layers} layers (quantize_scaled + GEMM; `_fused`: nvfp4_gemm_bf16a "
                        f"with NVFP4_GEMM_FUSE_QUANT=1, the GEMM quantizing its own activation tiles), "
                        f"shapes alternating Mx{N}x{K} and Mx{K}x{N}, one CUDA graph, programmatic dependent launch",
            "layers": layers, "per_M": out,
            "note": "weights 6.3 MB per layer stay in L2 across replays (the chain is launch- and "
                    "latency-bound, which is what it measures)"}


def run_decode(args):
    """Few token rows: the same shapes through the tensor-core kernel
    (NVFP4_GEMM_GEMV=0) and through the CUDA-core kernel at each weight-row
    count per CTA (NVFP4_GEMM_GEMV=16, NVFP4_GEMM_GEMV_RW=1|2|4), plus the
    default dispatch, each as graph-replayed back-to-back calls over rotating
    buffers; microseconds per GEMM."""
    import torch
    import nvfp4_block_scaled_gemm_b200 as nv
    dev = torch.device("cuda", 0)
    nv.lib()
    hbm_gbs = load_peaks()[0]
    stream = torch.cuda.Stream()
    settings = (("tensor_cores", {"NVFP4_GEMM_GEMV": "0"}),
                ("cuda_cores_rw1", {"NVFP4_GEMM_GEMV": "16", "NVFP4_GEMM_GEMV_RW": "1"}),
                ("cuda_cores_rw2", {"NVFP4_GEMM_GEMV": "16", "NVFP4_GEMM_GEMV_RW": "2"}),
                ("cuda_cores_rw4", {"NVFP4_GEMM_GEMV": "16", "NVFP4_GEMM_GEMV_RW": "4"}),
                ("default", {}))
    keys = ("NVFP4_GEMM_GEMV", "NVFP4_GEMM_GEMV_RW")
    saved = {k: os.environ.get(k) for k in keys}
    rows = []
    try:
        for (Nn, Kk) in ((768, 6144), (2048, 6144), (256, 6144), (8192, 8192), (6144, 768)):
            for M in (1, 2, 4, 8):
                row = {"M": M, "N": Nn, "K": Kk}
                for name, env in settings:
                    for k in keys:
                        os.environ.pop(k, None)
                    os.environ.update(env)
                    us = time_single_shape(nv, torch, dev, M, Nn, Kk, "moe", 1700 + M, min(args.steps, 2000), stream,
                                           b_constant=True)
                    row[name] = round(us, 2)
                row["default_hbm_frac"] = round(accounting.gemm_bytes(M, Nn, Kk) / row["default"] / 1e3 / hbm_gbs, 4)
                rows.append(row)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    return {"workload": "decode: M in {1,2,4,8} on the attention, MoE and two larger weight shapes, tensor-core vs "
                        "CUDA-core kernel (us per GEMM, graph-replayed back-to-back calls, rotating buffers > L2, "
                        "constant weights)",
            "hbm_gbs": hbm_gbs, "shapes": rows}


def run_sparse(args):
    """2:4-sparse weights against dense ones on decode shapes: the same token
    rows and the same (pruned) weights, once compressed through
    nvfp4_gemm_sparse24 and once expanded through nvfp4_gemm; graph-replayed
    back-to-back calls over rotating buffers, us per GEMM."""
    import torch
    import nvfp4_block_scaled_gemm_b200 as nv
    dev = torch.device("cuda", 0)
    nv.lib()
    hbm_gbs = load_peaks()[0]
    stream = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    rows = []
    for (Nn, Kk) in ((768, 6144), (2048, 6144), (8192, 8192)):
        gen = torch.Generator(device=dev)
        gen.manual_seed(2300 + Nn)
        W = torch.randn((Nn, Kk), generator=gen, device=dev) * 0.02
        # prune on the device with the oracle's rule (keep the 2 pairs of each
        # 4 with the largest element magnitude), then quantize densely
        key = W.abs().view(Nn, Kk // 8, 4, 2).amax(dim=3)
        idx = torch.topk(key, 2, dim=2, largest=True, sorted=False).indices
        keep = torch.zeros_like(key, dtype=torch.bool).scatter_(2, idx, True)
        Wp = torch.where(keep.repeat_interleave(2, dim=2).view(Nn, Kk), W, torch.zeros_like(W))
        cb, sb, gb = nv.quantize(Wp)
        # compress: kept bytes in position order and their nibbles
        grp = cb.view(Nn, Kk // 8, 4)
        pos = torch.sort(idx, dim=2).values
        bv = torch.gather(grp, 2, pos.to(torch.int64)).reshape(Nn, Kk // 4).contiguous()
        nib = (pos[..., 0] | (pos[..., 1] << 2)).to(torch.uint8)
        bm = (nib[:, 0::2] | (nib[:, 1::2] << 4)).contiguous()
        for M in (1, 2, 4, 8):
            A32 = torch.randn((M, Kk), generator=gen, device=dev)
            ca, sa, ga = nv.quantize(A32)
            alpha = float(ga.item() * gb.item())
            per_set = Nn * Kk // 2 + Nn * Kk // 16
            R = int(max(2, min(64, -(-4 * l2 // per_set))))
            dense_sets = [(cb.clone(), sb.clone(), torch.empty((M, Nn), dtype=torch.bfloat16, device=dev))
                          for _ in range(R)]
            sparse_sets = [(bv.clone(), bm.clone(), sb.clone(), torch.empty((M, Nn), dtype=torch.bfloat16, device=dev))
                           for _ in range(R)]

            def timed(enqueue):
                with torch.cuda.stream(stream):
                    enqueue()
                stream.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    enqueue()
                reps = max(1, min(args.steps, 2000) // R)
                with torch.cuda.stream(stream):
                    g.replay()
                stream.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(reps):
                        g.replay()
                    e1.record(stream)
                stream.synchronize()
                assert nv.get_device_error(stream) == 0
                return e0.elapsed_time(e1) * 1e3 / (reps * R)

            us_dense = timed(lambda: [nv.gemm(ca, sa, b, s, alpha, out=o, stream=stream, b_constant=True)
                                      for (b, s, o) in dense_sets])
            us_sparse = timed(lambda: [nv.gemm_sparse24(ca, sa, v, m, s, alpha, out=o, stream=stream, b_constant=True)
                                       for (v, m, s, o) in sparse_sets])
            sparse_bytes = M * Kk // 2 + M * Kk // 16 + Nn * Kk // 4 + 2 * Nn * Kk // 16 + 2 * M * Nn
            rows.append({"M": M, "N": Nn, "K": Kk, "us_dense": round(us_dense, 2), "us_sparse": round(us_sparse, 2),
                         "sparse_GBps": round(sparse_bytes / us_sparse / 1e3, 1),
                         "sparse_hbm_frac": round(sparse_bytes / us_sparse / 1e3 / hbm_gbs, 4)})
    return {"workload": "2:4-sparse weights vs dense on decode shapes (us per GEMM, graph-replayed back-to-back "
                        "calls, rotating buffers > 4x L2)", "hbm_gbs": hbm_gbs, "shapes": rows}


def run_mxfp4(args):
    """MXFP4 (nvfp4_gemm_mxfp4) on the attention and MoE shapes, graph-replayed
    back-to-back calls over rotating buffers (> 4x L2), us per GEMM, beside
    the NVFP4 GEMM of the same shape.  Inputs are random codes and E8M0
    scales near 1 (the GEMM's work does not depend on the values)."""
    import torch
    import nvfp4_block_scaled_gemm_b200 as nv
    dev = torch.device("cuda", 0)
    nv.lib()
    hbm_gbs = load_peaks()[0]
    stream = torch.cuda.Stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    rows = []
    for (M, Nn, Kk) in ((1, 768, 6144), (16, 768, 6144), (128, 768, 6144), (512, 768, 6144), (1, 2048, 6144),
                        (64, 2048, 6144), (2048, 2048, 6144)):
        g = torch.Generator(device=dev)
        g.manual_seed(M + Nn)
        a = torch.randint(0, 256, (M, Kk // 2), generator=g, device=dev, dtype=torch.uint8)
        b = torch.randint(0, 256, (Nn, Kk // 2), generator=g, device=dev, dtype=torch.uint8)
        sa = torch.randint(120, 134, (M, Kk // 32), generator=g, device=dev, dtype=torch.uint8)
        sb = torch.randint(120, 134, (Nn, Kk // 32), generator=g, device=dev, dtype=torch.uint8)
        nbytes = M * Kk // 2 + Nn * Kk // 2 + (M + Nn) * Kk // 32 + 2 * M * Nn
        R = int(max(2, min(64, -(-4 * l2 // nbytes))))
        sets = [(a.clone(), sa.clone(), b.clone(), sb.clone(), torch.empty((M, Nn), dtype=torch.bfloat16, device=dev))
                for _ in range(R)]

        def enqueue():
            for x in sets:
                nv.gemm_mxfp4(x[0], x[1], x[2], x[3], 1.0, out=x[4], stream=stream, b_constant=True)

        with torch.cuda.stream(stream):
            enqueue()
        stream.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            enqueue()
        reps = max(1, min(args.steps, 2000) // R)
        with torch.cuda.stream(stream):
            gr.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                gr.replay()
            e1.record(stream)
        stream.synchronize()
        assert nv.get_device_error(stream) == 0
        us = e0.elapsed_time(e1) * 1e3 / (reps * R)
        us_nv = time_single_shape(nv, torch, dev, M, Nn, Kk, "normal", 1600 + M, min(args.steps, 2000), stream,
                                  b_constant=True)
        rows.append({"M": M, "N": Nn, "K": Kk, "us_mxfp4": round(us, 2), "us_nvfp4": round(us_nv, 2),
                     "mxfp4_GBps": round(nbytes / us / 1e3, 1), "mxfp4_hbm_frac": round(nbytes / us / 1e3 / hbm_gbs, 4),
                     "mxfp4_TFLOPS": round(2 * M * Nn * Kk / us / 1e6, 1)})
    return {"workload": "MXFP4 GEMM (E8M0 scale per 32 values) vs NVFP4 on the same shapes, us per GEMM "
                        "(graph-replayed back-to-back calls, rotating buffers > 4x L2, constant weights)",
            "hbm_gbs": hbm_gbs, "shapes": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration section of the line")
    ap.add_argument("--no-b-constant", action="store_true",
                    help="call the GEMMs without NVFP4_GEMM_B_CONSTANT (the weights are constant either way)")
    ap.add_argument("--workload", choices=["attn", "moe", "saturation", "grouped", "chain", "pages", "decode",
                                           "sparse", "mxfp4"],
                    default="attn",
                    help="attn (default) prints the benchmark line; the others print a per-shape report")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.workload != "attn":
        if rank == 0:
            if args.workload == "grouped":
                print(json.dumps(run_grouped(args)), flush=True)
            elif args.workload == "chain":
                print(json.dumps(run_chain(args)), flush=True)
            elif args.workload == "decode":
                print(json.dumps(run_decode(args)), flush=True)
            elif args.workload == "sparse":
                print(json.dumps(run_sparse(args)), flush=True)
            elif args.workload == "mxfp4":
                print(json.dumps(run_mxfp4(args)), flush=True)
            else:
                shapes = {"moe": synth.moe_sweep, "pages": synth.pages_sweep}.get(args.workload, synth.saturation_sweep)()
                print(json.dumps(run_shapes(args, shapes, args.workload)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline_record()
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
