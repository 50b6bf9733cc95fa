"""Run a few NVFP4 GEMMs of given shapes, for profiling one kernel under ncu.

    python -m nvfp4_block_scaled_gemm_b200.profile_case --shapes 512x768x6144 --iters 3
    python -m nvfp4_block_scaled_gemm_b200.profile_case --shapes attn --iters 2
    python -m nvfp4_block_scaled_gemm_b200.profile_case --grouped 64 --iters 3

`--traffic-csv FILE` (no GPU) instead turns the CSV log of an ncu run of
`--shapes attn --iters 2` with the metrics gpu__time_duration.sum,
dram__bytes_read.sum and dram__bytes_write.sum on the GEMM kernels
(every kernel named nvfp4_gemm_* or nvfp4_gemv_*) into the per-launch DRAM
summary that bench.py reports as `roofline.traffic`
(profiles/traffic_attn_sweep.json), stamped with the hash of the kernel code
it was taken on.

`attn` expands to the attention-projection sweep (M in {1,16,64,128,256,512},
N=768, K=6144).  Inputs are seeded N(0,1) fp32 quantised on the GPU; every
launch of a shape uses the same buffers (ncu flushes the caches between its
replay passes, so DRAM counters still see the compulsory traffic).

`--grouped E` runs the grouped MoE GEMM instead, on the MoE routing recipe
(top-8, Zipf(1.1) popularity) with E experts of [2048 x 6144] and the tokens
scaled with E (512 x E / 256), so experts keep about 16 rows each: E = 64
keeps the device footprint near half a GB while the weights (0.4 GB) still
exceed the L2, so a multi-pass ncu capture of the grouped kernel stays small.
"""
from __future__ import annotations

import argparse

import torch

import nvfp4_block_scaled_gemm_b200 as nv
from nvfp4_block_scaled_gemm_b200 import accounting, synth


def parse_shapes(text: str):
    out = []
    for item in text.split(","):
        if item == "attn":
            out += [(m, synth.ATTN_N, synth.HIDDEN_K) for m in synth.ATTN_SWEEP_M]
        else:
            m, n, k = (int(x) for x in item.lower().split("x"))
            out.append((m, n, k))
    return out


def summarize_traffic(csv_path: str, out_path: str, iters: int = 2) -> dict:
    """Per-launch DRAM bytes of the attention sweep from an ncu CSV log (the
    last of the `iters` launches of each shape, in sweep order)."""
    import csv
    import json
    import re

    from nvfp4_block_scaled_gemm_b200.build import source_hash

    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    launches = {}
    for row in csv.DictReader(lines):
        name = re.search(r"nvfp4_gem[mv]_\w*", row["Kernel Name"])
        if not name:
            continue
        rec = launches.setdefault(int(row["ID"]), {})
        rec["kernel"] = name.group(0)
        unit = row["Metric Unit"].strip().lower()
        val = float(row["Metric Value"].replace(",", ""))
        scale = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "ns": 1e-3, "nsecond": 1e-3, "us": 1.0,
                 "usecond": 1.0, "ms": 1e3, "msecond": 1e3}.get(unit, 1.0)
        rec[row["Metric Name"]] = val * scale
    ids = sorted(launches)
    shapes = parse_shapes("attn")
    if len(ids) != iters * len(shapes):
        raise SystemExit(f"expected {iters * len(shapes)} GEMM launches in {csv_path}, found {len(ids)}")
    per_read, per_write, per_us, per_kernel = {}, {}, {}, {}
    for i, (m, _, _) in enumerate(shapes):
        rec = launches[ids[iters * i + iters - 1]]
        per_kernel[f"M{m}"] = rec["kernel"]
        per_read[f"M{m}"] = int(rec["dram__bytes_read.sum"])
        per_write[f"M{m}"] = int(rec["dram__bytes_write.sum"])
        per_us[f"M{m}"] = round(rec["gpu__time_duration.sum"], 2)
    mean = sum(per_read[k] + per_write[k] for k in per_read) / len(per_read)
    out = {
        "kernel": "the GEMM launch of each shape (per_shape_kernel)",
        "per_shape_kernel": per_kernel,
        "workload": "attention sweep M in {1,16,64,128,256,512}, N=768, K=6144",
        "dram_bytes_per_launch": int(round(mean)),
        "per_shape_dram_read": per_read,
        "per_shape_dram_write": per_write,
        "per_shape_us_under_ncu": per_us,
        "source_hash": source_hash(),
        "command": "ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum "
                   "--clock-control none -k regex:nvfp4_gem --csv --log-file traffic_attn.csv "
                   "python -m nvfp4_block_scaled_gemm_b200.profile_case --shapes attn --iters 2",
    }
    with open(out_path, "w") as f:
        json.dump(out, f, indent=1)
    return out


def run_grouped(experts: int, iters: int, seed: int):
    import numpy as np

    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    tokens = max(synth.MOE_TOPK, synth.MOE_TOKENS * experts // synth.MOE_EXPERTS)
    r = synth.moe_routing(tokens=tokens, experts=experts)
    Mt, N, K = int(r.row_offsets[-1]), synth.MOE_N, synth.HIDDEN_K
    ct, st, ga = nv.quantize(torch.randn((tokens, K), generator=gen, device=dev))
    tok = torch.from_numpy(r.token_of_row.astype(np.int64)).to(dev)
    A, sA = ct[tok].contiguous(), st[tok].contiguous()
    B = torch.empty((experts, N, K // 2), dtype=torch.uint8, device=dev)
    sB = torch.empty((experts, N, K // 16), dtype=torch.uint8, device=dev)
    alpha = torch.empty((experts,), dtype=torch.float32, device=dev)
    for g in range(experts):
        cb, sb, gb = nv.quantize(torch.randn((N, K), generator=gen, device=dev) * 0.02)
        B[g].copy_(cb)
        sB[g].copy_(sb)
        alpha[g] = ga[0] * gb[0]
    off = torch.from_numpy(r.row_offsets.astype(np.int32)).to(dev)
    D = torch.empty((Mt, N), dtype=torch.bfloat16, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        nv.grouped_gemm(A, sA, B, sB, alpha, off, out=D)
    e1.record()
    torch.cuda.synchronize()
    status = nv.get_device_error()
    if status != 0:
        raise SystemExit(f"device error status {status}")
    counts = [int(c) for c in np.diff(r.row_offsets)]
    us = e0.elapsed_time(e1) * 1e3 / iters
    print(f"grouped {experts} experts x [{N} x {K}], {tokens} tokens top-{synth.MOE_TOPK} -> {Mt} rows "
          f"({sum(c > 0 for c in counts)} active, at most {max(counts)} per expert): "
          f"{us:.2f} us/launch (eager), {accounting.grouped_bytes(counts, N, K) / us / 1e3:.0f} GB/s algorithmic")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--shapes", default="512x768x6144")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--traffic-csv", default=None, help="ncu CSV of `--shapes attn --iters 2` (pass --iters 2)")
    ap.add_argument("--traffic-out", default="profiles/traffic_attn_sweep.json")
    ap.add_argument("--grouped", type=int, default=0, help="run the grouped MoE GEMM with this many experts")
    args = ap.parse_args()
    if args.traffic_csv:
        print(summarize_traffic(args.traffic_csv, args.traffic_out, args.iters))
        return
    if args.grouped:
        run_grouped(args.grouped, args.iters, args.seed)
        return
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    for (M, N, K) in parse_shapes(args.shapes):
        gen.manual_seed(args.seed)
        a, sa, ga = nv.quantize(torch.randn((M, K), generator=gen, device=dev))
        b, sb, gb = nv.quantize(torch.randn((N, K), generator=gen, device=dev))
        alpha = float(ga.item() * gb.item())
        D = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.iters):
            nv.gemm(a, sa, b, sb, alpha, out=D)
        e1.record()
        torch.cuda.synchronize()
        status = nv.get_device_error()
        if status != 0:
            raise SystemExit(f"device error status {status}")
        us = e0.elapsed_time(e1) * 1e3 / args.iters
        print(f"{M}x{N}x{K}: {us:.2f} us/launch (eager, includes launch gaps), "
              f"{accounting.gemm_bytes(M, N, K) / us / 1e3:.0f} GB/s algorithmic")


if __name__ == "__main__":
    main()
