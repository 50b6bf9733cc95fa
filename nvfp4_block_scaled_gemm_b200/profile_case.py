"""Run a few NVFP4 GEMMs of given shapes, for profiling one kernel under ncu.

    python -m nvfp4_block_scaled_gemm_b200.profile_case --shapes 512x768x6144 --iters 3
    python -m nvfp4_block_scaled_gemm_b200.profile_case --shapes attn --iters 2

`attn` expands to the attention-projection sweep (M in {1,16,64,128,256,512},
N=768, K=6144).  Inputs are seeded N(0,1) fp32 quantised on the GPU; every
launch of a shape uses the same buffers (ncu flushes the caches between its
replay passes, so DRAM counters still see the compulsory traffic).
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--shapes", default="512x768x6144")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1)
    args = ap.parse_args()
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
