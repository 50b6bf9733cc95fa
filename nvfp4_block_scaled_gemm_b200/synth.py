"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no NVFP4 arithmetic: it only draws fp32 source matrices,
random byte patterns and MoE routings from seeded numpy generators.  Both the
CUDA path and the CPU oracle take their inputs from here; quantisation happens
afterwards, on either side, from the fp32 matrices.

Workload shapes ("Peeling the Kernel Onion"):
  * attention projection (M, 768, 6144) and MoE projection (M, 2048, 6144),
    section "The Chain of Reasoning";
  * per-GPU TP8 shapes 6144/8 = 768 and 2048/8 = 256, section
    "The Benchmark Design";
  * saturation sweep from (2048, 2048, 6144) up to (16384, 8192, 8192),
    sections "The Benchmark Design" and "The Results";
  * MoE routing, 256 experts, 8 per token, 512 concurrent tokens, about 16
    rows per expert, section "The Critical Connection to Real Inference".
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ATTN_N, MOE_N, MOE_N_TP8, HIDDEN_K = 768, 2048, 256, 6144
ATTN_SWEEP_M = (1, 16, 64, 128, 256, 512)
MOE_SWEEP_M = (1, 16, 64, 256, 512, 2048)
SATURATION_SHAPES = ((2048, 2048, 6144), (4096, 4096, 6144), (8192, 8192, 8192), (16384, 8192, 8192))
MOE_EXPERTS, MOE_TOPK, MOE_TOKENS, MOE_ZIPF_S = 256, 8, 512, 1.1


def normal(rows: int, K: int, seed: int, std: float = 1.0) -> np.ndarray:
    """fp32 [rows, K] drawn from N(0, std^2)."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((rows, K), dtype=np.float32) * np.float32(std)).astype(np.float32)


def uniform(rows: int, K: int, seed: int, lo: float = -1.0, hi: float = 1.0) -> np.ndarray:
    """fp32 [rows, K] drawn from U[lo, hi)."""
    rng = np.random.default_rng(seed)
    return rng.uniform(lo, hi, size=(rows, K)).astype(np.float32)


def activations_with_outliers(rows: int, K: int, seed: int, p: float = 0.01, factor: float = 20.0) -> np.ndarray:
    """N(0,1) activations where each element independently (probability p)
    is multiplied by `factor`, to stress the per-block scales."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((rows, K), dtype=np.float32)
    mask = rng.random((rows, K)) < p
    X[mask] *= np.float32(factor)
    return X


def random_codes(rows: int, K: int, seed: int) -> np.ndarray:
    """Uniformly random packed E2M1 bytes [rows, K/2] (every nibble value)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)


def random_scales(rows: int, K: int, seed: int, lo: int = 0x28, hi: int = 0x48) -> np.ndarray:
    """Random non-negative, non-NaN E4M3 scale bytes [rows, K/16] drawn
    uniformly from the byte range [lo, hi] (default about 2^-5 .. 2^2)."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=(rows, K // 16), dtype=np.uint8)


@dataclass
class Routing:
    expert_of_row: np.ndarray   # int32 [tokens*topk], non-decreasing
    token_of_row: np.ndarray    # int32 [tokens*topk], which token each grouped row is
    row_offsets: np.ndarray     # int32 [experts+1]


def moe_routing(tokens: int = MOE_TOKENS, experts: int = MOE_EXPERTS, topk: int = MOE_TOPK,
                zipf_s: float = MOE_ZIPF_S, seed: int = 1400) -> Routing:
    """Top-k routing with Zipf expert popularity.

    Expert popularity p_e is proportional to rank_e^-s, ranks being a seeded
    permutation of 1..experts.  Each token draws `topk` distinct experts by
    sequential weighted sampling without replacement.  The (token, expert)
    pairs are then stably sorted by expert, which gives the grouped row order
    and the per-expert row offsets.
    """
    rng = np.random.default_rng(seed)
    ranks = rng.permutation(experts).astype(np.float64) + 1.0
    weight = ranks ** (-zipf_s)
    pairs_tok, pairs_exp = [], []
    for t in range(tokens):
        w = weight.copy()
        for _ in range(topk):
            u = rng.random() * w.sum()
            e = int(np.searchsorted(np.cumsum(w), u, side="right"))
            e = min(e, experts - 1)
            while w[e] == 0.0:          # guard against landing on a taken expert at a boundary
                e = (e + 1) % experts
            pairs_tok.append(t)
            pairs_exp.append(e)
            w[e] = 0.0
    pairs_tok = np.asarray(pairs_tok, np.int32)
    pairs_exp = np.asarray(pairs_exp, np.int32)
    order = np.argsort(pairs_exp, kind="stable")
    counts = np.bincount(pairs_exp, minlength=experts)
    offsets = np.zeros(experts + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    return Routing(pairs_exp[order], pairs_tok[order], offsets)


# Named workloads: (name, M, N, K, source kind, seed).
def attention_sweep():
    return [(f"attn_M{m}", m, ATTN_N, HIDDEN_K, "normal", 1100 + i) for i, m in enumerate(ATTN_SWEEP_M)]


def moe_sweep():
    out = []
    for j, n in enumerate((MOE_N, MOE_N_TP8)):
        for i, m in enumerate(MOE_SWEEP_M):
            out.append((f"moe_N{n}_M{m}", m, n, HIDDEN_K, "moe", 1200 + 10 * j + i))
    return out


def saturation_sweep():
    return [(f"sat_{m}x{n}x{k}", m, n, k, "uniform", 1300 + i) for i, (m, n, k) in enumerate(SATURATION_SHAPES)]


# The six shapes of the results table in "Peeling the Kernel Onion" (section
# "The Results": MoE up-projection at 2K/4K/8K batch, attention QKV at
# 1K/2K/4K batch), for a like-for-like comparison with the numbers printed
# there for another GPU.
PAGES_RESULT_SHAPES = [(2048, 2048, 6144), (4096, 2048, 6144), (8192, 2048, 6144),
                       (1024, 6144, 6144), (2048, 6144, 6144), (4096, 6144, 6144)]


def pages_sweep():
    return [(f"pages_{m}x{n}x{k}", m, n, k, "uniform", 1350 + i) for i, (m, n, k) in enumerate(PAGES_RESULT_SHAPES)]


def source(kind: str, M: int, N: int, K: int, seed: int):
    """fp32 (A [M,K], B [N,K]) for a named source kind."""
    if kind == "normal":
        return normal(M, K, seed), normal(N, K, seed + 100000)
    if kind == "moe":
        return activations_with_outliers(M, K, seed), normal(N, K, seed + 100000, std=0.02)
    if kind == "uniform":
        return uniform(M, K, seed), uniform(N, K, seed + 100000)
    raise ValueError(kind)
