"""Seeded synthetic inputs for the Sparse-BitLinear layer shapes.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from it.  Every array is produced on the host with numpy ``PCG64`` so that the
identical bytes can be copied to the GPU and handed to the oracle.

Distributions (Sparse-BitNet experiments on Qwen2.5 backbones; BitNet b1.58
2B4T layer shapes):
  * master weights W ~ N(0, 0.02) fp32, row-major [d_out, d_in];
  * activations X ~ N(0, 1) rounded to bf16 (round-to-nearest-even),
    row-major [tokens, d_in]; the small single-layer case additionally scales
    1% of the input channels (at least one, picked by a seeded permutation)
    by 20 to create outlier channels;
  * output gradients dY ~ N(0, 1) bf16, row-major [tokens, d_out].
Sub-seeds: seed*16 + {0: W, 1: X, 2: dY, 3: outlier channels}, plus the layer
index * 256 so every linear of a workload gets its own stream.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple

import numpy as np


def _rng(seed: int, sub: int, layer: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed * 16 + sub + layer * 256))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even) and return the uint16 bit patterns.
    Input generation only: turns N(0,1) draws into bf16 test activations."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def master_weights(d_out: int, d_in: int, seed: int, layer: int = 0, std: float = 0.02) -> np.ndarray:
    return (_rng(seed, 0, layer).standard_normal((d_out, d_in), dtype=np.float32) * np.float32(std))


def activations(tokens: int, d_in: int, seed: int, layer: int = 0,
                outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> np.ndarray:
    x = _rng(seed, 1, layer).standard_normal((tokens, d_in), dtype=np.float32)
    if outlier_frac > 0.0:
        n_out = max(1, int(round(outlier_frac * d_in)))
        cols = _rng(seed, 3, layer).permutation(d_in)[:n_out]
        x[:, cols] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x)


def output_grad(tokens: int, d_out: int, seed: int, layer: int = 0) -> np.ndarray:
    return f32_to_bf16_bits(_rng(seed, 2, layer).standard_normal((tokens, d_out), dtype=np.float32))


@dataclass
class Linear:
    name: str
    d_in: int
    d_out: int
    inp: str = ""  # the activation it reads: linears with the same name read one tensor ("": its own)


@dataclass
class Workload:
    name: str
    seed: int
    tokens: List[int]
    linears: List[Linear]
    patterns: List[Tuple[int, int]]
    mode: str                      # "forward", "decode" or "train"
    outlier_frac: float = 0.0
    notes: str = ""
    extra: dict = field(default_factory=dict)


# The five layer workloads of the Sparse-BitNet / BitNet b1.58 2B4T shapes.
WORKLOADS = {
    "single_256x128": Workload(
        "single_256x128", 0, [64], [Linear("layer", 256, 128)], [(6, 8)], "forward",
        outlier_frac=0.01,
        notes="one Sparse-BitLinear layer, T=64, K=256, O=128, 6:8, 1% outlier channels x20"),
    "qwen05b_mlp": Workload(
        "qwen05b_mlp", 2, [4096],
        [Linear("gate", 896, 4864, "x"), Linear("up", 896, 4864, "x"), Linear("down", 4864, 896, "act")],
        [(6, 8), (2, 4)], "forward",
        notes="Qwen2.5-0.5B MLP linears, T=4096, forward at 6:8 and 2:4"),
    "qwen15b_decoder": Workload(
        "qwen15b_decoder", 3, [8192],
        [Linear("q", 1536, 1536, "x"), Linear("k", 1536, 256, "x"), Linear("v", 1536, 256, "x"),
         Linear("o", 1536, 1536, "attn"), Linear("gate", 1536, 8960, "h"), Linear("up", 1536, 8960, "h"),
         Linear("down", 8960, 1536, "act")],
        [(7, 8), (6, 8), (5, 8), (4, 8), (3, 8), (2, 8), (2, 4)], "forward",
        notes="Qwen2.5-1.5B decoder linears, T=8192, N:M sweep"),
    "bitnet2b_decode": Workload(
        "bitnet2b_decode", 4, [1, 4, 16],
        [Linear("up", 2560, 6912), Linear("down", 6912, 2560)], [(2, 4)], "decode",
        notes="BitNet-2B decode GEMV from pre-packed 2:4 ternary weights"),
    "qwen3b_train": Workload(
        "qwen3b_train", 5, [16384],
        [Linear("up", 2048, 11008), Linear("down", 11008, 2048)], [(6, 8)], "train",
        notes="Qwen2.5-3B training step: re-mask, forward, Dual-STE backward, 6:8"),
}
