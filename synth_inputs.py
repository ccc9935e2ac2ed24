"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no BitLinear arithmetic: it only draws random tensors on the
CPU with ``torch.Generator`` so that the CUDA path and the CPU oracle see the
same bytes.

Recipe (the pages' workloads, with no checkpoint or dataset):
  * weights     W ~ N(0, 0.02^2), fp32 [N, K]
  * activations x ~ N(0, 1), fp32 [M, K], then, when outliers are requested,
                  max(1, round(0.001 * M * K)) positions chosen by a random
                  permutation are multiplied by 20; cast to bf16 (round to
                  nearest even) where the workload is bf16.

Layer shapes of a 2.4B-parameter BitNet b1.58 model (hidden 2560, FFN 6912,
GQA k/v width 640) and of 100B-scale layers (hidden 8192, FFN 28672).
"""
from __future__ import annotations

import torch

HIDDEN_2B = 2560
FFN_2B = 6912
KV_2B = 640
LAYERS_2B = 30

# (name, K, N) of one decoder layer's BitLinear products, 2.4B model.
LAYER_SHAPES_2B = [
    ("q", HIDDEN_2B, HIDDEN_2B),
    ("k", HIDDEN_2B, KV_2B),
    ("v", HIDDEN_2B, KV_2B),
    ("o", HIDDEN_2B, HIDDEN_2B),
    ("gate", HIDDEN_2B, FFN_2B),
    ("up", HIDDEN_2B, FFN_2B),
    ("down", FFN_2B, HIDDEN_2B),
]

# The four distinct (K, N) shapes of the 2.4B decode workload.
DECODE_SHAPES_2B = [(2560, 2560), (2560, 640), (2560, 6912), (6912, 2560)]
# 100B-scale decode layers.
DECODE_SHAPES_100B = [(8192, 28672), (28672, 8192)]
# Prefill shapes: (K, N) and token counts.
PREFILL_SHAPES = [(2560, 6912), (6912, 2560)]
PREFILL_TOKENS = [512, 2048, 8192]
SMALL_BATCH_M = [1, 2, 4, 8, 16]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight(N: int, K: int, seed: int = 0, std: float = 0.02) -> torch.Tensor:
    """fp32 [N, K] ~ N(0, std^2)."""
    return torch.randn(N, K, generator=_gen(seed), dtype=torch.float32) * std


def activations(M: int, K: int, seed: int = 0, outliers: bool = True,
                dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """[M, K] ~ N(0, 1) with optional x20 outliers on 0.1% of the entries."""
    g = _gen(seed + 1_000_003)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if outliers:
        count = max(1, round(0.001 * M * K))
        idx = torch.randperm(M * K, generator=g)[:count]
        flat = x.view(-1)
        flat[idx] = flat[idx] * 20.0
    return x.to(dtype)
