"""Shapes, seeds and distributions of the synthetic workloads (no arithmetic).

The pages size the problem by decoder-layer linears of 3B/7B/100B-class models
("1.58-bit 大模型极限量化实战", chenxutan.com/d/5049.html §5.2 and §6.1: Q/K/V/O
projections and the MLP linears become BitLinear; decode reads every weight
once per token).  Every matrix is W ~ N(0, σ²) float32 (the layer's own init
draws randn·0.02, §4.2) and every activation is N(0, 1), stored as bfloat16
except in the tiny case; "outliers" adds 0.1% ×20 channels (§6.2).
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Linear:
    name: str
    K: int          # input features
    N: int          # output features
    M: int          # tokens
    seed: int       # weight stream
    x_seed: int     # activation stream
    w_std: float
    outliers: bool
    x_dtype: str = "bf16"


HIDDEN_7B, FFN_7B = 4096, 11008
_LAYER = (("q", HIDDEN_7B, HIDDEN_7B), ("k", HIDDEN_7B, HIDDEN_7B), ("v", HIDDEN_7B, HIDDEN_7B),
          ("o", HIDDEN_7B, HIDDEN_7B), ("gate", HIDDEN_7B, FFN_7B), ("up", HIDDEN_7B, FFN_7B),
          ("down", FFN_7B, HIDDEN_7B))


def tiny() -> Linear:
    """M=1, K=N=256, float32 x and W, seed 0."""
    return Linear("tiny", 256, 256, 1, 0, 0, 0.02, False, "f32")


def decode_7b_layer_set(M: int = 1, layer: int = 0, base_seed: int = 2000) -> list[Linear]:
    """The seven linears of one 7B-shaped decoder layer, each with its own input."""
    out = []
    for i, (name, K, N) in enumerate(_LAYER):
        s = base_seed + 7 * layer + i
        out.append(Linear(name, K, N, M, s, s, 0.02, True))
    return out


def batched_decode_100b(K: int, N: int, M: int) -> Linear:
    """One 100B-shaped matrix, (K, N) ∈ {(8192, 28672), (28672, 8192)}."""
    shape = 0 if (K, N) == (8192, 28672) else 1
    return Linear(f"100b_K{K}_N{N}", K, N, M, 3000 + shape, 3000 + 100 * M + shape, 0.015, False)


def prefill(K: int, N: int, M: int = 2048) -> Linear:
    """Prefill of M tokens; (K, N) ∈ {(4096, 4096), (4096, 11008), (11008, 4096)}."""
    shape = {(4096, 4096): 0, (4096, 11008): 1, (11008, 4096): 2}[(K, N)]
    return Linear(f"prefill_K{K}_N{N}", K, N, M, 4000 + shape, 4100 + shape, 0.02, True)


def packed_bytes(spec: Linear) -> int:
    return spec.N * 16 * ((spec.K + 63) // 64)
