"""Seeded synthetic workloads for the BitLinear hot path.

This module only draws random numbers and lists shapes. It holds none of the
method's arithmetic (no quantisation, packing or contraction), so both the
CPU oracle tests and the CUDA path can take their inputs from it.

Shapes follow the models named on the pages:
  * BitNet b1.58 2B-4T linears (hidden 2560; qkv 2560->3840, o 2560->2560,
    gate+up 2560->13824, down 6912->2560), as in "Core AI model zoo - BitVLA"
    §2 (down_proj K=6912, K % 512 = 256).
  * SigLIP-SO400M vision linears (fc1 1152->4304, fc2 4304->1152), same page §2.
  * BitNet-Embeddings 0.6B (hidden 1024, intermediate 3072) and 270M
    (640, 2048), "BitNet-Embeddings I2_S guide" §2 model table.

Weights are drawn like a trained BitLinear master: N(0, 0.02) or
Laplace(0, 0.02) (the latter gives roughly 40% zero ternary codes, in line with
the 42.8% zero fraction reported for trained ternary weights on the BitMar
summary page). Activations are N(0, 1) with the outlier structure each
workload names. No dataset or checkpoint is used.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np

__all__ = [
    "Layer",
    "Workload",
    "WORKLOADS",
    "weight",
    "activations",
    "rng_for",
]


@dataclass(frozen=True)
class Layer:
    """One BitLinear: y[M, N] = BitLinear(x[M, K]; W[N, K])."""

    name: str
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    key: str
    description: str
    seed: int
    M: Tuple[int, ...]
    layers: Tuple[Layer, ...]
    w_dist: str  # "normal" | "laplace"
    x_dist: str  # "normal" | "student_t" | "outlier_channels" | "outlier_tokens"
    meta: Dict[str, float] = field(default_factory=dict)


_B2 = (
    Layer("qkv", 2560, 3840),
    Layer("o", 2560, 2560),
    Layer("gate_up", 2560, 13824),
    Layer("down", 6912, 2560),
)

WORKLOADS: Dict[str, Workload] = {
    w.key: w
    for w in [
        Workload(
            "decode_2560", "single BitLinear decode, M=1, 2560->2560",
            1000, (1,), (Layer("proj", 2560, 2560),), "normal", "normal"),
        Workload(
            "decode_layer_set", "BitNet-b1.58-2B-4T decode layer set, M=1",
            1001, (1,), _B2, "normal", "student_t", {"df": 3.0}),
        Workload(
            "siglip_m256", "SigLIP-SO400M-shaped vision linears, M=256",
            1002, (256,),
            (Layer("fc1", 1152, 4304), Layer("fc2", 4304, 1152)),
            "normal", "outlier_channels", {"frac": 0.01, "scale": 20.0}),
        Workload(
            "prefill_sweep", "BitNet-2B-shaped prefill sweep",
            1003, (512, 2048, 4096),
            (Layer("qkv", 2560, 3840), Layer("gate_up", 2560, 13824),
             Layer("down", 6912, 2560)),
            "laplace", "normal"),
        Workload(
            "embed_batch", "embedding-model batch, 64 seqs x 512 tokens",
            1004, (32768,),
            (Layer("e06_gate", 1024, 3072), Layer("e06_up", 1024, 3072),
             Layer("e06_down", 3072, 1024), Layer("e27_gate", 640, 2048),
             Layer("e27_up", 640, 2048), Layer("e27_down", 2048, 640)),
            "normal", "outlier_tokens", {"frac": 0.01, "scale": 20.0, "df": 3.0}),
    ]
}

W_SIGMA = 0.02


def rng_for(seed: int, *path: int) -> np.random.Generator:
    """Independent generator for (workload seed, layer index, stream id, ...)."""
    return np.random.default_rng([int(seed), *[int(p) for p in path]])


def weight(N: int, K: int, dist: str, seed: int, layer: int = 0) -> np.ndarray:
    """fp32 master weight [N, K] (torch Linear.weight layout)."""
    g = rng_for(seed, layer, 0)
    if dist == "normal":
        w = g.standard_normal((N, K), dtype=np.float32) * np.float32(W_SIGMA)
    elif dist == "laplace":
        w = g.laplace(0.0, W_SIGMA, size=(N, K)).astype(np.float32)
    else:
        raise ValueError(f"unknown weight distribution {dist!r}")
    return np.ascontiguousarray(w, dtype=np.float32)


def activations(M: int, K: int, dist: str, seed: int, layer: int = 0,
                meta: Dict[str, float] | None = None) -> np.ndarray:
    """fp32 activations [M, K] with the outlier structure of the workload."""
    meta = meta or {}
    g = rng_for(seed, layer, 1, M)
    if dist == "normal":
        x = g.standard_normal((M, K), dtype=np.float32)
    elif dist == "student_t":
        x = g.standard_t(meta.get("df", 3.0), size=(M, K)).astype(np.float32)
    elif dist == "outlier_channels":
        x = g.standard_normal((M, K), dtype=np.float32)
        n_out = max(1, int(round(meta.get("frac", 0.01) * K)))
        # A fixed channel set per K, shared by all tokens.
        ch = rng_for(seed, K, 7).choice(K, size=n_out, replace=False)
        x[:, ch] *= np.float32(meta.get("scale", 20.0))
    elif dist == "outlier_tokens":
        x = g.standard_normal((M, K), dtype=np.float32)
        n_out = max(1, int(round(meta.get("frac", 0.01) * M)))
        rows = rng_for(seed, M, 8).choice(M, size=n_out, replace=False)
        tails = g.standard_t(meta.get("df", 3.0), size=(n_out, K)).astype(np.float32)
        x[rows] = tails * np.float32(meta.get("scale", 20.0))
    else:
        raise ValueError(f"unknown activation distribution {dist!r}")
    return np.ascontiguousarray(x, dtype=np.float32)


def outlier_rows(M: int, seed: int, frac: float = 0.01) -> np.ndarray:
    """Token rows that `activations(..., 'outlier_tokens')` scales (for sampling)."""
    n_out = max(1, int(round(frac * M)))
    return np.sort(rng_for(seed, M, 8).choice(M, size=n_out, replace=False))


def layer_list(key: str) -> List[Tuple[int, Layer]]:
    return list(enumerate(WORKLOADS[key].layers))
