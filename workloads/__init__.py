"""Seeded synthetic inputs and the workload shapes.

This module is shared by the tests, the benchmark and the smoke check.  It
holds shapes and random-number draws only -- none of the quantization or
matmul arithmetic -- so the CPU oracle and the CUDA library can both be fed
from it without sharing any of the method's code.

Distributions: weights W ~ N(0, 0.02) and activations x ~ N(0, 1), both drawn
in fp32 and rounded to bf16.  The pages measure on real PersonaPlex weights
and recordings, which are not available; these Gaussians stand in for them.

Seeds: workload c (1-based, in the order below) uses seed c-1; tensor t inside
it is drawn from ``torch.Generator().manual_seed(1000 * seed + t)`` (CPU) or
the CUDA generator with the same seed when the workload is too large to draw
on the host.

Shapes (from the pages):
* the temporal transformer is 32 layers, 4096 wide, ~7B parameters; its
  feed-forward is SwiGLU (Swift/MLX blog, architecture diagram; GeekNews
  summary, "Pipeline pemrosesan suara"), with 11264-wide gate/up, and a text
  head 4096 -> 32000 (32k SentencePiece vocabulary, ONNX README "Files in this
  variant");
* the depformer is 6 layers, 1024 wide, with a separate weight slice for each
  of 16 codebook steps stored as one stacked tensor (Swift/MLX blog,
  "Depformer: per-step weight switching").
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import torch

W_STD = 0.02
X_STD = 1.0


@dataclass(frozen=True)
class Proj:
    name: str
    N: int  # output features (weight rows)
    K: int  # input features (weight columns)


TEMPORAL_LAYER: Tuple[Proj, ...] = (
    Proj("q", 4096, 4096),
    Proj("k", 4096, 4096),
    Proj("v", 4096, 4096),
    Proj("o", 4096, 4096),
    Proj("gate", 11264, 4096),
    Proj("up", 11264, 4096),
    Proj("down", 4096, 11264),
)
TEXT_HEAD = Proj("head", 32000, 4096)
TEMPORAL_LAYERS = 32

DEPFORMER_LAYER: Tuple[Proj, ...] = (
    Proj("q", 1024, 1024),
    Proj("k", 1024, 1024),
    Proj("v", 1024, 1024),
    Proj("o", 1024, 1024),
    Proj("gate", 2816, 1024),
    Proj("up", 2816, 1024),
    Proj("down", 1024, 2816),
)
DEPFORMER_HEAD = Proj("head", 2048, 1024)
DEPFORMER_LAYERS = 6
DEPFORMER_STEPS = 16

BATCHED_M = (4, 64, 256)

# Workload names, in the seed order described above.
WORKLOADS = ("tiny_1024", "temporal_layer", "temporal_stream", "depformer_steps", "batched_layer")


def seed_of(workload: str) -> int:
    return WORKLOADS.index(workload)


def stream_projs() -> List[Proj]:
    """The full temporal weight stream: 32 layers x 7 projections + text head."""
    out = []
    for layer in range(TEMPORAL_LAYERS):
        out += [Proj(f"L{layer}.{p.name}", p.N, p.K) for p in TEMPORAL_LAYER]
    out.append(TEXT_HEAD)
    return out


def depformer_projs() -> List[Proj]:
    """Per-step depformer projections (each stored stacked over 16 steps)."""
    out = []
    for layer in range(DEPFORMER_LAYERS):
        out += [Proj(f"D{layer}.{p.name}", p.N, p.K) for p in DEPFORMER_LAYER]
    out.append(DEPFORMER_HEAD)
    return out


def generator(seed: int, tensor: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + tensor)
    return g


def gaussian_bf16(shape, std: float, seed: int, tensor: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 with a dedicated generator, rounded to bf16."""
    g = generator(seed, tensor, device)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    return (t * std).to(torch.bfloat16)


def weight(N: int, K: int, seed: int, tensor: int, device="cpu") -> torch.Tensor:
    return gaussian_bf16((N, K), W_STD, seed, tensor, device)


def activation(M: int, K: int, seed: int, tensor: int, device="cpu") -> torch.Tensor:
    return gaussian_bf16((M, K), X_STD, seed, tensor, device)


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor's bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
