"""Seeded synthetic inputs for the Sparse-BitLinear forward.

This module only draws random numbers and rounds them to the storage type a
caller asks for; it holds none of the layer's arithmetic (no mask, scale,
quantisation or contraction).  Both the CUDA path's tests/benchmark and the
CPU oracle take their inputs from here, so the two sides see identical bytes.

Recipe (the workloads of the model cards and the Sparse-BitNet Guide, which
train on web text; no dataset is used here, these draws stand in for it):

* latent weights ``W``: fp32 ``[O, K]`` drawn i.i.d. N(0, sigma^2), sigma = 0.02
  by default (a typical initialisation spread for the transformer skeletons
  the model cards name; the pages print no weight statistics);
* activations ``x``: N(0, 1) drawn in fp32, optionally with each element
  independently (Bernoulli(p)) multiplied by an outlier factor, then rounded
  to bf16 with round-to-nearest-even; returned as the raw bf16 bit pattern
  (``uint16``) and as the exactly widened fp32 values.

Every tensor has its own stream: ``numpy.random.Generator(PCG64)`` seeded from
``SeedSequence([seed, tag])`` where ``tag`` names the tensor, so adding a tensor
never shifts the draws of another.
"""
from __future__ import annotations

import zlib

import numpy as np


def _rng(seed: int, tag: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), zlib.crc32(tag.encode())])))


def latent_weights(O: int, K: int, seed: int = 0, tag: str = "W", sigma: float = 0.02) -> np.ndarray:
    """fp32 [O, K] latent weights, i.i.d. N(0, sigma^2)."""
    g = _rng(seed, tag)
    w = g.standard_normal((O, K), dtype=np.float32)
    return (w * np.float32(sigma)).astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns.

    Storage conversion only.  NaN inputs are not expected from the generators.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activations(T: int, K: int, seed: int = 0, tag: str = "x", outlier_p: float = 0.0,
                outlier_scale: float = 20.0):
    """bf16 activations [T, K]: returns (bits uint16, values fp32).

    ``outlier_p`` > 0 multiplies each element independently with probability
    ``outlier_p`` by ``outlier_scale`` before rounding to bf16.
    """
    g = _rng(seed, tag)
    x = g.standard_normal((T, K), dtype=np.float32)
    if outlier_p > 0.0:
        hit = g.random((T, K)) < outlier_p
        x = np.where(hit, x * np.float32(outlier_scale), x).astype(np.float32)
    bits = f32_to_bf16_bits(x)
    return bits, bf16_bits_to_f32(bits)


def output_grads(T: int, O: int, seed: int = 0, tag: str = "dY") -> np.ndarray:
    """fp32 [T, O] loss gradients at the layer output, i.i.d. N(0, 1)."""
    return _rng(seed, tag).standard_normal((T, O), dtype=np.float32)


# Layer shapes (K -> O) of the workloads.  Qwen2.5-0.5B skeleton: d_model 896,
# d_ffn 4864, 14 heads / 2 KV heads of width 64 (halo card, "Recipe").  The
# hidden-2048 / FFN-7168 stack follows the tritter-500m card's shapes.
QWEN05_LAYER = (
    ("q", 896, 896), ("k", 896, 128), ("v", 896, 128), ("o", 896, 896),
    ("gate", 896, 4864), ("up", 896, 4864), ("down", 4864, 896),
)
QWEN05_FFN = (("gate", 896, 4864), ("up", 896, 4864), ("down", 4864, 896))
H2048_STACK = (
    ("q", 2048, 2048), ("o", 2048, 2048), ("gate", 2048, 7168), ("up", 2048, 7168), ("down", 7168, 2048),
)
SWEEP_LAYERS = (("up", 2048, 7168), ("down", 7168, 2048))
SWEEP_PATTERNS = ((2, 4), (3, 4), (6, 8))
SWEEP_TOKENS = (1, 8, 64, 512, 4096)
