"""Seeded synthetic inputs for the QLoRA linear layer.

This module only draws random numbers and rounds them to bf16 storage; it holds
none of the layer's arithmetic (no quantisation, no matmul).  Both the CUDA
path and the CPU oracle take their inputs from here, so they see identical
bytes.

Recipe (one independent stream per tensor, ``numpy.random.default_rng([seed,
tensor_id])``):

* W0 ~ N(0, 0.02), A ~ N(0, 1/r) (the tiny layer uses 1/8), B ~ N(0, 0.01),
  X ~ N(0, 1), dY ~ N(0, 1); "N(0, s)" is read as standard deviation s.
* Quantisation sweep matrices: every element is independently replaced, with
  probability 0.01, by an outlier drawn from N(0, 0.2).
* fp32 draws are rounded to bf16 with round-to-nearest-even on the bit
  pattern, and handed out as ``uint16`` bit arrays (or fp32 copies of them).

Tensor ids: W0=0, A=1, B=2, X=3, dY=4, outlier mask=5, outlier values=6.
Projections of one layer set use their index as the seed (``seed = p``), so
every weight matrix is distinct; rank rho of a data-parallel run draws its
tokens X and dY with ``seed = p + 1000 * rho``.
"""
from __future__ import annotations

import numpy as np

TID_W0, TID_A, TID_B, TID_X, TID_DY, TID_MASK, TID_OUTLIER = range(7)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # NaN never occurs in these draws; keep the plain rounding rule.
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(seed: int, tid: int, shape, std: float) -> np.ndarray:
    rng = np.random.default_rng([seed, tid])
    x = rng.standard_normal(size=shape, dtype=np.float32)
    x *= np.float32(std)
    return f32_to_bf16_bits(x)


def weight(d: int, k: int, seed: int = 0, std: float = 0.02, outliers: bool = False) -> np.ndarray:
    """W0 as a (d, k) uint16 bf16-bit array."""
    rng = np.random.default_rng([seed, TID_W0])
    w = rng.standard_normal(size=(d, k), dtype=np.float32) * np.float32(std)
    if outliers:
        mask = np.random.default_rng([seed, TID_MASK]).random(size=(d, k), dtype=np.float32) < np.float32(0.01)
        vals = np.random.default_rng([seed, TID_OUTLIER]).standard_normal(size=(d, k), dtype=np.float32)
        vals *= np.float32(0.2)
        w = np.where(mask, vals, w)
    return f32_to_bf16_bits(w)


def lora_a(r: int, k: int, seed: int = 0, std: float | None = None) -> np.ndarray:
    return _normal_bf16(seed, TID_A, (r, k), (1.0 / r) if std is None else std)


def lora_b(d: int, r: int, seed: int = 0, std: float = 0.01) -> np.ndarray:
    return _normal_bf16(seed, TID_B, (d, r), std)


def activations(m: int, k: int, seed: int = 0, std: float = 1.0) -> np.ndarray:
    return _normal_bf16(seed, TID_X, (m, k), std)


def grad_output(m: int, d: int, seed: int = 0, std: float = 1.0) -> np.ndarray:
    return _normal_bf16(seed, TID_DY, (m, d), std)


def layer(m: int, d: int, k: int, r: int, seed: int = 0, a_std: float | None = None,
          outliers: bool = False) -> dict:
    """All inputs of one QLoRA linear layer as bf16 bit arrays."""
    return {
        "W0": weight(d, k, seed, outliers=outliers),
        "A": lora_a(r, k, seed, a_std),
        "B": lora_b(d, r, seed),
        "X": activations(m, k, seed),
        "dY": grad_output(m, d, seed),
    }


# Workloads, named by what they are.  Sizes follow the layer shapes they model.
PROJ_7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
PROJ_65B = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
            ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]

WORKLOADS = {
    "tiny_512": dict(proj=[("w", 512, 512)], m=16, r=8, alpha=16.0, a_std=1.0 / 8, bwd=True),
    "llama7b_proj_set_m4096": dict(proj=PROJ_7B, m=4096, r=64, alpha=16.0, a_std=None, bwd=True),
    "decode_28672x8192": dict(proj=[("up", 28672, 8192), ("down", 8192, 28672)], m=(1, 8, 32, 128),
                              r=16, alpha=32.0, a_std=None, bwd=False),
    "llama65b_block_m8192": dict(proj=PROJ_65B, m=8192, r=64, alpha=16.0, a_std=None, bwd=True),
    # the same sets with q, k, v and gate, up grouped: each group reads one X
    "llama7b_proj_set_m4096_grouped": dict(proj=PROJ_7B, m=4096, r=64, alpha=16.0, a_std=None, bwd=True,
                                           groups=[[0, 1, 2], [3], [4, 5], [6]]),
    "llama65b_block_m8192_grouped": dict(proj=PROJ_65B, m=8192, r=64, alpha=16.0, a_std=None, bwd=True,
                                         groups=[[0, 1, 2], [3], [4, 5], [6]]),
    # the same sets with adapter dropout p = 0.05 (the lora_dropout of the PEFT configuration)
    "llama7b_proj_set_m4096_dropout": dict(proj=PROJ_7B, m=4096, r=64, alpha=16.0, a_std=None, bwd=True,
                                           dropout=0.05),
    "llama65b_block_m8192_dropout": dict(proj=PROJ_65B, m=8192, r=64, alpha=16.0, a_std=None, bwd=True,
                                         dropout=0.05),
    "proj_q_4096": dict(proj=[("q", 4096, 4096)], m=4096, r=64, alpha=16.0, a_std=None, bwd=True),
    "quant_sweep": dict(proj=[("sq", 4096, 4096), ("rect", 4096, 11008)], outliers=True),
    "merge_sweep": dict(proj=[("q", 4096, 4096), ("gate", 11008, 4096), ("down", 4096, 11008)], r=64, alpha=16.0),
}
