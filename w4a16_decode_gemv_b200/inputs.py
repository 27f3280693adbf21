"""Seeded synthetic inputs shaped like the workloads the pages describe.

This module only draws random numbers and rounds them to fp16.  It holds none
of the quantization or GEMV arithmetic, so both the CUDA path and the CPU
oracle can consume what it produces without sharing any of the method.

Recipe (one ``numpy.random.default_rng(seed)`` per workload, draws in this
order for each layer in the listed order):

1. ``W = sigma * standard_normal((N, K))``, rounded once to fp16.
2. ``idx = sort(rng.choice(K, floor(0.01 * K), replace=False))``: the outlier
   input channels (activation outliers sit in a few fixed channels: MIT 6.5940
   Lecture 13 guide, SmoothQuant section, slides 6-7; about 1% of channels:
   EfficientML.ai Lecture 13 summary, AWQ chapter).
3. ``x = standard_normal((M, K))`` with ``x[:, idx] *= 20``, rounded to fp16.

The calibration batch of the quantize+pack workload is drawn the same way as
``x`` with 512 tokens (MIT 6.5940 Lab 4 guide: mean |X| per input channel
collected on 512-token blocks).  The pages' real data (OPT / LLaMA weights,
wikitext-2, pile-val) is not available; these tensors only take its shapes and
its outlier structure.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

OUTLIER_GAIN = 20.0
CALIB_TOKENS = 512


@dataclass
class Layer:
    name: str
    N: int          # output channels (rows of W)
    K: int          # input channels (columns of W)
    W: np.ndarray   # fp16 [N, K]
    x: np.ndarray   # fp16 [M, K]
    outliers: np.ndarray = field(repr=False)


def _fp16_normal(rng: np.random.Generator, shape, scale: float, chunk_rows: int = 1024) -> np.ndarray:
    """Draw ``scale * standard_normal(shape)`` row-chunk by row-chunk, round to fp16.

    numpy's Generator fills C-order arrays from one sequential stream, so the
    chunked draw gives the same values as a single draw of the whole shape while
    holding only one fp64 chunk at a time.
    """
    rows, cols = shape
    out = np.empty(shape, dtype=np.float16)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        block = rng.standard_normal((r1 - r0, cols))
        if scale != 1.0:
            block *= scale
        out[r0:r1] = block.astype(np.float16)
    return out


def outlier_channels(rng: np.random.Generator, K: int) -> np.ndarray:
    return np.sort(rng.choice(K, K // 100, replace=False))


def activations(rng: np.random.Generator, M: int, K: int, idx: np.ndarray) -> np.ndarray:
    x = rng.standard_normal((M, K))
    x[:, idx] *= OUTLIER_GAIN
    return x.astype(np.float16)


def make_layer(rng: np.random.Generator, name: str, N: int, K: int, M: int, sigma: float) -> Layer:
    W = _fp16_normal(rng, (N, K), sigma)
    idx = outlier_channels(rng, K)
    x = activations(rng, M, K, idx)
    return Layer(name, N, K, W, x, idx)


# ---------------------------------------------------------------------------
# The five workloads.  Shapes follow the decode GEMVs of LLaMA-7B and -65B.
# ---------------------------------------------------------------------------

GEMV_4096 = dict(seed=0, sigma=0.02, M=1, layers=[("gemv", 4096, 4096)])
LLAMA7B = dict(seed=1, sigma=0.02, M=1, layers=[
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008)])
LLAMA65B = dict(seed=2, sigma=0.015, M=1, layers=[
    ("attn_8192x8192", 8192, 8192), ("up_22016x8192", 22016, 8192),
    ("down_8192x22016", 8192, 22016)])
SKINNY_M = (1, 4, 8, 12, 16, 32, 64)
SKINNY = dict(seed=3, sigma=0.015, M=max(SKINNY_M), layers=[("skinny_8192", 8192, 8192)])
QUANT = dict(seed=0, sigma=0.02, N=11008, K=4096, alpha=0.5)


def layer_set(spec: dict, only: str | None = None) -> list[Layer]:
    """All layers of a decode workload, drawn in order from one generator.

    ``only`` skips materialising the other layers' weights but still draws
    them, so a single layer is identical to the one in the full set.
    """
    rng = np.random.default_rng(spec["seed"])
    out = []
    for name, N, K in spec["layers"]:
        if only is not None and name != only:
            _skip_layer(rng, N, K, spec["M"])
            continue
        out.append(make_layer(rng, name, N, K, spec["M"], spec["sigma"]))
    return out


def _skip_layer(rng: np.random.Generator, N: int, K: int, M: int, chunk_rows: int = 1024) -> None:
    for r0 in range(0, N, chunk_rows):
        rng.standard_normal((min(N, r0 + chunk_rows) - r0, K))
    idx = outlier_channels(rng, K)
    activations(rng, M, K, idx)


def quant_workload(spec: dict = QUANT):
    """Weight [N, K] and calibration batch [512, K] of the quantize+pack workload."""
    rng = np.random.default_rng(spec["seed"])
    W = _fp16_normal(rng, (spec["N"], spec["K"]), spec["sigma"])
    idx = outlier_channels(rng, spec["K"])
    X = activations(rng, CALIB_TOKENS, spec["K"], idx)
    return W, X, idx


def random_case(seed: int, N: int, K: int, M: int = 1, sigma: float = 0.02, outliers: bool = True):
    """A small seeded case for parity tests (same recipe, arbitrary shape)."""
    rng = np.random.default_rng(seed)
    W = _fp16_normal(rng, (N, K), sigma)
    idx = outlier_channels(rng, K) if outliers else np.zeros(0, dtype=np.int64)
    x = activations(rng, M, K, idx)
    return W, x
