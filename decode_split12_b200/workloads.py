"""Seeded synthetic inputs for the Split12 workloads.

This module only draws numbers.  It holds none of the format's arithmetic
(no exponent windows, no codes, no escapes), so both the CUDA path and the
CPU oracle can be fed from it without sharing any of the method.

Recipes (one ``numpy.random.Generator(PCG64(seed + tensor_index))`` per
tensor, FP32 draws rounded to BF16 with round-to-nearest-even):

* ``single``   4096 x 4096, N(0, 0.02), 0.1 % of positions (uniform, without
  replacement) multiplied by U(10, 100); x ~ N(0, 1), batch 1.
* ``llama8b``  one Llama-style 8B decoder layer: q, o 4096 x 4096; k, v
  1024 x 4096; gate, up 14336 x 4096; down 4096 x 14336.  Each matrix is
  Student-t(5) divided by sqrt(5/3) (unit variance) and by sqrt(in_features).
  Activations N(0, 1) at batch 1, 4, 8.
* ``escape``   8192 x 8192 with an exact escape fraction: ordinary weights are
  N(0, 0.02) redrawn until their exponent field lies in [109, 123] (15
  values, one window); round(rate * R * C) positions, uniform without
  replacement, get exponent fields uniform in [140, 150] with random sign
  and mantissa, so every one of them must be an escape.
* ``mlp70b``   28672 x 8192 and 8192 x 28672, N(0, 1/sqrt(in)) with 0.05 %
  outliers x U(10, 100); activations N(0, 1) at M = 16 .. 256.
* ``stack``    32 ``llama8b`` layers (seed = layer index) plus an 8-expert
  MoE block (gate, up 14336 x 4096; down 4096 x 14336) with 64 tokens each
  routed to 2 distinct experts drawn uniformly.

The pages' own measurements are on real checkpoints (GLM-5.2, Qwen3-8B,
Llama 405B, Mistral 7B) that are not available; these shapes and
distributions stand in for them.
"""
from __future__ import annotations

import math

import numpy as np

LLAMA8B_SHAPES = {
    "q": (4096, 4096),
    "k": (1024, 4096),
    "v": (1024, 4096),
    "o": (4096, 4096),
    "gate": (14336, 4096),
    "up": (14336, 4096),
    "down": (4096, 14336),
}
MLP70B_SHAPES = {"up": (28672, 8192), "down": (8192, 28672)}
MOE_SHAPES = {"gate": (14336, 4096), "up": (14336, 4096), "down": (4096, 14336)}
ESCAPE_RATES = (0.0003, 0.0023, 0.02, 0.10)


def rng_for(seed: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed + index))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """FP32 -> BF16 bit patterns (uint16), round to nearest even.  NaNs keep
    a quiet NaN pattern."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_with_outliers(rows: int, cols: int, std: float, outlier_frac: float,
                         seed: int, index: int = 0) -> np.ndarray:
    g = rng_for(seed, index)
    w = g.standard_normal((rows, cols), dtype=np.float32) * np.float32(std)
    n_out = int(round(outlier_frac * rows * cols))
    if n_out:
        pos = g.choice(rows * cols, size=n_out, replace=False)
        w.reshape(-1)[pos] *= g.uniform(10.0, 100.0, size=n_out).astype(np.float32)
    return to_bf16_bits(w)


def student_t_scaled(rows: int, cols: int, seed: int, index: int = 0, nu: float = 5.0) -> np.ndarray:
    g = rng_for(seed, index)
    t = g.standard_t(nu, size=(rows, cols)).astype(np.float32)
    scale = 1.0 / math.sqrt(nu / (nu - 2.0)) / math.sqrt(cols)
    return to_bf16_bits(t * np.float32(scale))


def activations(m: int, k: int, seed: int, index: int = 1000) -> np.ndarray:
    g = rng_for(seed, index)
    return to_bf16_bits(g.standard_normal((m, k), dtype=np.float32))


def single_tensor(seed: int = 0, rows: int = 4096, cols: int = 4096):
    w = normal_with_outliers(rows, cols, 0.02, 0.001, seed, 0)
    x = activations(1, cols, seed)
    return w, x


def llama8b_layer(seed: int = 0, batch: int = 1, names=None):
    names = list(LLAMA8B_SHAPES) if names is None else names
    mats = {}
    for i, name in enumerate(LLAMA8B_SHAPES):
        if name not in names:
            continue
        r, c = LLAMA8B_SHAPES[name]
        mats[name] = student_t_scaled(r, c, seed, i)
    xs = {name: activations(batch, LLAMA8B_SHAPES[name][1], seed, 1000 + i)
          for i, name in enumerate(LLAMA8B_SHAPES) if name in names}
    return mats, xs


def escape_stress(rate: float, seed: int = 0, rows: int = 8192, cols: int = 8192):
    """Returns (w, n_escapes_planted)."""
    g = rng_for(seed, 0)
    n = rows * cols
    w = to_bf16_bits(g.standard_normal(n, dtype=np.float32) * np.float32(0.02))
    while True:
        e = (w >> 7) & 0xFF
        bad = (e < 109) | (e > 123)
        nb = int(bad.sum())
        if nb == 0:
            break
        w[bad] = to_bf16_bits(g.standard_normal(nb, dtype=np.float32) * np.float32(0.02))
    n_esc = int(round(rate * n))
    if n_esc:
        pos = g.choice(n, size=n_esc, replace=False)
        sign = g.integers(0, 2, size=n_esc, dtype=np.uint16)
        expo = g.integers(140, 151, size=n_esc, dtype=np.uint16)
        mant = g.integers(0, 128, size=n_esc, dtype=np.uint16)
        w[pos] = (sign << 15) | (expo << 7) | mant
    return w.reshape(rows, cols), n_esc


def mlp70b(name: str, seed: int = 0):
    r, c = MLP70B_SHAPES[name]
    idx = list(MLP70B_SHAPES).index(name)
    return normal_with_outliers(r, c, 1.0 / math.sqrt(c), 0.0005, seed, idx)


def moe_routing(tokens: int = 64, experts: int = 8, top_k: int = 2, seed: int = 0) -> np.ndarray:
    """tokens x top_k expert ids, distinct per token, uniform."""
    g = rng_for(seed, 5000)
    return np.stack([g.choice(experts, size=top_k, replace=False) for _ in range(tokens)])


def random_bf16_patterns(n: int, seed: int = 0) -> np.ndarray:
    """Uniformly random 16-bit patterns (every exponent, NaN and Inf included)."""
    return rng_for(seed, 7).integers(0, 1 << 16, size=n, dtype=np.uint32).astype(np.uint16)
