"""Seeded synthetic inputs for the factorised linear: signs, scales, activations.

This module draws random numbers and converts them to the storage dtypes; it holds none
of the layer's arithmetic (no packing, no products, no sums).  Both the CUDA path and the
CPU oracle are fed from it, so neither produces the other's inputs.

Value distributions (the workloads of the factorised-linear benchmarks):
  * sign entries of U and V: i.i.d. Bernoulli(0.5) -> {+1, -1}
  * scale vectors s1, s2: U(0.5, 1.5) * 0.02, rounded to fp16
  * activations x: N(0, 1), rounded to bfloat16 (round to nearest even)
Every draw is keyed by an integer seed plus a tuple of tags (layer, tensor name, ...)
through numpy's SeedSequence, so any single tensor can be regenerated alone.
"""
from __future__ import annotations

import zlib

import numpy as np


def _rng(seed: int, *tags) -> np.random.Generator:
    words = [int(seed) & 0xFFFFFFFF]
    for t in tags:
        if isinstance(t, str):
            words.append(zlib.crc32(t.encode()))
        else:
            words.append(int(t) & 0xFFFFFFFF)
    return np.random.default_rng(np.random.SeedSequence(words))


def signs(rows: int, cols: int, seed: int, *tags) -> np.ndarray:
    """rows x cols int8 in {+1, -1}, each entry +1 with probability 1/2."""
    bits = _rng(seed, "signs", rows, cols, *tags).integers(0, 2, size=(rows, cols), dtype=np.int8)
    return (2 * bits - 1).astype(np.int8)


def random_words(rows: int, words: int, seed: int, *tags) -> np.ndarray:
    """rows x words uint32 of independent fair random bits.

    Under the one-bit-per-sign storage (bit 1 = +1) these are exactly the stored form of
    i.i.d. Bernoulli(0.5) sign matrices; large benchmark weights are drawn this way to
    avoid materialising billions of int8 signs on the host.
    """
    g = _rng(seed, "words", rows, words, *tags)
    return g.integers(0, 1 << 32, size=(rows, words), dtype=np.uint64).astype(np.uint32)


def scales_f16(length: int, seed: int, *tags) -> np.ndarray:
    """length fp16 values U(0.5, 1.5) * 0.02, returned as their uint16 bit patterns."""
    u = _rng(seed, "scales", length, *tags).uniform(0.5, 1.5, size=length) * 0.02
    return u.astype(np.float16).view(np.uint16)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations_bf16(batch: int, n: int, seed: int, *tags) -> np.ndarray:
    """batch x n bfloat16 N(0, 1) activations, as uint16 bit patterns."""
    z = _rng(seed, "x", batch, n, *tags).standard_normal(size=(batch, n)).astype(np.float32)
    return f32_to_bf16_bits(z)


def f16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


# Layer shapes of the benchmark workloads: (name, m_out, n_in, rank).
LLAMA2_7B_LAYERS = [
    ("q", 4096, 4096, 1664),
    ("k", 4096, 4096, 1664),
    ("v", 4096, 4096, 1664),
    ("o", 4096, 4096, 1664),
    ("gate", 11008, 4096, 2432),
    ("up", 11008, 4096, 2432),
    ("down", 4096, 11008, 2432),
]

LLAMA2_70B_LAYERS = [
    ("q", 8192, 8192, 2432),
    ("k", 1024, 8192, 384),
    ("v", 1024, 8192, 384),
    ("o", 8192, 8192, 2432),
    ("gate", 28672, 8192, 3840),
    ("up", 28672, 8192, 3840),
    ("down", 8192, 28672, 3840),
]

SMALL_LAYER = ("single", 512, 512, 128)

PREFILL_SHAPE = ("gate", 11008, 4096, 2432)
PREFILL_BATCHES = (16, 128, 1024, 4096)


# Decode chain of 32 Llama-2-7B-shaped blocks (7 factorised linears each), and a small
# chain with the same wiring for quick checks (hidden 256, MLP 384, ranks 128).
CHAIN_7B_BLOCKS = 32
CHAIN_SMALL_LAYERS = [
    ("q", 256, 256, 128),
    ("k", 256, 256, 128),
    ("v", 256, 256, 128),
    ("o", 256, 256, 128),
    ("gate", 384, 256, 128),
    ("up", 384, 256, 128),
    ("down", 256, 384, 128),
]


def chain_weights(nblocks: int, layers, seed: int):
    """Stored weights of a decode chain on the host: one dict per block,
    {name: (Upk uint32, Vpk uint32, s1 uint16, s2 uint16, m, n, r)}, signs as fair random
    words (the stored form of Bernoulli(0.5) signs), scales as ``scales_f16``."""
    blocks = []
    for b in range(nblocks):
        w = {}
        for (name, m, n, r) in layers:
            w[name] = (random_words(m, (r + 31) // 32, seed, "chain", b, name, "U"),
                       random_words(r, (n + 31) // 32, seed, "chain", b, name, "V"),
                       scales_f16(m, seed, "chain", b, name, "s1"),
                       scales_f16(n, seed, "chain", b, name, "s2"), m, n, r)
        blocks.append(w)
    return blocks


# Activations with the value structure of real decoder activations, for accuracy tests at
# the edges of the kernels' number formats.  All are drawn, then rounded to bfloat16.

def activations_outliers_bf16(batch: int, n: int, seed: int, *tags, per_chunk: int = 3, chunk: int = 1024,
                              lo: float = 1e2, hi: float = 1e4) -> np.ndarray:
    """N(0, 1) activations in which `per_chunk` columns of every `chunk`-column block carry
    outliers of magnitude log-uniform in [lo, hi] with a random sign (the few huge
    "massive activation" channels of decoder hidden states), as bf16 bit patterns."""
    g = _rng(seed, "x-outliers", batch, n, per_chunk, chunk, *tags)
    z = g.standard_normal(size=(batch, n))
    for c0 in range(0, n, chunk):
        width = min(chunk, n - c0)
        for b in range(batch):
            cols = c0 + g.choice(width, size=min(per_chunk, width), replace=False)
            mag = 10.0 ** g.uniform(np.log10(lo), np.log10(hi), size=cols.size)
            z[b, cols] = np.where(g.integers(0, 2, size=cols.size) == 1, mag, -mag)
    return f32_to_bf16_bits(z.astype(np.float32))


def activations_wide_range_bf16(batch: int, n: int, seed: int, *tags, lo_exp: float = -20.0,
                                hi_exp: float = 10.0) -> np.ndarray:
    """Activations of magnitude 2^u, u uniform in [lo_exp, hi_exp], random signs: every
    column block spans the whole dynamic range.  bf16 bit patterns."""
    g = _rng(seed, "x-wide", batch, n, *tags)
    mag = np.exp2(g.uniform(lo_exp, hi_exp, size=(batch, n)))
    sign = np.where(g.integers(0, 2, size=(batch, n)) == 1, 1.0, -1.0)
    return f32_to_bf16_bits((sign * mag).astype(np.float32))


def activations_token_scaled_bf16(n: int, seed: int, token_scales, *tags) -> np.ndarray:
    """One row per entry of `token_scales`: N(0, 1) activations times that factor, rounded
    to bfloat16 (tokens of very different magnitude in one call)."""
    sc = np.asarray(token_scales, dtype=np.float64)
    z = _rng(seed, "x-token-scaled", sc.size, n, *tags).standard_normal(size=(sc.size, n))
    return f32_to_bf16_bits((z * sc[:, None]).astype(np.float32))


# Inputs of the LB-ADMM initialiser: a dense weight matrix and the start block.

def weights_bf16(m: int, n: int, seed: int, *tags, spread: float = 0.5) -> np.ndarray:
    """m x n bfloat16 weights N(0, 1) * exp(spread N(0, 1))_row * exp(spread N(0, 1))_col
    * 0.02 (Gaussian entries with log-normal row and column magnitudes, the structure the
    per-row and per-column scales of the factorisation capture), as bf16 bit patterns."""
    g = _rng(seed, "weights", m, n, *tags)
    rows = np.exp(spread * g.standard_normal(m))
    cols = np.exp(spread * g.standard_normal(n))
    z = g.standard_normal((m, n)) * rows[:, None] * cols[None, :] * 0.02
    return f32_to_bf16_bits(z.astype(np.float32))


def gaussian_f32(rows: int, cols: int, seed: int, *tags) -> np.ndarray:
    """rows x cols float32 standard normal draws (the initialiser's start block)."""
    return _rng(seed, "gauss", rows, cols, *tags).standard_normal(size=(rows, cols)).astype(np.float32)
