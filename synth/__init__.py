"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds none of the method's arithmetic: it only draws random
numbers (numpy PCG64, seeded) and encodes them into the plain storage types the
inputs use (float32 weights, FP16 scale bit patterns, BF16 activation bit
patterns, int8 trits, raw code bytes).  Nothing here packs, decodes or
multiplies.

Workload recipe (the pages' model shapes, values chosen by the configuration):

* binary weights: float W ~ N(0, 0.02) (then packed by the caller), or raw
  uniform code bytes (every bit an independent fair sign);
* trits: P(-1) = P(+1) = 0.35, P(0) = 0.30;
* FP16 group scales: uniform in [0.005, 0.05], rounded to FP16;
* activations: BF16 bit patterns of x ~ N(0, 1) (float32 rounded to nearest
  even BF16).
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 0xB200

# Qwen3-8B decode-layer matrix shapes (N = output rows, K = input length) and
# its LM head; 27B-class shapes of the hybrid model's projections.
QWEN3_8B_LAYER = {
    "q": (4096, 4096), "k": (1024, 4096), "v": (1024, 4096), "o": (4096, 4096),
    "gate": (12288, 4096), "up": (12288, 4096), "down": (4096, 12288),
}
QWEN3_8B_LM_HEAD = (151936, 4096)
QWEN3_8B_BLOCKS = 36
CLASS27B_LAYER = {
    "q": (6144, 5120), "k": (1024, 5120), "v": (1024, 5120), "o": (5120, 6144),
    "gate": (17408, 5120), "up": (17408, 5120), "down": (5120, 17408),
}
CLASS27B_LM_HEAD = (248320, 5120)
CLASS27B_BLOCKS = 64
PREFILL_SHAPES = [(17408, 5120), (5120, 17408)]
PREFILL_TOKENS = [1, 8, 64, 512, 4096]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def float32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Storage encoding of float32 values as BF16 bit patterns (nearest even).

    Inputs are finite draws of a normal distribution, so no NaN handling."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def weights_normal(g: np.random.Generator, n: int, k: int, std: float = 0.02) -> np.ndarray:
    return g.normal(0.0, std, size=(n, k)).astype(np.float32)


def trits(g: np.random.Generator, n: int, k: int, p_neg=0.35, p_zero=0.30) -> np.ndarray:
    u = g.random(size=(n, k))
    t = np.ones((n, k), dtype=np.int8)
    t[u < p_neg + p_zero] = 0
    t[u < p_neg] = -1
    return t


def scales_uniform(g: np.random.Generator, n: int, groups: int, lo=0.005, hi=0.05) -> np.ndarray:
    """FP16 bit patterns of uniform draws in [lo, hi]."""
    return g.uniform(lo, hi, size=(n, groups)).astype(np.float16).view(np.uint16)


def x_bf16(g: np.random.Generator, batch: int, k: int) -> np.ndarray:
    return float32_to_bf16_bits(g.standard_normal(size=(batch, k)).astype(np.float32))


def code_bytes_uniform(g: np.random.Generator, nbytes: int) -> np.ndarray:
    return g.integers(0, 256, size=nbytes, dtype=np.uint8)


def fp16_bits_to_float32(h: np.ndarray) -> np.ndarray:
    """Storage decoding used to build w = t * s for given-scale packing."""
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float32)
