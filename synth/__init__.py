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

# Decode attention of Qwen3-8B ("1-bit Bonsai 8B" notes, Table 1: 32 query /
# 8 KV heads, hidden 4096, so head dimension 128; 65,536-token context).
QWEN3_8B_ATTN = {"hq": 32, "hkv": 8, "d": 128, "max_ctx": 65536}


def kv4_cache_bytes(g: np.random.Generator, b: int, hkv: int, l_cap: int, d: int, s_lo=0.02, s_hi=0.2):
    """Random 4-bit cache contents: uniform code bytes, FP16 scales uniform in
    [s_lo, s_hi], FP16 biases -7.5 s (1 + u), u uniform in [-0.1, 0.1], packed
    as (s | z << 16).  Returns (codes uint8 [b][hkv][l_cap][d/2], params uint32
    [b][hkv][l_cap][d/128])."""
    codes = g.integers(0, 256, size=(b, hkv, l_cap, d // 2), dtype=np.uint8)
    s = g.uniform(s_lo, s_hi, size=(b, hkv, l_cap, d // 128))
    z = -7.5 * s * (1.0 + g.uniform(-0.1, 0.1, size=s.shape))
    sb = s.astype(np.float16).view(np.uint16).astype(np.uint32)
    zb = z.astype(np.float16).view(np.uint16).astype(np.uint32)
    return codes, (sb | (zb << 16)).astype(np.uint32)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def float32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Storage encoding of float32 values as BF16 bit patterns (nearest even).

    Inputs are finite draws of a normal distribution, so no NaN handling."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def weights_normal(g: np.random.Generator, n: int, k: int, std: float = 0.02) -> np.ndarray:
    w = g.standard_normal(size=(n, k), dtype=np.float32)
    w *= np.float32(std)
    return w


def trits(g: np.random.Generator, n: int, k: int) -> np.ndarray:
    """P(-1) = P(+1) = 7/20 = 0.35, P(0) = 6/20 = 0.30."""
    u = g.integers(0, 20, size=(n, k), dtype=np.uint8)
    t = np.ones((n, k), dtype=np.int8)
    t[u < 13] = 0
    t[u < 7] = -1
    return t


def scales_uniform(g: np.random.Generator, n: int, groups: int, lo=0.005, hi=0.05) -> np.ndarray:
    """FP16 bit patterns of uniform draws in [lo, hi]."""
    return g.uniform(lo, hi, size=(n, groups)).astype(np.float16).view(np.uint16)


def x_bf16(g: np.random.Generator, batch: int, k: int) -> np.ndarray:
    return float32_to_bf16_bits(g.standard_normal(size=(batch, k), dtype=np.float32))


def code_bytes_uniform(g: np.random.Generator, nbytes: int) -> np.ndarray:
    return g.integers(0, 256, size=nbytes, dtype=np.uint8)


def fp16_bits_to_float32(h: np.ndarray) -> np.ndarray:
    """Storage decoding used to build w = t * s for given-scale packing."""
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float32)


# ------------------------------------------------------------ on the device
# Full-size workloads (up to 1.3e9 weights) are drawn on the GPU with a seeded
# torch generator; the oracle reads back whatever rows it checks.
def device_generator(seed: int, device="cuda"):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return gen


def device_weights_normal(gen, n: int, k: int, std: float = 0.02, device="cuda"):
    import torch
    return torch.randn((n, k), generator=gen, device=device, dtype=torch.float32) * std


def device_trits(gen, n: int, k: int, device="cuda"):
    import torch
    u = torch.randint(0, 20, (n, k), generator=gen, device=device, dtype=torch.int16)
    t = torch.ones((n, k), device=device, dtype=torch.int8)
    t[u < 13] = 0
    t[u < 7] = -1
    return t


def device_scales_uniform(gen, n: int, groups: int, lo=0.005, hi=0.05, device="cuda"):
    """FP16 bit patterns (int16 tensor) of uniform draws in [lo, hi]."""
    import torch
    u = torch.rand((n, groups), generator=gen, device=device, dtype=torch.float32)
    return (lo + (hi - lo) * u).to(torch.float16).view(torch.int16)


def device_x_bf16(gen, batch: int, k: int, device="cuda"):
    import torch
    return torch.randn((batch, k), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def device_code_bytes(gen, nbytes: int, device="cuda"):
    import torch
    return torch.randint(0, 256, (nbytes,), generator=gen, device=device, dtype=torch.int16).to(torch.uint8)


def device_kv4_cache(gen, b: int, hkv: int, l_cap: int, d: int, s_lo=0.02, s_hi=0.2, device="cuda"):
    """kv4_cache_bytes drawn on the device (torch's CUDA generator): (codes
    uint8 [b][hkv][l_cap][d/2], params int32 [b][hkv][l_cap][d/128])."""
    import torch
    codes = torch.randint(0, 256, (b, hkv, l_cap, d // 2), generator=gen, device=device,
                          dtype=torch.int16).to(torch.uint8)
    shape = (b, hkv, l_cap, d // 128)
    s = torch.rand(shape, generator=gen, device=device) * (s_hi - s_lo) + s_lo
    z = -7.5 * s * (1.0 + (torch.rand(shape, generator=gen, device=device) * 0.2 - 0.1))
    sb = s.to(torch.float16).view(torch.int16).to(torch.int32) & 0xFFFF
    zb = z.to(torch.float16).view(torch.int16).to(torch.int32) << 16
    return codes, sb | zb
