"""CPU oracle for the 4-bit KV cache and its decode attention -- TEST
INFRASTRUCTURE ONLY (the same rule as the rest of ``oracle``: only tests, the
smoke entry point and the bench's CPU legs may call it).

Pages: "Bonsai-27B-mlx-1bit ... Binary g128" (sections "峰值内存管理" and
"KV压缩潜力": the KV cache is quantised to 4 bits for long contexts) and
"Ternary Bonsai" (the hybrid-attention section: 4-bit KV-cache quantisation);
"1-bit Bonsai 8B" notes, Table 1 (grouped-query attention, 32 query / 8 KV
heads).  The pages name the bit width only; the format below is a reading:

* every cached K or V vector of head dimension D (D % 128 == 0) is cut into
  groups of 128 values, like the weights' g128 groups;
* a group is quantised min-max affine with 16 levels: with lo / hi the
  smallest / largest value, s = FP16(RNE((hi - lo) / 15)), z = FP16(RNE(lo)),
  code c = clamp(rint((x - z) / s), 0, 15) (c = 0 when s == 0), value s c + z
  (the scale-and-bias form the MLX page uses for its weight groups);
* codes: two per byte, element 2i in the low nibble of byte i; params: one
  32-bit word per group, FP16 s in the low half, FP16 z in the high half.

Decode attention (plain definition, FP64): for query head h of sequence b,
with kv = h // G (G = Hq / Hkv) and the first len[b] cached tokens,
    a_t = scale * <q_h, K_t>,   p_t = exp(a_t - max a),
    out_h = sum_t p_t V_t / sum_t p_t          (zeros when len[b] == 0).

Arithmetic: numpy float64 throughout (FP16 / BF16 decode by bit reinterpretation,
which is exact; FP16 encode by numpy's round-to-nearest-even conversion; the
products by float64 matmul).
"""
from __future__ import annotations

import numpy as np

KV_GROUP = 128
ERR_OK, ERR_NONFINITE, ERR_SCALE_RANGE = 0, 4, 5


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _f64_to_f16_bits(v: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def codes_bytes(rows: int, d: int) -> int:
    return rows * d // 2


def params_bytes(rows: int, d: int) -> int:
    return rows * (d // KV_GROUP) * 4


def quantize(x_bf16: np.ndarray, d: int):
    """Quantise rows of BF16 bit patterns [rows][d] to the 4-bit g128 format.

    Returns (codes uint8 [rows][d/2], params uint32 [rows][d/128], status).
    status: ERR_NONFINITE if a value is NaN/Inf, ERR_SCALE_RANGE if s or z of a
    group overflows FP16 (then that group is stored as s = z = 0, codes 0);
    ERR_OK otherwise.  The first failing kind in row order is reported."""
    x = _bf16_to_f64(np.asarray(x_bf16).reshape(-1, d))
    rows = x.shape[0]
    g = x.reshape(rows, d // KV_GROUP, KV_GROUP)
    status = ERR_OK
    finite = np.isfinite(g).all(axis=2)
    lo = np.where(finite, g.min(axis=2, initial=np.inf, where=np.isfinite(g)), 0.0)
    hi = np.where(finite, g.max(axis=2, initial=-np.inf, where=np.isfinite(g)), 0.0)
    s_bits = _f64_to_f16_bits((hi - lo) / 15.0)
    z_bits = _f64_to_f16_bits(lo)
    s = _f16_bits_to_f64(s_bits)
    z = _f16_bits_to_f64(z_bits)
    ok = finite & np.isfinite(s) & np.isfinite(z)
    if not finite.all():
        status = ERR_NONFINITE
    elif not ok.all():
        status = ERR_SCALE_RANGE
    s_bits = np.where(ok, s_bits, 0).astype(np.uint16)
    z_bits = np.where(ok, z_bits, 0).astype(np.uint16)
    s = np.where(ok, s, 0.0)
    z = np.where(ok, z, 0.0)
    with np.errstate(invalid="ignore", divide="ignore"):
        c = np.rint((g - z[..., None]) / s[..., None])
    c = np.where((s[..., None] > 0) & ok[..., None], np.clip(c, 0, 15), 0).astype(np.uint8)
    c = c.reshape(rows, d)
    codes = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    params = (s_bits.astype(np.uint32) | (z_bits.astype(np.uint32) << 16)).astype(np.uint32)
    return codes, params, status


def dequant(codes: np.ndarray, params: np.ndarray, d: int) -> np.ndarray:
    """Values s c + z (FP64) of rows stored as (codes [rows][d/2], params [rows][d/128])."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1, d // 2)
    params = np.asarray(params, dtype=np.uint32).reshape(-1, d // KV_GROUP)
    rows = codes.shape[0]
    c = np.empty((rows, d), dtype=np.float64)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    s = _f16_bits_to_f64((params & 0xFFFF).astype(np.uint16))
    z = _f16_bits_to_f64((params >> 16).astype(np.uint16))
    return (c.reshape(rows, d // KV_GROUP, KV_GROUP) * s[..., None] + z[..., None]).reshape(rows, d)


def attention_decode(q_bf16, k_codes, k_params, v_codes, v_params, lens, hkv: int, d: int, l_cap: int,
                     scale: float, heads=None):
    """Decode attention of every (sequence, query head) over the 4-bit cache.

    q_bf16: BF16 bits [B][Hq][d]; caches: codes [B][Hkv][l_cap][d/2], params
    [B][Hkv][l_cap][d/128]; lens: [B].  heads: optional list of (b, h) pairs to
    compute (others are left NaN).
    Returns (out [B][Hq][d] FP64, mag [B][Hq][d] FP64) where
    mag[b][h][j] = sum_t p_t (|V_tj| + 8 |s_t|) / sum_t p_t, the size of the
    terms the output averages (s_t the scale of V_tj's group; 8 |s_t| bounds the
    centred code part |s_t (c - 8)| of V_tj = s_t (c - 8) + (z_t + 8 s_t))."""
    q = _bf16_to_f64(q_bf16)
    B, hq = q.shape[0], q.shape[1]
    G = hq // hkv
    kc = np.asarray(k_codes).reshape(B, hkv, l_cap, d // 2)
    kp = np.asarray(k_params).reshape(B, hkv, l_cap, d // KV_GROUP)
    vc = np.asarray(v_codes).reshape(B, hkv, l_cap, d // 2)
    vp = np.asarray(v_params).reshape(B, hkv, l_cap, d // KV_GROUP)
    out = np.full((B, hq, d), np.nan)
    mag = np.full((B, hq, d), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(hq)]
    cache = {}
    for b, h in todo:
        kv = h // G
        n = int(lens[b])
        if n == 0:
            out[b, h] = 0.0
            mag[b, h] = 0.0
            continue
        if (b, kv) not in cache:
            K = dequant(kc[b, kv, :n], kp[b, kv, :n], d)
            V = dequant(vc[b, kv, :n], vp[b, kv, :n], d)
            p = vp[b, kv, :n]
            sz = 8.0 * np.abs(_f16_bits_to_f64((p & 0xFFFF).astype(np.uint16)))
            cache[(b, kv)] = (K, V, np.abs(V) + np.repeat(sz, KV_GROUP, axis=1))
        K, V, A = cache[(b, kv)]
        a = scale * (K @ q[b, h])
        p = np.exp(a - a.max())
        out[b, h] = (p @ V) / p.sum()
        mag[b, h] = (p @ A) / p.sum()
    return out, mag
