"""Pins of the 4-bit KV-cache oracle (oracle.kv4) to facts that do not come
from the oracle itself: quantiser cases whose codes follow by hand, the
dequantisation error bound of round-to-nearest, nibble order, and attention
closed forms (one token, equal keys, one dominant key, two tokens, the GQA
head map, token-order invariance, scale 0 giving the mean)."""
import math

import numpy as np
import pytest

from oracle import kv4


def bf16_bits(v):
    """BF16 bit patterns of float values that are exactly representable."""
    f = np.asarray(v, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "test value not exact in BF16"
    return (bits >> 16).astype(np.uint16)


def f16(bits):
    return float(np.uint16(bits).view(np.float16))


def test_ramp_group_is_exact():
    """Values i % 16 (lo 0, hi 15): s = 1, z = 0 and the codes are the values."""
    x = np.arange(128) % 16
    codes, params, st = kv4.quantize(bf16_bits(x.astype(np.float32))[None, :], 128)
    assert st == kv4.ERR_OK
    assert f16(params[0, 0] & 0xFFFF) == 1.0 and f16(params[0, 0] >> 16) == 0.0
    assert np.array_equal(kv4.dequant(codes, params, 128)[0], x.astype(np.float64))
    # element 2i in the low nibble, 2i+1 in the high nibble
    assert codes[0, 0] == 0x10 and codes[0, 7] == 0xFE


def test_shifted_ramp_and_second_group():
    """2 (i % 16) - 7 gives s = 2, z = -7; a second group of the row has its own
    parameters (a constant -3: s = 0, z = -3, codes 0)."""
    x = np.concatenate([2.0 * (np.arange(128) % 16) - 7.0, np.full(128, -3.0)])
    codes, params, st = kv4.quantize(bf16_bits(x.astype(np.float32))[None, :], 256)
    assert st == kv4.ERR_OK
    assert (f16(params[0, 0] & 0xFFFF), f16(params[0, 0] >> 16)) == (2.0, -7.0)
    assert (f16(params[0, 1] & 0xFFFF), f16(params[0, 1] >> 16)) == (0.0, -3.0)
    assert np.all(codes[0, 64:] == 0)
    assert np.array_equal(kv4.dequant(codes, params, 256)[0], x)


def test_rounding_ties_and_clamp():
    """lo 0, hi 30 (s = 2): a value 3 sits at code 1.5 and goes to the even code 2,
    5 (2.5) to 2, 7 (3.5) to 4."""
    x = np.zeros(128)
    x[1] = 30.0
    x[2], x[3], x[4] = 3.0, 5.0, 7.0
    codes, params, st = kv4.quantize(bf16_bits(x.astype(np.float32))[None, :], 128)
    c = np.empty(128, dtype=int)
    c[0::2], c[1::2] = codes[0] & 15, codes[0] >> 4
    assert (c[0], c[1], c[2], c[3], c[4]) == (0, 15, 2, 2, 4)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dequant_error_bound(seed):
    """Round to nearest: |x - (s c + z)| <= s / 2 plus what the FP16 rounding of
    z and s moves (|lo - z| + 15 s 2^-11 at the clamped top code)."""
    g = np.random.default_rng(seed)
    x = (g.standard_normal((64, 256)) * g.uniform(0.01, 30, (64, 1))).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    xb = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    codes, params, st = kv4.quantize(bits, 256)
    assert st == kv4.ERR_OK
    deq = kv4.dequant(codes, params, 256)
    for gi in range(2):
        sl = slice(128 * gi, 128 * gi + 128)
        s = params[:, gi] & 0xFFFF
        z = params[:, gi] >> 16
        s = s.astype(np.uint16).view(np.float16).astype(np.float64)
        z = z.astype(np.uint16).view(np.float16).astype(np.float64)
        lo = xb[:, sl].min(axis=1)
        bound = s / 2 + np.abs(lo - z) + 16 * s * 2.0 ** -11
        assert np.all(np.abs(xb[:, sl] - deq[:, sl]) <= bound[:, None] * (1 + 1e-12))


def test_quantize_errors():
    x = np.zeros((2, 128), dtype=np.float32)
    x[1, 5] = np.inf
    assert kv4.quantize((x.view(np.uint32) >> 16).astype(np.uint16), 128)[2] == kv4.ERR_NONFINITE
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 0], x[0, 1] = -1e6, 1e6          # z and s overflow FP16
    codes, params, st = kv4.quantize((x.view(np.uint32) >> 16).astype(np.uint16), 128)
    assert st == kv4.ERR_SCALE_RANGE and params[0, 0] == 0 and not codes.any()


def _cache(vals, d):
    """Quantise per-token values [B][Hkv][L][d] into the cache arrays."""
    B, H, L, _ = vals.shape
    bits = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    c, p, st = kv4.quantize(bits.reshape(-1, d), d)
    assert st == kv4.ERR_OK
    return c.reshape(B, H, L, d // 2), p.reshape(B, H, L, d // 128)


def _q(vals):
    return (np.asarray(vals, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_attention_single_token_and_empty():
    """One cached token: the output is its V, whatever q; len 0: zeros."""
    g = np.random.default_rng(5)
    d, L = 128, 64
    K = g.standard_normal((2, 1, L, d))
    V = g.standard_normal((2, 1, L, d))
    kc, kp = _cache(K, d)
    vc, vp = _cache(V, d)
    q = _q(g.standard_normal((2, 4, d)))
    out, _ = kv4.attention_decode(q, kc, kp, vc, vp, [1, 0], 1, d, L, 0.1)
    v0 = kv4.dequant(vc[0, 0, :1], vp[0, 0, :1], d)[0]
    for h in range(4):
        assert np.array_equal(out[0, h], v0)
        assert np.all(out[1, h] == 0)


def test_attention_equal_keys_give_the_mean():
    """All keys equal: every weight is the same and the output is the mean of V."""
    g = np.random.default_rng(6)
    d, L = 128, 128
    K = np.repeat(g.standard_normal((1, 1, 1, d)), L, axis=2)
    V = g.standard_normal((1, 1, L, d))
    kc, kp = _cache(K, d)
    vc, vp = _cache(V, d)
    n = 77
    out, mag = kv4.attention_decode(_q(g.standard_normal((1, 2, d))), kc, kp, vc, vp, [n], 1, d, L, 1.0)
    mean = kv4.dequant(vc[0, 0, :n], vp[0, 0, :n], d).mean(axis=0)
    assert np.allclose(out[0, 0], mean, rtol=0, atol=1e-12) and np.allclose(out[0, 1], mean, rtol=0, atol=1e-12)
    assert np.all(mag >= np.abs(out) - 1e-12)


def test_attention_dominant_key_and_two_token_closed_form():
    """Key 3 along q with a large scale takes all the weight; with two tokens the
    output is (e^a1 v1 + e^a2 v2) / (e^a1 + e^a2), a1, a2 the scaled dots
    taken from the dequantised keys."""
    d, L = 128, 64
    g = np.random.default_rng(7)
    qv = np.zeros(d)
    qv[:8] = 1.0
    K = np.zeros((1, 1, L, d))
    K[0, 0, :, 8:] = g.standard_normal((L, d - 8))
    K[0, 0, 3, :8] = 4.0
    V = g.standard_normal((1, 1, L, d))
    kc, kp = _cache(K, d)
    vc, vp = _cache(V, d)
    out, _ = kv4.attention_decode(_q(qv[None, None, :]), kc, kp, vc, vp, [L], 1, d, L, 50.0)
    v3 = kv4.dequant(vc[0, 0, 3:4], vp[0, 0, 3:4], d)[0]
    assert np.allclose(out[0, 0], v3, rtol=0, atol=1e-9)
    out2, _ = kv4.attention_decode(_q(qv[None, None, :]), kc, kp, vc, vp, [2], 1, d, L, 0.3)
    Kd = kv4.dequant(kc[0, 0, :2], kp[0, 0, :2], d)
    Vd = kv4.dequant(vc[0, 0, :2], vp[0, 0, :2], d)
    a1 = 0.3 * sum(qv[i] * Kd[0, i] for i in range(d))
    a2 = 0.3 * sum(qv[i] * Kd[1, i] for i in range(d))
    e1, e2 = math.exp(a1), math.exp(a2)
    for j in range(0, d, 17):
        assert abs(out2[0, 0, j] - (e1 * Vd[0, j] + e2 * Vd[1, j]) / (e1 + e2)) <= 1e-12


def test_attention_gqa_head_map_and_invariances():
    """Query head h reads KV head h // G: with V constant per KV head, every
    query head returns its KV head's constant.  Reordering the tokens changes
    nothing, and scale 0 (every score equal) gives the plain mean of V."""
    d, L, hkv, G = 128, 64, 3, 4
    g = np.random.default_rng(8)
    K = g.standard_normal((1, hkv, L, d))
    V = np.zeros((1, hkv, L, d))
    for kv in range(hkv):
        V[0, kv] = float(kv + 1)
    kc, kp = _cache(K, d)
    vc, vp = _cache(V, d)
    q = _q(g.standard_normal((1, hkv * G, d)))
    out, _ = kv4.attention_decode(q, kc, kp, vc, vp, [L], hkv, d, L, 0.5)
    for h in range(hkv * G):
        assert np.allclose(out[0, h], float(h // G + 1), rtol=0, atol=1e-12), h
    V = g.standard_normal((1, hkv, L, d))
    vc, vp = _cache(V, d)
    out, _ = kv4.attention_decode(q, kc, kp, vc, vp, [L], hkv, d, L, 0.5)
    perm = g.permutation(L)
    out_p, _ = kv4.attention_decode(q, kc[:, :, perm], kp[:, :, perm], vc[:, :, perm], vp[:, :, perm], [L],
                                    hkv, d, L, 0.5)
    assert np.allclose(out, out_p, rtol=0, atol=1e-12)
    out0, _ = kv4.attention_decode(q, kc, kp, vc, vp, [L], hkv, d, L, 0.0)
    for h in range(hkv * G):
        mean = kv4.dequant(vc[0, h // G], vp[0, h // G], d).mean(axis=0)
        assert np.allclose(out0[0, h], mean, rtol=0, atol=1e-12)


def test_cache_bytes_per_token():
    """4 bits per value plus one 32-bit (s, z) word per 128 values: 68 bytes for
    a 128-dimensional head vector, 4.25 bits per value."""
    assert kv4.codes_bytes(1, 128) + kv4.params_bytes(1, 128) == 68
    assert 8 * (kv4.codes_bytes(1, 256) + kv4.params_bytes(1, 256)) / 256 == 4.25
