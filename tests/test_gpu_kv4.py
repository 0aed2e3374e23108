"""The 4-bit KV cache on the GPU against the FP64 oracle (oracle.kv4): the
quantiser and the decode-step append bit for bit, and decode attention element
by element within |out - exact| <= 2e-3 * sum_t p_t (|V_tj| + 8 |s_t|) / sum_t p_t
plus the output rounding.  (The kernel rounds P s_t 2^sigma to FP16 before the
P V product, at most 2^-11 of each term's |s_t (c - 8)| <= 8 |s_t|; the bias
part sum_t p_t (z_t + 8 s_t) and the scores stay in FP32.)  Every cache the attention reads is either
random bytes (synth) or the oracle's quantisation of random values."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, to_dev

pytestmark = pytest.mark.gpu
kv4 = oracle.kv4


def _bf16(a):
    return synth.float32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _dev_bf16(bits):
    import torch
    return to_dev(bits.astype(np.int16), torch.bfloat16)


def _host(t, dtype):
    return t.cpu().numpy().view(dtype)


# ---------------------------------------------------------------- quantiser
def _quant_inputs(g, rows, d):
    x = g.standard_normal((rows, d)).astype(np.float32) * np.exp(g.uniform(-12, 7, (rows, 1))).astype(np.float32)
    x[0] = 0.0                                        # constant group: s = 0
    x[1] = np.float32(3.0)
    x[2, :] = (np.arange(d) % 16) * 2.0 - 7.0         # exact ramp
    x[3, :] = 0.0                                     # ties: lo 0, hi 30 (s = 2), 3 / 5 / 7 at .5 codes
    x[3, 1], x[3, 2], x[3, 3], x[3, 4] = 30.0, 3.0, 5.0, 7.0
    x[4] = g.standard_normal(d) * 1e-6                # FP16-subnormal scales
    x[5] = g.standard_normal(d) * 2000.0              # large, still finite in FP16
    return _bf16(x)


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("rows", [6, 1000, 4097])
def test_quantize_bit_exact(d, rows):
    import torch
    bits = _quant_inputs(synth.rng(900 + rows + d), rows, d)
    codes_ref, params_ref, st = kv4.quantize(bits, d)
    assert st == kv4.ERR_OK
    codes, params = bq.bq_kv4_quantize(_dev_bf16(bits))
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    assert np.array_equal(_host(codes, np.uint8), codes_ref)
    assert np.array_equal(_host(params, np.uint32), params_ref)


def test_quantize_errors_are_reported():
    import torch
    x = np.zeros((3, 128), dtype=np.float32)
    x[1, 7] = np.nan
    codes, params = bq.bq_kv4_quantize(_dev_bf16(_bf16(x)))
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_ERR_NONFINITE
    assert not codes[1].any() and int(params[1, 0]) == 0
    x = np.zeros((2, 128), dtype=np.float32)
    x[0, 0], x[0, 1] = -1e6, 1e6
    codes, params = bq.bq_kv4_quantize(_dev_bf16(_bf16(x)))
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_ERR_SCALE_RANGE
    assert not codes[0].any() and int(params[0, 0]) == 0
    assert bq.bq_check() == bq.BQ_OK


@pytest.mark.parametrize("d", [128, 256])
def test_append_writes_one_row_per_sequence(d):
    """Rows pos[b] of every (sequence, KV head) get the oracle's quantisation of
    the new K and V; every other byte of the caches is unchanged.  A position
    outside the cache writes nothing and is reported."""
    import torch
    g = synth.rng(910 + d)
    B, hkv, l_cap = 3, 2, 128
    kc0, kp0 = synth.kv4_cache_bytes(g, B, hkv, l_cap, d)
    vc0, vp0 = synth.kv4_cache_bytes(g, B, hkv, l_cap, d)
    kn = _bf16(g.standard_normal((B, hkv, d)))
    vn = _bf16(g.standard_normal((B, hkv, d)) * 5.0)
    dev = [to_dev(a) for a in (kc0, kp0.view(np.int32), vc0, vp0.view(np.int32))]
    for pos in ([0, 127, 64], [-1, 128, 5]):
        kc, kp, vc, vp = [t.clone() for t in dev]
        bq.bq_kv4_append(_dev_bf16(kn), _dev_bf16(vn), to_dev(np.array(pos, dtype=np.int32)), kc, kp, vc, vp)
        torch.cuda.synchronize()
        bad = any(p < 0 or p >= l_cap for p in pos)
        assert bq.bq_check() == (bq.BQ_ERR_SHAPE if bad else bq.BQ_OK)
        want = [a.copy() for a in (kc0, kp0, vc0, vp0)]
        for b, p in enumerate(pos):
            if 0 <= p < l_cap:
                for h in range(hkv):
                    c, pr, _ = kv4.quantize(kn[b, h][None], d)
                    want[0][b, h, p], want[1][b, h, p] = c[0], pr[0]
                    c, pr, _ = kv4.quantize(vn[b, h][None], d)
                    want[2][b, h, p], want[3][b, h, p] = c[0], pr[0]
        got = [_host(kc, np.uint8), _host(kp, np.uint32), _host(vc, np.uint8), _host(vp, np.uint32)]
        for gw, ww in zip(got, want):
            assert np.array_equal(gw, ww)


# ---------------------------------------------------------------- attention
def _attend(q_bits, caches, lens, hkv, d, l_cap, max_len, scale, out_dtype, workspace=None):
    import torch
    kc, kp, vc, vp = caches
    out, ws = bq.bq_kv4_attention_decode(_dev_bf16(q_bits), to_dev(kc), to_dev(kp.view(np.int32)), to_dev(vc),
                                         to_dev(vp.view(np.int32)), to_dev(np.asarray(lens, dtype=np.int32)),
                                         max_len, scale, out_dtype=out_dtype, workspace=workspace)
    torch.cuda.synchronize()
    return out, ws


def _check_attention(out, q_bits, caches, lens, hkv, d, l_cap, scale, what, heads=None):
    kc, kp, vc, vp = caches
    ref, mag = kv4.attention_decode(q_bits, kc, kp, vc, vp, lens, hkv, d, l_cap, scale, heads=heads)
    import torch
    name = "f32" if out.dtype == torch.float32 else "bf16"
    if heads is None:
        check_close(out, ref, mag, name, strict=(name == "f32"), what=what)
    else:
        ob = out.to(torch.float64).cpu().numpy()
        sel = tuple(np.array(heads).T)
        check_close(ob[sel], ref[sel], mag[sel], name, strict=(name == "f32"), what=what)


CASES = [
    # B, hq, hkv, d, l_cap, lens, max_len
    (3, 8, 2, 128, 1024, [1, 77, 1000], 1000),
    (4, 32, 8, 128, 8192, [8192, 5000, 3, 0], 8192),
    (2, 6, 2, 256, 2048, [2048, 700], 2048),
    (1, 4, 4, 128, 640, [600], 640),
    (2, 16, 2, 128, 4096, [4095, 129], 4096),
    (5, 5, 1, 256, 512, [512, 1, 100, 255, 300], 512),
    (16, 32, 8, 128, 512, [512 - 7 * i for i in range(16)], 512),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}-hq{c[1]}-hkv{c[2]}-d{c[3]}-L{c[4]}")
@pytest.mark.parametrize("out_dtype", [bq.BQ_F32, bq.BQ_BF16])
def test_attention_matches_oracle(case, out_dtype):
    B, hq, hkv, d, l_cap, lens, max_len = case
    g = synth.rng(920 + B + hq + d + l_cap)
    caches = synth.kv4_cache_bytes(g, B, hkv, l_cap, d) + synth.kv4_cache_bytes(g, B, hkv, l_cap, d, 0.05, 0.5)
    q = _bf16(g.standard_normal((B, hq, d)))
    scale = 1.0 / np.sqrt(d)
    out, ws = _attend(q, caches, lens, hkv, d, l_cap, max_len, scale, out_dtype)
    assert bq.bq_check() == bq.BQ_OK
    cnt = ((B * hkv * 4 + 255) // 256) * 256   # the split counters end the workspace
    if bq.bq_kv4_attention_workspace_bytes(B, hq, hkv, d, l_cap, max_len) > 0:
        assert int(ws[-cnt:].sum()) == 0       # left zero for the next call
    _check_attention(out, q, caches, lens, hkv, d, l_cap, scale, f"attn {case} dt{out_dtype}")


def test_attention_peaked_and_wide_scales():
    """A query along one cached key (nearly one-hot softmax), V scales spread
    over 1e-3 .. 300 (the per-warp power-of-two rescale of P s_V), and a large
    softmax scale."""
    import torch
    B, hq, hkv, d, l_cap = 2, 8, 2, 128, 4096
    lens = [4096, 2000]
    g = synth.rng(940)
    kc, kp = synth.kv4_cache_bytes(g, B, hkv, l_cap, d)
    vc, vp = synth.kv4_cache_bytes(g, B, hkv, l_cap, d)
    s = np.exp(g.uniform(np.log(1e-3), np.log(300.0), size=vp.shape))
    z = -7.5 * s * (1.0 + g.uniform(-0.2, 0.2, size=s.shape))
    vp = (s.astype(np.float16).view(np.uint16).astype(np.uint32) |
          (z.astype(np.float16).view(np.uint16).astype(np.uint32) << 16)).astype(np.uint32)
    caches = (kc, kp, vc, vp)
    q = np.empty((B, hq, d), dtype=np.uint16)
    for b in range(B):
        for h in range(hq):
            t = int(g.integers(0, lens[b]))
            krow = kv4.dequant(kc[b, h // (hq // hkv), t:t + 1], kp[b, h // (hq // hkv), t:t + 1], d)[0]
            q[b, h] = _bf16(krow / np.linalg.norm(krow) * (h + 1.0))
    for scale in (1.0 / np.sqrt(d), 4.0):
        out, _ = _attend(q, caches, lens, hkv, d, l_cap, l_cap, scale, bq.BQ_F32)
        assert bq.bq_check() == bq.BQ_OK
        _check_attention(out, q, caches, lens, hkv, d, l_cap, scale, f"peaked scale {scale}")


def test_attention_from_quantised_values_and_determinism():
    """Caches made by the oracle quantiser from random K / V; two calls on the
    same workspace give identical bits."""
    import torch
    B, hq, hkv, d, l_cap = 2, 8, 4, 128, 2048
    lens = [2048, 1500]
    g = synth.rng(950)
    K = _bf16(g.standard_normal((B, hkv, l_cap, d)) * 2.0)
    V = _bf16(g.standard_normal((B, hkv, l_cap, d)))
    kc, kp, _ = kv4.quantize(K.reshape(-1, d), d)
    vc, vp, _ = kv4.quantize(V.reshape(-1, d), d)
    caches = (kc.reshape(B, hkv, l_cap, d // 2), kp.reshape(B, hkv, l_cap, 1),
              vc.reshape(B, hkv, l_cap, d // 2), vp.reshape(B, hkv, l_cap, 1))
    q = _bf16(g.standard_normal((B, hq, d)))
    scale = 1.0 / np.sqrt(d)
    out1, ws = _attend(q, caches, lens, hkv, d, l_cap, l_cap, scale, bq.BQ_BF16)
    out2, _ = _attend(q, caches, lens, hkv, d, l_cap, l_cap, scale, bq.BQ_BF16, workspace=ws)
    assert bq.bq_check() == bq.BQ_OK
    assert torch.equal(out1, out2)
    _check_attention(out1, q, caches, lens, hkv, d, l_cap, scale, "quantised caches")


@pytest.mark.parametrize("B,ctx", [(1, 65536), (16, 4096)])
def test_attention_qwen3_8b_sampled(B, ctx):
    """Qwen3-8B decode attention (32 query / 8 KV heads, d 128) at its full
    65,536-token context and at batch 16 x 4096: sampled heads against the
    oracle."""
    A = synth.QWEN3_8B_ATTN
    hq, hkv, d = A["hq"], A["hkv"], A["d"]
    g = synth.rng(960 + B)
    caches = synth.kv4_cache_bytes(g, B, hkv, ctx, d) + synth.kv4_cache_bytes(g, B, hkv, ctx, d)
    lens = [ctx - 37 * b for b in range(B)]
    q = _bf16(g.standard_normal((B, hq, d)))
    scale = 1.0 / np.sqrt(d)
    out, _ = _attend(q, caches, lens, hkv, d, ctx, ctx, scale, bq.BQ_BF16)
    assert bq.bq_check() == bq.BQ_OK
    heads = sorted({(int(b), int(h)) for b, h in zip(g.integers(0, B, 6), g.integers(0, hq, 6))} |
                   {(0, 0), (B - 1, hq - 1)})
    _check_attention(out, q, caches, lens, hkv, d, ctx, scale, f"qwen3-8b B{B} ctx{ctx}", heads=heads)


def test_attention_length_errors_and_empty():
    """A length above max_len is clamped and reported; max_len 0 gives zeros."""
    import torch
    B, hq, hkv, d, l_cap = 2, 4, 1, 128, 256
    g = synth.rng(970)
    caches = synth.kv4_cache_bytes(g, B, hkv, l_cap, d) + synth.kv4_cache_bytes(g, B, hkv, l_cap, d)
    q = _bf16(g.standard_normal((B, hq, d)))
    out, _ = _attend(q, caches, [300, 100], hkv, d, l_cap, 200, 0.1, bq.BQ_F32)
    assert bq.bq_check() == bq.BQ_ERR_SHAPE
    _check_attention(out, q, caches, [200, 100], hkv, d, l_cap, 0.1, "clamped length")
    out, _ = _attend(q, caches, [0, 0], hkv, d, l_cap, 0, 0.1, bq.BQ_F32)
    assert bq.bq_check() == bq.BQ_OK
    assert torch.all(out == 0)


def test_attention_argument_errors():
    import torch
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 1, 64, 64), dtype=torch.uint8, device="cuda")
    kp = torch.zeros((1, 1, 64, 1), dtype=torch.int32, device="cuda")
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_kv4_attention_decode(q, kc, kp, kc, kp, lens, 128, 0.1)   # max_len > L_cap
    assert e.value.status == bq.BQ_ERR_SHAPE
    q9 = torch.zeros((1, 9, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_kv4_attention_decode(q9, kc, kp, kc, kp, lens, 64, 0.1)   # 9 query heads per KV head
    assert e.value.status == bq.BQ_ERR_SHAPE
    kc1 = torch.zeros((1, 2, 4096, 64), dtype=torch.uint8, device="cuda")
    kp1 = torch.zeros((1, 2, 4096, 1), dtype=torch.int32, device="cuda")
    q2 = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    assert bq.bq_kv4_attention_workspace_bytes(1, 8, 2, 128, 4096, 4096) > 0
    with pytest.raises(bq.BQError) as e:
        bq.bq_kv4_attention_decode(q2, kc1, kp1, kc1, kp1, lens, 4096, 0.1,
                                   workspace=torch.zeros(256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == bq.BQ_ERR_WORKSPACE
