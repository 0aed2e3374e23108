"""Pins for the CPU oracle: each test checks it against something other than
itself -- a number printed on the pages, a library routine, a closed form, an
invariant or an exact brute-force computation -- so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

G = 128


# ----------------------------------------------------------------- IEEE types
def test_half_decode_exhaustive_vs_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros keep their sign
    assert math.copysign(1.0, oracle.half_to_double(0x8000)) == -1.0


def test_half_encode_rne_vs_numpy():
    g = synth.rng(1)
    vals = np.concatenate([
        g.standard_normal(20000) * 10.0 ** g.integers(-9, 6, 20000),
        g.uniform(-70000, 70000, 2000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
         2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 * (1 - 2.0 ** -12)],
    ])
    # exact midpoints between consecutive representable halves (ties -> even)
    mids = []
    for b in range(0x0000, 0x7BFF, 97):
        lo = np.uint16(b).view(np.float16).astype(np.float64)
        hi = np.uint16(b + 1).view(np.float16).astype(np.float64)
        mids += [(lo + hi) / 2, -(lo + hi) / 2]
    vals = np.concatenate([vals, mids])
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_decode_exhaustive_vs_torch():
    torch = pytest.importorskip("torch")
    bits = np.arange(65536, dtype=np.int64)
    t = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    nan = np.isnan(t)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], t[~nan])


def test_bf16_encode_rne_vs_torch():
    torch = pytest.importorskip("torch")
    g = synth.rng(2)
    vals = g.standard_normal(20000) * 10.0 ** g.integers(-30, 30, 20000)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.double_to_bf16(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------ page facts
def _facts(golden_dir):
    with open(os.path.join(golden_dir, "page_facts.json")) as f:
        return json.load(f)


def test_bits_per_weight_page_facts(golden_dir):
    facts = _facts(golden_dir)
    assert oracle.effective_bits("q1g128") == facts["binary_bits_per_weight"]["value"]
    # 2-bit slots and 5 trits per byte (+ the FP16 scale)
    assert oracle.effective_bits("t2g128") == 2.0 + 16 / 128
    assert oracle.effective_bits("t5p8") == 26 * 8 / 128 + 16 / 128
    # the ~1.71 figure is the information content log2(3) plus the scale share;
    # 5-per-byte storage sits between it and the 2-bit slots
    entropy = math.log2(3) + 16 / 128
    assert round(entropy, 2) == facts["ternary_effective_bits"]["value"]
    assert entropy < oracle.effective_bits("t5p8") < oracle.effective_bits("t2g128")


def test_trit_packing_bounds(golden_dir):
    facts = _facts(golden_dir)
    tb = facts["trits_per_byte"]
    assert 3 ** tb["trits"] <= 2 ** tb["bits"] < 3 ** (tb["trits"] + 1)
    assert tb["bits"] / tb["trits"] == tb["bits_per_trit"]
    t27 = facts["trits_per_27_bits"]
    assert 3 ** t27["trits"] <= 2 ** t27["bits"]
    assert round(t27["bits"] / t27["trits"], 3) == t27["bits_per_trit"]
    # a 128-trit group in 5-per-byte storage: 25 full bytes + one byte of 3
    assert oracle.codes_bytes("t5p8", 1, 128) == 26 == math.ceil(128 / tb["trits"])


def test_table2_byte_count_identity(golden_dir):
    t2 = _facts(golden_dir)["table2_bytes"]
    params = t2["fp16_safetensors"] // 2
    assert params * 2 == t2["fp16_safetensors"]
    # params = rows x 128: codes + scales of the binary format
    rows = params // 128
    assert rows * 128 == params
    total = oracle.codes_bytes("q1g128", rows, 128) + oracle.scales_bytes(rows, 128)
    assert total == t2["gguf_q1_0_g128"]


def test_sign_convention(golden_dir):
    sc = _facts(golden_dir)["binary_sign_convention"]
    row = np.zeros(16, dtype=np.uint8)
    row[0] = 0b10  # weight 0 -> bit 0, weight 1 -> bit 1
    assert oracle.weight_code("q1g128", row, 0) == sc["bit0"]
    assert oracle.weight_code("q1g128", row, 1) == sc["bit1"]


# --------------------------------------------------------------- packing
def test_pack_binary_signs_and_zero():
    w = np.zeros((1, G), dtype=np.float32)
    w[0, :4] = [1.0, -1.0, 0.0, -0.0]
    w[0, 4:] = np.linspace(-2, 2, G - 4, dtype=np.float32)
    codes, scales = oracle.pack("q1g128", w)
    q = oracle.unpack("q1g128", codes, 1, G)[0]
    assert list(q[:4]) == [1, -1, 1, 1]  # zero (either sign) maps to +1
    assert np.array_equal(q[4:], np.where(w[0, 4:] >= 0, 1, -1))
    # LSB-first bit order inside each byte
    assert codes[0] & 1 == 1 and (codes[0] >> 1) & 1 == 0


def test_scale_is_fp16_of_mean_abs_and_l2_optimal():
    g = synth.rng(3)
    w = synth.weights_normal(g, 8, 4 * G)
    codes, scales = oracle.pack("q1g128", w)
    s = scales.view(np.float16).astype(np.float64).reshape(8, 4)
    wg = w.astype(np.float64).reshape(8, 4, G)
    mean_abs = np.abs(wg).mean(axis=2)
    assert np.array_equal(scales.reshape(8, 4), mean_abs.astype(np.float16).view(np.uint16))
    # closed form: for fixed signs, argmin_a sum (w - a sign(w))^2 = mean |w|
    sgn = np.where(wg >= 0, 1.0, -1.0)
    def sse(a):
        return ((wg - a[..., None] * sgn) ** 2).sum(axis=2)
    for d in (1e-4, -1e-4):
        assert np.all(sse(mean_abs) < sse(mean_abs + d))
    assert np.all(np.abs(s - mean_abs) <= np.abs(mean_abs) * 2.0 ** -11 + 2.0 ** -25)


def test_ternary_threshold_is_clamped_round_half_even():
    s_bits = np.array([[np.float16(0.03125).view(np.uint16)]], dtype=np.uint16)
    s = 0.03125
    vals = np.array([0, s / 2, -s / 2, np.nextafter(np.float32(s / 2), np.float32(1)),
                     -np.nextafter(np.float32(s / 2), np.float32(1)), s, -s, 1.5 * s, 3 * s,
                     -7 * s, 1e-9, -1e-9], dtype=np.float32)
    w = np.zeros((1, G), dtype=np.float32)
    w[0, :vals.size] = vals
    for fmt in ("t2g128", "t5p8"):
        codes, scales = oracle.pack(fmt, w, scales_in=s_bits)
        q = oracle.unpack(fmt, codes, 1, G)[0, :vals.size]
        ref = np.clip(np.rint(vals.astype(np.float64) / s), -1, 1).astype(np.int8)
        assert np.array_equal(q, ref), fmt


def test_ternary_mean_abs_scale_matches_binary_rule():
    g = synth.rng(4)
    w = synth.weights_normal(g, 4, 2 * G)
    _, s1 = oracle.pack("q1g128", w)
    for fmt in ("t2g128", "t5p8"):
        _, st = oracle.pack(fmt, w)
        assert np.array_equal(s1, st)


@pytest.mark.parametrize("fmt", ["t2g128", "t5p8"])
def test_ternary_given_scale_roundtrip(fmt):
    g = synth.rng(5)
    n, k = 7, 3 * G
    t = synth.trits(g, n, k)
    s = synth.scales_uniform(g, n, k // G)
    w = t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), G, axis=1)
    codes, scales = oracle.pack(fmt, w, scales_in=s)
    assert np.array_equal(scales, s.reshape(-1))
    assert np.array_equal(oracle.unpack(fmt, codes, n, k), t)


def test_t2_code_layout_and_invalid_pattern():
    # trits -1, 0, +1, 0 -> codes 0, 1, 2, 1 at bits 0,2,4,6
    w = np.zeros((1, G), dtype=np.float32)
    w[0, :4] = [-1, 0, 1, 0]
    codes, _ = oracle.pack("t2g128", w, scales_in=np.array([[0x3C00]], dtype=np.uint16))
    assert codes[0] == (0 | 1 << 2 | 2 << 4 | 1 << 6)
    assert oracle.codes_bytes("t2g128", 1, G) == 32
    bad = codes.copy()
    bad[0] |= 3  # the unused fourth pattern
    with pytest.raises(oracle.OracleError):
        oracle.unpack("t2g128", bad, 1, G)


def test_t5p8_every_byte_value_decodes_as_base3():
    row = np.zeros(26, dtype=np.uint8)
    for v in range(256):
        row[0] = v
        got = [oracle.weight_code("t5p8", row, i) for i in range(5)]
        if v >= 243:
            assert all(c == -2 for c in got)
            continue
        digits = [int(ch) for ch in np.base_repr(v, 3).zfill(5)[::-1]]  # least significant first
        assert got == [d - 1 for d in digits]
    for v in range(256):  # tail byte of a group holds three trits
        row[25] = v
        got = [oracle.weight_code("t5p8", row, 125 + i) for i in range(3)]
        if v >= 27:
            assert all(c == -2 for c in got)
        else:
            assert got == [int(ch) - 1 for ch in np.base_repr(v, 3).zfill(3)[::-1]]


def test_pack_errors():
    w = np.ones((2, G), dtype=np.float32)
    assert oracle.pack_status("q1g128", np.ones((2, 100), dtype=np.float32))[0] == oracle.ERR_SHAPE
    wn = w.copy(); wn[1, 5] = np.nan
    assert oracle.pack_status("q1g128", wn)[0] == oracle.ERR_NONFINITE
    wi = w.copy(); wi[0, 0] = np.inf
    assert oracle.pack_status("t2g128", wi)[0] == oracle.ERR_NONFINITE
    big = np.full((1, G), 70000.0, dtype=np.float32)
    assert oracle.pack_status("q1g128", big)[0] == oracle.ERR_SCALE_RANGE
    ok_big = np.full((1, G), 65504.0, dtype=np.float32)
    assert oracle.pack_status("q1g128", ok_big)[0] == oracle.OK
    neg = np.array([[0xBC00]], dtype=np.uint16)
    assert oracle.pack_status("t2g128", np.ones((1, G), np.float32), neg)[0] == oracle.ERR_SCALE_RANGE
    assert oracle.pack_status("t5p8", np.zeros((0, G), np.float32))[0] == oracle.OK


# --------------------------------------------------------------- products
def _exact_dot(t_row, s_row, x_row):
    """Exact rational sum_g s_g sum_k t_k x_k from the ORIGINAL trits/signs."""
    acc = Fraction(0)
    for gi in range(len(s_row)):
        s = Fraction(float(np.uint16(s_row[gi]).view(np.float16)))
        p = Fraction(0)
        for i in range(G):
            kk = gi * G + i
            xv = Fraction(float(x_row[kk]))
            p += int(t_row[kk]) * xv
        acc += s * p
    return acc


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
def test_brute_force_tiny_exact(fmt):
    import torch
    g = synth.rng(6)
    n, k, b = 5, 2 * G, 3
    if fmt == "q1g128":
        t = np.where(g.random((n, k)) < 0.5, -1, 1).astype(np.int8)
    else:
        t = synth.trits(g, n, k)
    s = synth.scales_uniform(g, n, k // G)
    w = t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), G, axis=1)
    codes, scales = oracle.pack(fmt, w, scales_in=s)
    x = synth.x_bf16(g, b, k)
    xf = torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    y, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    for bi in range(b):
        for r in range(n):
            ex = _exact_dot(t[r], s[r], xf[bi])
            assert abs(Fraction(y[bi, r]) - ex) <= abs(ex) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)
            sab = sum(abs(Fraction(float(np.uint16(s[r, kk // G]).view(np.float16))) * Fraction(float(xf[bi, kk])))
                      for kk in range(k))
            assert abs(Fraction(bound[bi, r]) - sab) <= sab * Fraction(1, 2 ** 50)


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
def test_matmul_vs_numpy_matmul(fmt):
    import torch
    g = synth.rng(7)
    n, k, b = 64, 8 * G, 4
    w = synth.weights_normal(g, n, k)
    codes, scales = oracle.pack(fmt, w)
    x = synth.x_bf16(g, b, k)
    xf = torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    wd = oracle.dequant(fmt, codes, scales, n, k)
    ref = xf @ wd.T  # library primitive
    y, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
    s_rep = np.repeat(scales.view(np.float16).astype(np.float64).reshape(n, -1), G, axis=1)
    assert np.allclose(bound, np.abs(xf) @ s_rep.T, rtol=1e-13, atol=0)


def test_closed_form_all_ones_x_binary():
    g = synth.rng(8)
    n, k = 6, 3 * G
    codes = synth.code_bytes_uniform(g, oracle.codes_bytes("q1g128", n, k))
    scales = synth.scales_uniform(g, n, k // G).reshape(-1)
    x = np.full((1, k), 0x3F80, dtype=np.uint16)  # BF16 1.0
    y, _ = oracle.matmul("q1g128", codes, scales, n, k, x)
    cb = codes.reshape(n, k // 8)
    for r in range(n):
        exp = 0.0
        for gi in range(k // G):
            pop = sum(bin(int(v)).count("1") for v in cb[r, gi * 16:(gi + 1) * 16])
            exp += float(np.uint16(scales[r * (k // G) + gi]).view(np.float16)) * (2 * pop - G)
        assert y[0, r] == exp


@pytest.mark.parametrize("fmt", ["t2g128", "t5p8"])
def test_closed_form_all_ones_x_ternary(fmt):
    g = synth.rng(9)
    n, k = 5, 2 * G
    t = synth.trits(g, n, k)
    s = synth.scales_uniform(g, n, k // G)
    w = t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), G, axis=1)
    codes, scales = oracle.pack(fmt, w, scales_in=s)
    x = np.full((1, k), 0x3F80, dtype=np.uint16)
    y, _ = oracle.matmul(fmt, codes, scales, n, k, x)
    tg = t.reshape(n, k // G, G)
    exp = ((tg == 1).sum(axis=2) - (tg == -1).sum(axis=2)) * s.view(np.float16).astype(np.float64)
    assert np.array_equal(y[0], exp.sum(axis=1))


@pytest.mark.parametrize("fmt", ["t2g128", "t5p8"])
def test_all_zero_trits_give_exact_zero(fmt):
    n, k = 3, 2 * G
    w = np.zeros((n, k), dtype=np.float32)
    s = np.full((n, k // G), 0x3C00, dtype=np.uint16)
    codes, scales = oracle.pack(fmt, w, scales_in=s)
    x = synth.x_bf16(synth.rng(10), 2, k)
    y, _ = oracle.matmul(fmt, codes, scales, n, k, x)
    assert np.all(y == 0.0)


def test_flipping_every_bit_negates_binary():
    g = synth.rng(11)
    n, k = 9, 4 * G
    codes = synth.code_bytes_uniform(g, oracle.codes_bytes("q1g128", n, k))
    scales = synth.scales_uniform(g, n, k // G).reshape(-1)
    x = synth.x_bf16(g, 2, k)
    y, _ = oracle.matmul("q1g128", codes, scales, n, k, x)
    y2, _ = oracle.matmul("q1g128", codes ^ 0xFF, scales, n, k, x)
    assert np.array_equal(y2, -y)


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
def test_one_hot_x_returns_effective_weight_column(fmt):
    g = synth.rng(12)
    n, k = 7, 2 * G
    w = synth.weights_normal(g, n, k)
    codes, scales = oracle.pack(fmt, w)
    wd = oracle.dequant(fmt, codes, scales, n, k)
    for col in (0, 1, 127, 128, 255):
        x = np.zeros((1, k), dtype=np.uint16)
        x[0, col] = 0x3F80
        y, _ = oracle.matmul(fmt, codes, scales, n, k, x)
        assert np.array_equal(y[0], wd[:, col])
        # and the column is s * q with the page's sign meaning
        s = scales.view(np.float16).astype(np.float64).reshape(n, -1)[:, col // G]
        q = oracle.unpack(fmt, codes, n, k)[:, col]
        assert np.array_equal(wd[:, col], s * q)


def test_small_integer_exact_product():
    # power-of-two scales and small-integer activations: the product is an exact integer
    g = synth.rng(13)
    n, k = 4, 2 * G
    t = synth.trits(g, n, k)
    s = np.full((n, k // G), np.float16(2.0).view(np.uint16), dtype=np.uint16)
    w = t.astype(np.float32) * 2.0
    codes, scales = oracle.pack("t2g128", w, scales_in=s)
    xi = g.integers(-8, 9, size=(1, k))
    x = synth.float32_to_bf16_bits(xi.astype(np.float32))
    y, _ = oracle.matmul("t2g128", codes, scales, n, k, x)
    assert np.array_equal(y[0], 2.0 * (t.astype(np.int64) @ xi[0]).astype(np.float64))


def test_rows_variant_matches_full():
    g = synth.rng(14)
    n, k = 50, 2 * G
    w = synth.weights_normal(g, n, k)
    codes, scales = oracle.pack("t5p8", w)
    x = synth.x_bf16(g, 3, k)
    y, b = oracle.matmul("t5p8", codes, scales, n, k, x)
    rows = np.array([49, 0, 17, 17, 3])
    yr, br = oracle.matmul_rows("t5p8", codes, scales, n, k, x, rows)
    assert np.array_equal(yr, y[:, rows]) and np.array_equal(br, b[:, rows])


def test_swiglu_pins():
    """SwiGLU activation of a gated MLP block (8B notes, Table 1), pinned to
    values its definition takes rather than to a retyped formula: sigma(1) =
    e / (1 + e); the BF16 bits of silu(+-1), of a zero gate and of a large
    negative gate (underflow to -0); the odd-part identity silu(v) - silu(-v) = v;
    and the MLP composition on all-plus-one weights."""
    e = 2.718281828459045
    bits, vals = oracle.swiglu(np.array([[1.0, -1.0, 0.0, -100.0, 1.0, 1.0, 5.0, 2.0]]))
    assert vals[0, 0] == pytest.approx(e / (1.0 + e), rel=1e-15)    # 0.7310585786300049
    assert vals[0, 1] == pytest.approx(-1.0 / (1.0 + e), rel=1e-15)  # -0.2689414213699951
    assert list(bits[0]) == [0x3F3B, 0xBE8A, 0x0000, 0x8000]          # 0.73046875, -0.26953125, 0, -0
    # gate 2, up 3: 3 * 2 * sigma(2), sigma(2) = e^2 / (1 + e^2) (a dropped up factor,
    # or gate and up swapped, gives another value)
    bits, vals = oracle.swiglu(np.array([[2.0, 3.0]]))
    assert vals[0, 0] == pytest.approx(6.0 * e * e / (1.0 + e * e), rel=1e-15)  # 5.284782467867294
    assert bits[0, 0] == 0x40A9                                                # 5.28125
    # odd part: gate = [v, -v], up = 1  ->  act[j] - act[inter + j] = v_j
    v = synth.rng(7).normal(0.0, 4.0, 64)
    _, a = oracle.swiglu(np.concatenate([v, -v, np.ones(128)]).reshape(1, -1))
    np.testing.assert_allclose(a[0, :64] - a[0, 64:], v, rtol=1e-13, atol=1e-13)
    # composition: every weight +1 with scale 1 and x one-hot (x_0 = 1) make every
    # gate and up value 1, so act = BF16(silu(1)) = 0.73046875 and each output is
    # inter * 0.73046875 exactly
    hidden, inter = 256, 384
    gu = np.full(oracle.codes_bytes("q1g128", 2 * inter, hidden), 0xFF, dtype=np.uint8)
    gs = np.full(2 * inter * hidden // 128, 0x3C00, dtype=np.uint16)
    dn = np.full(oracle.codes_bytes("q1g128", hidden, inter), 0xFF, dtype=np.uint8)
    ds = np.full(hidden * inter // 128, 0x3C00, dtype=np.uint16)
    x = np.zeros((1, hidden), dtype=np.uint16)
    x[0, 0] = 0x3F80  # BF16 1.0
    y, bound, act = oracle.mlp_swiglu("q1g128", gu, gs, dn, ds, hidden, inter, x)
    assert np.all(act == 0x3F3B)
    assert np.all(y == inter * 0.73046875)
    assert np.all(bound == inter * 0.73046875)


def test_embed_rows_pins():
    """Embedding lookup (8B notes, section 3 and Table 1: the embedding layer is
    low-bit too), pinned to values the definition fixes: bit 1 -> +s and bit 0
    -> -s; a ternary zero is +0; the FP16 scale rounded once to BF16, ties to
    even (1 + 2^-8 is a tie -> 1.0; 1 + 3 2^-8 -> 1 + 2^-6); the rows are the
    ones asked for, in the order asked for; an id past the table is an error."""
    n, k = 4, 256
    codes = np.zeros(oracle.codes_bytes("q1g128", n, k), dtype=np.uint8).reshape(n, k // 8)
    codes[1] = 0xFF                                 # row 1: every weight +s
    codes[2, 0] = 0x01                              # row 2: weight 0 +s, the rest -s
    scales = np.array([[0x3C00, 0x3C00], [0x3C04, 0x3C0C], [0x4000, 0x3800], [0x0001, 0x7BFF]],
                      dtype=np.uint16)              # 1, 1; 1+2^-8, 1+3*2^-8; 2, 0.5; 2^-24, 65504
    out = oracle.embed_rows("q1g128", codes.reshape(-1), scales.reshape(-1), n, k, [1, 0, 2, 3, 1])
    assert out.shape == (5, k)
    assert np.all(out[0, :128] == 0x3F80) and np.all(out[0, 128:] == 0x3F82)   # +1.0 (tie), +1.015625
    assert np.array_equal(out[4], out[0])
    assert np.all(out[1] == 0xBF80)                                              # row 0: all -1.0
    assert out[2, 0] == 0x4000 and np.all(out[2, 1:128] == 0xC000) and np.all(out[2, 128:] == 0xBF00)
    assert np.all(out[3, :128] == 0xB380)           # -2^-24 in BF16 (exactly representable)
    assert np.all(out[3, 128:] == 0xC780)           # -65504 -> BF16 RNE -65536
    # ternary: zero trits give +0, t = +-1 gives +-s
    t = np.array([[0, 1, -1, 0] * 32], dtype=np.float32)
    tc, ts = oracle.pack("t2g128", t * 0.5, scales_in=np.array([0x3800], dtype=np.uint16))
    o2 = oracle.embed_rows("t2g128", tc, ts, 1, 128, [0])
    assert list(o2[0, :4]) == [0x0000, 0x3F00, 0xBF00, 0x0000]
    t5c, t5s = oracle.pack("t5p8", t * 0.5, scales_in=np.array([0x3800], dtype=np.uint16))
    assert np.array_equal(oracle.embed_rows("t5p8", t5c, t5s, 1, 128, [0]), o2)
    with pytest.raises(oracle.OracleError):
        oracle.embed_rows("q1g128", codes.reshape(-1), scales.reshape(-1), n, k, [4])
    with pytest.raises(oracle.OracleError):
        oracle.embed_rows("q1g128", codes.reshape(-1), scales.reshape(-1), n, k, [-1])


def test_affine_storage_pins(golden_dir):
    """Affine 1-bit g128 (MLX-style): one bit plus an FP16 (scale, bias) pair per
    128 weights is 1 + 32/128 = 1.25 bits/weight (page 1, 'MLX打包优化': a scale
    and a bias per group).  For the weight count behind Table 2's GGUF figure
    (1,151,820,864 B at 18 B per 128 weights) that is GGUF x 20/18 =
    1,279,800,960 B, 0.026% under Table 2's MLX 1-bit (g128) package
    (1,280,131,424 B, which also holds the tensors kept unquantised)."""
    facts = json.load(open(os.path.join(golden_dir, "page_facts.json")))
    t2 = facts["table2_bytes"]
    assert oracle.effective_bits("a1g128") == 1.25
    assert oracle.codes_bytes("a1g128", 3, 256) == 3 * 32
    weights = t2["gguf_q1_0_g128"] * 128 // 18
    affine_bytes = weights * (16 + 4) // 128
    assert affine_bytes * 18 == t2["gguf_q1_0_g128"] * 20
    assert 0 < t2["mlx_1bit_g128"] - affine_bytes < 0.0003 * t2["mlx_1bit_g128"]
    assert facts["mlx_scale_and_bias"]["params_per_group"] == ["scale", "bias"]


def test_affine_oracle_pins():
    """The affine product pinned to the native binary product: a native group
    (bits, s) written as affine pairs (2s, -s) gives the same y (w' = 2 s b - s);
    two-level groups reconstruct exactly; a weight exactly half a step above the
    bias takes bit 0 (round half to even), just above it bit 1; one-hot x returns
    the dequantised column; brute force against numpy on a tiny matrix."""
    g = synth.rng(71)
    n, k = 24, 512
    w = synth.weights_normal(g, n, k)
    qc, qs = oracle.pack("q1g128", w)
    x = synth.x_bf16(g, 3, k)
    y_native, _ = oracle.matmul("q1g128", qc, qs, n, k, x)
    s = np.array([oracle.half_to_double(h) for h in qs], dtype=np.float64)
    pairs = np.stack([np.array([oracle.double_to_half(2 * v) for v in s], dtype=np.uint16),
                      np.array([oracle.double_to_half(-v) for v in s], dtype=np.uint16)], axis=1)
    ac, ap = oracle.pack_affine(oracle.dequant("q1g128", qc, qs, n, k).astype(np.float32), params_in=pairs)
    assert np.array_equal(ac, qc)                 # the same bits
    y_aff, bound = oracle.matmul_affine(ac, ap, n, k, x)
    np.testing.assert_allclose(y_aff, y_native, rtol=1e-12, atol=1e-300)
    assert np.all(bound > 0)
    # two levels a < b (FP16-exact, b - a FP16-exact): exact reconstruction
    a, b = -0.375, 0.625
    lv = np.where(g.random((2, 256)) < 0.5, a, b).astype(np.float32)
    lv[:, 0], lv[:, 1] = a, b
    c2, p2 = oracle.pack_affine(lv)
    assert list(p2[:2]) == [oracle.double_to_half(1.0), oracle.double_to_half(a)]
    one = np.zeros((1, 256), dtype=np.uint16)
    for kk in (0, 1, 130, 255):
        xh = one.copy()
        xh[0, kk] = 0x3F80                         # BF16 1.0
        yy, _ = oracle.matmul_affine(c2, p2, 2, 256, xh)
        assert list(yy[0]) == list(lv[:, kk].astype(np.float64))
    # tie: min 0, max 1 -> s = 1, z = 0; w = 0.5 -> bit 0, w = 0.5 + 2^-20 -> bit 1
    tw = np.zeros((1, 128), dtype=np.float32)
    tw[0, 1] = 1.0
    tw[0, 2] = 0.5
    tw[0, 3] = 0.5 + 2.0 ** -20
    tc, tp = oracle.pack_affine(tw)
    assert (tc[0] >> 1) & 1 == 1 and (tc[0] >> 2) & 1 == 0 and (tc[0] >> 3) & 1 == 1
    # brute force against numpy: bits from the pinned binary decoder, (s, z) from the pairs
    wt = synth.weights_normal(g, 5, 256)
    cc, pp = oracle.pack_affine(wt)
    bits = (oracle.unpack("q1g128", cc, 5, 256).astype(np.float64) + 1) / 2
    sz = np.array([oracle.half_to_double(h) for h in pp], dtype=np.float64).reshape(5, 2, 2)
    wd = bits * np.repeat(sz[:, :, 0], 128, axis=1) + np.repeat(sz[:, :, 1], 128, axis=1)
    xt = synth.x_bf16(g, 2, 256)
    xf = np.array([[oracle.bf16_to_double(v) for v in row] for row in xt])
    yb, _ = oracle.matmul_affine(cc, pp, 5, 256, xt)
    np.testing.assert_allclose(yb, xf @ wd.T, rtol=1e-12, atol=1e-15)
    # every reconstruction within half a step of its weight (plus the FP16 roundings)
    err = np.abs(wd - wt.astype(np.float64))
    step = np.repeat(sz[:, :, 0], 128, axis=1)
    assert np.all(err <= step / 2 + 2.0 ** -10 * (np.abs(wt) + step))
    # embedding: the dequantised row rounded once to BF16
    e = oracle.embed_rows_affine(cc, pp, 5, 256, [4, 0])
    assert e[0, 0] == oracle.double_to_bf16(wd[4, 0]) and e[1, 255] == oracle.double_to_bf16(wd[0, 255])
