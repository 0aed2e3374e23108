"""The 5-trit decode of the prefill GEMM and the wide-batch GEMV takes the
base-3 digits of a packed byte from four multiply-shift quotients computed on
two bytes at once (held in the 16-bit halves of a 32-bit word):

    q1 = (x * 171 >> 9)  & 0x007F007F     floor(v / 3)
    q2 = (x *  57 >> 9)  & 0x007F007F     floor(v / 9)
    q3 = (x *  19 >> 9)  & 0x007F007F     floor(v / 27)
    q4 = (x * 203 >> 14) & 0x00030003     floor(v / 81)
    digit i = q_i - 3 q_(i+1)  (q_0 = v, q_5 = 0)

This checks, for every pair of bytes, that the halves do not mix, that each
quotient is exact, that no digit subtraction borrows across the halves, and
that the digits of every valid code (v < 3^5) are its little-endian base-3
digits, the packing rule of the five-trits-per-byte format ("把 27B 模型压到
4GB 跑在手机上", section 2.4: five trits in 8 bits, 3^5 = 243 <= 256)."""
import numpy as np

M32 = 0xFFFFFFFF


def _digits_packed(x):
    q1 = ((x * 171 & M32) >> 9) & 0x007F007F
    q2 = ((x * 57 & M32) >> 9) & 0x007F007F
    q3 = ((x * 19 & M32) >> 9) & 0x007F007F
    q4 = ((x * 203 & M32) >> 14) & 0x00030003
    d = [(x - 3 * q1) & M32, (q1 - 3 * q2) & M32, (q2 - 3 * q3) & M32, (q3 - 3 * q4) & M32, q4]
    return (q1, q2, q3, q4), d


def test_quotients_and_digits_every_byte_pair():
    lo, hi = np.meshgrid(np.arange(256, dtype=np.uint64), np.arange(256, dtype=np.uint64))
    lo, hi = lo.ravel(), hi.ravel()
    x = lo | (hi << np.uint64(16))
    qs, d = _digits_packed(x)
    for half, v in ((0, lo), (16, hi)):
        got = [(q >> np.uint64(half)) & np.uint64(0xFFFF) for q in qs]
        want = [v // 3, v // 9, v // 27, v // 81]
        for g, w in zip(got, want):
            assert np.array_equal(g, w)
        # every digit lies in 0..2 (v mod 3, and floor(v / 3^i) mod 3), so a
        # subtraction never borrows from the other half
        dig = [(e >> np.uint64(half)) & np.uint64(0xFFFF) for e in d]
        for i in range(4):
            assert np.array_equal(dig[i], (v // 3 ** i) % 3)
        assert np.array_equal(dig[4], v // 81)
        valid = v < 243
        assert np.array_equal(dig[4][valid], ((v // 81) % 3)[valid])


def test_single_byte_examples():
    # 0 -> all zero digits; 242 = 2*(1+3+9+27+81) -> all twos; 121 = 1*(1+3+9+27+81) -> all ones
    for v, want in ((0, [0] * 5), (242, [2] * 5), (121, [1] * 5), (5, [2, 1, 0, 0, 0]), (81, [0, 0, 0, 0, 1])):
        _, d = _digits_packed(np.uint64(v))
        assert [int(e) & 0xFFFF for e in d] == want
