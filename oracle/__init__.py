"""CPU oracle for the binary / ternary g128 weight path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline
leg and its reference arm) may import this package.  The CUDA library never
imports it and it never imports the CUDA library; the two share no code.

Everything is computed in FP64 by plain C (``bq_oracle.c``), following the
pages it cites:

* "Bonsai-27B-mlx-1bit ... Binary g128" (binary g128 representation: sign bit
  0 -> -scale, 1 -> +scale, one FP16 scale per 128 weights, 1.125 bits/weight);
* "Ternary Bonsai" (trits times an FP16 group scale, ~1.71 bits/weight, stored
  in 2-bit slots);
* "把 27B 模型压到 4GB 跑在手机上" section 2.4 (2-bit slots waste a code; five
  trits per byte since 3^5 = 243 <= 256);
* "1-bit Bonsai 8B" notes section 4.1 (bits mapped to signed values times the
  group scale, decoded inside the matmul), Table 2 (package sizes) and Table 1
  (SwiGLU feed-forward: ``swiglu`` / ``mlp_swiglu``, with the BF16 rounding of
  the activation a reading, not a page fact).

The 4-bit KV cache and its decode attention live in ``oracle.kv4`` (numpy
FP64; "Bonsai-27B-mlx-1bit ... Binary g128", sections "峰值内存管理" and
"KV压缩潜力"; "Ternary Bonsai", hybrid attention with a 4-bit KV cache).

Parity status: the packing rules (mean-|w| scale, zero maps to +1, ternary
threshold s/2, bit order, base-3 digit order) are readings of pages that do not
state them; they are pinned to closed forms and invariants, not to any
published artefact.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build
from . import kv4  # noqa: F401  (4-bit KV cache oracle)

Q1G128, T2G128, T5P8G128, A1G128 = 1, 2, 3, 4
FORMATS = {"q1g128": Q1G128, "t2g128": T2G128, "t5p8": T5P8G128, "a1g128": A1G128}
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_NONFINITE, ERR_SCALE_RANGE, ERR_FORMAT = range(7)
GROUP = 128

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i8p = ctypes.POINTER(ctypes.c_int8)
        L.bqo_half_to_double.argtypes = [ctypes.c_uint16]
        L.bqo_half_to_double.restype = ctypes.c_double
        L.bqo_double_to_half.argtypes = [ctypes.c_double]
        L.bqo_double_to_half.restype = ctypes.c_uint16
        L.bqo_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.bqo_bf16_to_double.restype = ctypes.c_double
        L.bqo_double_to_bf16.argtypes = [ctypes.c_double]
        L.bqo_double_to_bf16.restype = ctypes.c_uint16
        L.bqo_codes_bytes.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64]
        L.bqo_codes_bytes.restype = ctypes.c_int64
        L.bqo_scales_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        L.bqo_scales_bytes.restype = ctypes.c_int64
        L.bqo_effective_bits.argtypes = [ctypes.c_int]
        L.bqo_effective_bits.restype = ctypes.c_double
        L.bqo_weight_code.argtypes = [ctypes.c_int, u8p, ctypes.c_int64]
        L.bqo_weight_code.restype = ctypes.c_int
        L.bqo_pack.argtypes = [ctypes.c_int, f32p, ctypes.c_int64, ctypes.c_int64, u16p, u8p, u16p]
        L.bqo_pack.restype = ctypes.c_int
        L.bqo_unpack.argtypes = [ctypes.c_int, u8p, ctypes.c_int64, ctypes.c_int64, i8p]
        L.bqo_unpack.restype = ctypes.c_int
        L.bqo_matmul.argtypes = [ctypes.c_int, u8p, u16p, ctypes.c_int64, ctypes.c_int64, u16p,
                                 ctypes.c_int64, f64p, f64p, ctypes.c_int]
        L.bqo_matmul.restype = ctypes.c_int
        L.bqo_matmul_rows.argtypes = [ctypes.c_int, u8p, u16p, ctypes.c_int64, ctypes.c_int64, u16p,
                                      ctypes.c_int64, i64p, ctypes.c_int64, f64p, f64p, ctypes.c_int]
        L.bqo_matmul_rows.restype = ctypes.c_int
        L.bqo_swiglu.argtypes = [f64p, ctypes.c_int64, ctypes.c_int64, u16p, f64p]
        L.bqo_swiglu.restype = ctypes.c_int
        L.bqo_embed_rows.argtypes = [ctypes.c_int, u8p, u16p, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.POINTER(ctypes.c_int32), ctypes.c_int64, u16p]
        L.bqo_embed_rows.restype = ctypes.c_int
        L.bqo_pack_affine.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_int64, ctypes.c_int64, u16p, u8p, u16p]
        L.bqo_pack_affine.restype = ctypes.c_int
        L.bqo_matmul_affine.argtypes = [u8p, u16p, ctypes.c_int64, ctypes.c_int64, u16p, ctypes.c_int64, i64p,
                                        ctypes.c_int64, f64p, f64p, ctypes.c_int]
        L.bqo_matmul_affine.restype = ctypes.c_int
        L.bqo_embed_rows_affine.argtypes = [u8p, u16p, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.POINTER(ctypes.c_int32), ctypes.c_int64, u16p]
        L.bqo_embed_rows_affine.restype = ctypes.c_int
        L.bqo_max_threads.argtypes = []
        L.bqo_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"oracle {what} failed with status {status}")
        self.status = status


# ---------------------------------------------------------------- conversions
def half_to_double(h: int) -> float:
    return lib().bqo_half_to_double(int(h))


def double_to_half(v: float) -> int:
    return int(lib().bqo_double_to_half(float(v)))


def bf16_to_double(b: int) -> float:
    return lib().bqo_bf16_to_double(int(b))


def double_to_bf16(v: float) -> int:
    return int(lib().bqo_double_to_bf16(float(v)))


# ------------------------------------------------------------------- storage
def codes_bytes(fmt, n: int, k: int) -> int:
    return int(lib().bqo_codes_bytes(_fmt(fmt), n, k))


def scales_bytes(n: int, k: int) -> int:
    return int(lib().bqo_scales_bytes(n, k))


def effective_bits(fmt) -> float:
    return float(lib().bqo_effective_bits(_fmt(fmt)))


def weight_code(fmt, row_codes: np.ndarray, k: int) -> int:
    row_codes = np.ascontiguousarray(row_codes, dtype=np.uint8)
    return int(lib().bqo_weight_code(_fmt(fmt), _ptr(row_codes, ctypes.c_uint8), k))


# ---------------------------------------------------------------------- pack
def pack_status(fmt, w: np.ndarray, scales_in: np.ndarray | None = None):
    """Returns (status, codes, scales).  w: float32 [n][k]."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    f = _fmt(fmt)
    cb = max(codes_bytes(f, n, k), 0)
    sb = max(scales_bytes(n, k), 0)
    codes = np.zeros(cb, dtype=np.uint8)
    scales = np.zeros(sb // 2, dtype=np.uint16)
    sin = None
    if scales_in is not None:
        sin = np.ascontiguousarray(scales_in, dtype=np.uint16).reshape(-1)
    st = lib().bqo_pack(f, _ptr(w, ctypes.c_float), n, k,
                        _ptr(sin, ctypes.c_uint16) if sin is not None else None,
                        _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint16))
    return st, codes, scales


def pack(fmt, w: np.ndarray, scales_in: np.ndarray | None = None):
    st, codes, scales = pack_status(fmt, w, scales_in)
    if st != OK:
        raise OracleError(st, "pack")
    return codes, scales


def unpack(fmt, codes: np.ndarray, n: int, k: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    q = np.zeros((n, k), dtype=np.int8)
    st = lib().bqo_unpack(_fmt(fmt), _ptr(codes, ctypes.c_uint8), n, k, _ptr(q, ctypes.c_int8))
    if st != OK:
        raise OracleError(st, "unpack")
    return q


def dequant(fmt, codes: np.ndarray, scales: np.ndarray, n: int, k: int) -> np.ndarray:
    """FP64 effective weights s * q, [n][k]."""
    q = unpack(fmt, codes, n, k).astype(np.float64)
    s = np.array([half_to_double(h) for h in np.asarray(scales, dtype=np.uint16).reshape(-1)],
                 dtype=np.float64).reshape(n, k // GROUP)
    return q * np.repeat(s, GROUP, axis=1)


# -------------------------------------------------------------------- matmul
def matmul(fmt, codes, scales, n: int, k: int, x_bf16: np.ndarray, nthreads: int = 0):
    """y[b][n] (FP64) and bound[b][n] = sum_k |s x| for BF16 x[b][k]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, k)
    batch = x.shape[0]
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    y = np.zeros((batch, n), dtype=np.float64)
    bound = np.zeros((batch, n), dtype=np.float64)
    st = lib().bqo_matmul(_fmt(fmt), _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint16),
                          n, k, _ptr(x, ctypes.c_uint16), batch,
                          _ptr(y, ctypes.c_double), _ptr(bound, ctypes.c_double), int(nthreads))
    if st != OK:
        raise OracleError(st, "matmul")
    return y, bound


def matmul_rows(fmt, codes, scales, n: int, k: int, x_bf16: np.ndarray, rows, nthreads: int = 0):
    """Like matmul but only for the listed rows: outputs [b][len(rows)]."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, k)
    batch = x.shape[0]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    y = np.zeros((batch, rows.size), dtype=np.float64)
    bound = np.zeros((batch, rows.size), dtype=np.float64)
    st = lib().bqo_matmul_rows(_fmt(fmt), _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint16),
                               n, k, _ptr(x, ctypes.c_uint16), batch,
                               _ptr(rows, ctypes.c_int64), rows.size,
                               _ptr(y, ctypes.c_double), _ptr(bound, ctypes.c_double), int(nthreads))
    if st != OK:
        raise OracleError(st, "matmul_rows")
    return y, bound


def swiglu(h: np.ndarray):
    """SwiGLU of h[b] = [gate | up] (FP64, length 2 * inter): act[b][j] =
    BF16_RNE(silu(gate_j) * up_j), silu(v) = v / (1 + e^-v).  Returns the BF16
    bits [b][inter] and the unrounded FP64 values."""
    h = np.ascontiguousarray(h, dtype=np.float64)
    if h.ndim == 1:
        h = h.reshape(1, -1)
    batch, two_i = h.shape
    if two_i % 2:
        raise OracleError(ERR_SHAPE, "swiglu")
    inter = two_i // 2
    bits = np.zeros((batch, inter), dtype=np.uint16)
    vals = np.zeros((batch, inter), dtype=np.float64)
    st = lib().bqo_swiglu(_ptr(h, ctypes.c_double), batch, inter, _ptr(bits, ctypes.c_uint16),
                          _ptr(vals, ctypes.c_double))
    if st != OK:
        raise OracleError(st, "swiglu")
    return bits, vals


def mlp_swiglu(fmt, gu_codes, gu_scales, d_codes, d_scales, hidden: int, inter: int, x_bf16: np.ndarray):
    """A gated MLP block on low-bit weights: h = W_gate|up x ([2 inter][hidden]
    weights), act = swiglu(h) in BF16, y = W_down act ([hidden][inter]
    weights).  Returns y, its bound sum |s act| for the BF16 act, and act's bits."""
    h, _ = matmul(fmt, gu_codes, gu_scales, 2 * inter, hidden, x_bf16)
    act, _ = swiglu(h)
    y, bound = matmul(fmt, d_codes, d_scales, hidden, inter, act)
    return y, bound, act


def embed_rows(fmt, codes, scales, n: int, k: int, ids) -> np.ndarray:
    """BF16 bits [count][k] of the dequantised rows ids of an n x k table."""
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.zeros((ids.size, k), dtype=np.uint16)
    st = lib().bqo_embed_rows(_fmt(fmt), _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_uint16), n, k,
                              _ptr(ids, ctypes.c_int32), ids.size, _ptr(out, ctypes.c_uint16))
    if st != OK:
        raise OracleError(st, "embed_rows")
    return out


def pack_affine(w: np.ndarray, params_in: np.ndarray | None = None):
    """Affine 1-bit g128 (w' = s b + z): codes (as the binary format) and the
    FP16 (s, z) pairs [N][G][2] (uint16 bits, flattened)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    codes = np.zeros(n * (k // 8), dtype=np.uint8)
    params = np.zeros(n * (k // GROUP) * 2, dtype=np.uint16)
    pin = None if params_in is None else np.ascontiguousarray(params_in, dtype=np.uint16).reshape(-1)
    st = lib().bqo_pack_affine(w.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), n, k,
                               None if pin is None else _ptr(pin, ctypes.c_uint16),
                               _ptr(codes, ctypes.c_uint8), _ptr(params, ctypes.c_uint16))
    if st != OK:
        raise OracleError(st, "pack_affine")
    return codes, params


def matmul_affine(codes, params, n: int, k: int, x_bf16: np.ndarray, rows=None, nthreads: int = 0):
    """y[b][rows] and bound[b][rows] of the affine product (all rows if rows is None)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, k)
    batch = x.shape[0]
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    params = np.ascontiguousarray(params, dtype=np.uint16)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    R = n if r is None else r.size
    y = np.zeros((batch, R), dtype=np.float64)
    bound = np.zeros((batch, R), dtype=np.float64)
    st = lib().bqo_matmul_affine(_ptr(codes, ctypes.c_uint8), _ptr(params, ctypes.c_uint16), n, k,
                                 _ptr(x, ctypes.c_uint16), batch, None if r is None else _ptr(r, ctypes.c_int64),
                                 R, _ptr(y, ctypes.c_double), _ptr(bound, ctypes.c_double), int(nthreads))
    if st != OK:
        raise OracleError(st, "matmul_affine")
    return y, bound


def embed_rows_affine(codes, params, n: int, k: int, ids) -> np.ndarray:
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    params = np.ascontiguousarray(params, dtype=np.uint16)
    out = np.zeros((ids.size, k), dtype=np.uint16)
    st = lib().bqo_embed_rows_affine(_ptr(codes, ctypes.c_uint8), _ptr(params, ctypes.c_uint16), n, k,
                                     _ptr(ids, ctypes.c_int32), ids.size, _ptr(out, ctypes.c_uint16))
    if st != OK:
        raise OracleError(st, "embed_rows_affine")
    return out


def max_threads() -> int:
    return int(lib().bqo_max_threads())
