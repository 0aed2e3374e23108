"""Python binding of the bq C ABI (include/bq.h) for B200.

Argument marshalling only: every step of packing and of the products runs in
the CUDA kernels of ``libbq.so``.  PyTorch supplies device memory and the
current stream.  There is no fallback: if ``libbq.so`` is missing or a CUDA
device is absent, the calls raise.

Function names match the C entry points.  Tensors are CUDA tensors; shapes and
dtypes follow bq.h (codes uint8, scales uint16 FP16 bits viewed as int16 is
also accepted, x BF16 [B][K]).
"""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libbq.so")

BQ_OK, BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_ALIGN, BQ_ERR_NONFINITE = 0, 1, 2, 3, 4
BQ_ERR_SCALE_RANGE, BQ_ERR_FORMAT, BQ_ERR_CUDA, BQ_ERR_TIMEOUT, BQ_ERR_WORKSPACE = 5, 6, 7, 8, 9
BQ_Q1G128, BQ_T2G128, BQ_T5P8G128, BQ_A1G128 = 1, 2, 3, 4
BQ_BF16, BQ_F32 = 0, 1
BQ_GROUP, BQ_MAX_BATCH = 128, 16
FORMATS = {"q1g128": BQ_Q1G128, "t2g128": BQ_T2G128, "t5p8": BQ_T5P8G128, "a1g128": BQ_A1G128}

EXPORTED = [
    "bq_codes_bytes", "bq_scales_bytes", "bq_group_params_bytes", "bq_effective_bits",
    "bq_pack_q1g128", "bq_pack_t2g128", "bq_pack_t5p8", "bq_pack_a1g128",
    "bq_gemv_workspace_bytes", "bq_gemv_launches", "bq_gemv", "bq_gemv_noalloc",
    "bq_gemm_workspace_bytes", "bq_gemm_launches", "bq_gemm",
    "bq_gemv_chain_workspace_bytes", "bq_gemv_chain", "bq_embed_rows",
    "bq_kv4_codes_bytes", "bq_kv4_params_bytes", "bq_kv4_quantize", "bq_kv4_append",
    "bq_kv4_attention_workspace_bytes", "bq_kv4_attention_decode",
    "bq_check", "bq_debug_wait_timeout", "bq_status_string", "bq_version",
]

_lib = None
BQ_MAX_CHAIN_STEPS = 8


class ChainStep(ctypes.Structure):
    """bq_chain_step of bq.h (device pointers)."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("k", ctypes.c_int64), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("y_dtype", ctypes.c_int),
                ("swiglu", ctypes.c_int)]


class BQError(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call}: {status_string(status)} (status {status})")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbq.so (built by ternary_g128_weight_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python ternary_g128_weight_b200/build.py`"
                           " (there is no CPU fallback)")
    L = ctypes.CDLL(path)
    i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    L.bq_codes_bytes.argtypes = [i32, i64, i64]; L.bq_codes_bytes.restype = i64
    L.bq_scales_bytes.argtypes = [i64, i64]; L.bq_scales_bytes.restype = i64
    L.bq_group_params_bytes.argtypes = [i32, i64, i64]; L.bq_group_params_bytes.restype = i64
    L.bq_effective_bits.argtypes = [i32]; L.bq_effective_bits.restype = ctypes.c_double
    for name in ("bq_pack_q1g128", "bq_pack_t2g128", "bq_pack_t5p8", "bq_pack_a1g128"):
        f = getattr(L, name)
        f.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        f.restype = i32
    L.bq_gemv_workspace_bytes.argtypes = [i32, i64, i64, i32]; L.bq_gemv_workspace_bytes.restype = i64
    L.bq_gemv_launches.argtypes = [i32, i64, i64, i32]; L.bq_gemv_launches.restype = i32
    L.bq_gemv.argtypes = [i32, vp, vp, i64, i64, vp, i32, vp, i32, vp, sz, vp]; L.bq_gemv.restype = i32
    L.bq_gemv_noalloc.argtypes = [i32, vp, vp, i64, i64, vp, i32, vp, i32, vp]; L.bq_gemv_noalloc.restype = i32
    L.bq_gemm_workspace_bytes.argtypes = [i32, i64, i64, i64]; L.bq_gemm_workspace_bytes.restype = i64
    L.bq_gemm_launches.argtypes = [i32, i64, i64, i64]; L.bq_gemm_launches.restype = i32
    L.bq_gemm.argtypes = [i32, vp, vp, i64, i64, vp, i64, vp, vp, sz, vp]; L.bq_gemm.restype = i32
    L.bq_embed_rows.argtypes = [i32, vp, vp, i64, i64, vp, i64, vp, vp]; L.bq_embed_rows.restype = i32
    L.bq_kv4_codes_bytes.argtypes = [i64, i32]; L.bq_kv4_codes_bytes.restype = i64
    L.bq_kv4_params_bytes.argtypes = [i64, i32]; L.bq_kv4_params_bytes.restype = i64
    L.bq_kv4_quantize.argtypes = [vp, i64, i32, vp, vp, vp]; L.bq_kv4_quantize.restype = i32
    L.bq_kv4_append.argtypes = [vp, vp, i32, i32, i32, vp, i64, vp, vp, vp, vp, vp]; L.bq_kv4_append.restype = i32
    L.bq_kv4_attention_workspace_bytes.argtypes = [i32, i32, i32, i32, i64, i64]
    L.bq_kv4_attention_workspace_bytes.restype = i64
    L.bq_kv4_attention_decode.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, i64, ctypes.c_float,
                                          vp, i32, vp, sz, vp]
    L.bq_kv4_attention_decode.restype = i32
    L.bq_gemv_chain_workspace_bytes.argtypes = []; L.bq_gemv_chain_workspace_bytes.restype = i64
    L.bq_gemv_chain.argtypes = [i32, ctypes.POINTER(ChainStep), i32, i32, vp, sz, vp]
    L.bq_gemv_chain.restype = i32
    L.bq_check.argtypes = [vp]; L.bq_check.restype = i32
    L.bq_debug_wait_timeout.argtypes = [i64, vp]; L.bq_debug_wait_timeout.restype = i32
    L.bq_status_string.argtypes = [i32]; L.bq_status_string.restype = ctypes.c_char_p
    L.bq_version.argtypes = []; L.bq_version.restype = i32
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().bq_status_string(int(status)).decode()


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, call: str):
    if status != BQ_OK:
        raise BQError(status, call)


# ------------------------------------------------------------------- sizes
def bq_codes_bytes(fmt, n: int, k: int) -> int:
    return int(load().bq_codes_bytes(_fmt(fmt), n, k))


def bq_scales_bytes(n: int, k: int) -> int:
    return int(load().bq_scales_bytes(n, k))


def bq_group_params_bytes(fmt, n: int, k: int) -> int:
    return int(load().bq_group_params_bytes(_fmt(fmt), n, k))


def bq_effective_bits(fmt) -> float:
    return float(load().bq_effective_bits(_fmt(fmt)))


def bq_version() -> int:
    return int(load().bq_version())


# ----------------------------------------------------------------- packers
def _pack(name: str, fmt: int, w, scales_in=None, codes=None, scales=None, stream=None):
    import torch
    n, k = w.shape
    cb, sb = bq_codes_bytes(fmt, n, k), bq_group_params_bytes(fmt, n, k)
    if cb < 0 or sb < 0:
        raise BQError(BQ_ERR_SHAPE, name)
    if codes is None:
        codes = torch.empty(cb, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(sb // 2, dtype=torch.int16, device=w.device)
    st = getattr(load(), name)(_ptr(w), n, k, _ptr(scales_in), _ptr(codes), _ptr(scales), _stream(stream))
    _check(st, name)
    return codes, scales


def bq_pack_q1g128(w, scales_in=None, codes=None, scales=None, stream=None):
    """float32 CUDA W [N][K] -> (codes uint8, scales int16 holding FP16 bits)."""
    return _pack("bq_pack_q1g128", BQ_Q1G128, w, scales_in, codes, scales, stream)


def bq_pack_t2g128(w, scales_in=None, codes=None, scales=None, stream=None):
    return _pack("bq_pack_t2g128", BQ_T2G128, w, scales_in, codes, scales, stream)


def bq_pack_t5p8(w, scales_in=None, codes=None, scales=None, stream=None):
    return _pack("bq_pack_t5p8", BQ_T5P8G128, w, scales_in, codes, scales, stream)


def bq_pack_a1g128(w, params_in=None, codes=None, params=None, stream=None):
    """Affine 1-bit: (codes uint8, params int16 holding FP16 (scale, bias) pairs [N][G][2])."""
    return _pack("bq_pack_a1g128", BQ_A1G128, w, params_in, codes, params, stream)


PACKERS = {BQ_Q1G128: bq_pack_q1g128, BQ_T2G128: bq_pack_t2g128, BQ_T5P8G128: bq_pack_t5p8,
           BQ_A1G128: bq_pack_a1g128}


def bq_pack(fmt, w, scales_in=None, codes=None, scales=None, stream=None):
    return PACKERS[_fmt(fmt)](w, scales_in, codes, scales, stream)


# -------------------------------------------------------------------- GEMV
def bq_gemv_workspace_bytes(fmt, n: int, k: int, batch: int) -> int:
    return int(load().bq_gemv_workspace_bytes(_fmt(fmt), n, k, batch))


def bq_gemv_launches(fmt, n: int, k: int, batch: int) -> int:
    return int(load().bq_gemv_launches(_fmt(fmt), n, k, batch))


def bq_gemv(fmt, codes, scales, n: int, k: int, x, y=None, y_dtype: int = BQ_BF16,
            workspace=None, stream=None):
    """y[b][r] = sum_k s q x (see bq.h).  x: BF16 CUDA tensor [batch][K]."""
    import torch
    f = _fmt(fmt)
    batch = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((batch, n), dtype=torch.float32 if y_dtype == BQ_F32 else torch.bfloat16,
                        device=x.device)
    need = bq_gemv_workspace_bytes(f, n, k, batch)
    if need > 0 and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().bq_gemv(f, _ptr(codes), _ptr(scales), n, k, _ptr(x), batch, _ptr(y), int(y_dtype),
                        _ptr(workspace), wsb, _stream(stream))
    _check(st, "bq_gemv")
    return y


BQ_NOALLOC_SCRATCH_BYTES = 4 << 20


def bq_gemv_noalloc(fmt, codes, scales, n: int, k: int, x, y=None, y_dtype: int = BQ_BF16, stream=None):
    """bq_gemv without a workspace argument: the library's fixed scratch array is
    used instead (for callers that cannot allocate device memory).  Calls that
    overlap on the GPU race on that array; make the first call on a device
    before capturing a stream."""
    import torch
    f = _fmt(fmt)
    batch = x.shape[0] if x.dim() == 2 else 1
    if y is None:
        y = torch.empty((batch, n), dtype=torch.float32 if y_dtype == BQ_F32 else torch.bfloat16,
                        device=x.device)
    st = load().bq_gemv_noalloc(f, _ptr(codes), _ptr(scales), n, k, _ptr(x), batch, _ptr(y), int(y_dtype),
                                _stream(stream))
    _check(st, "bq_gemv_noalloc")
    return y


# -------------------------------------------------------------------- GEMM
def bq_gemm_workspace_bytes(fmt, n: int, k: int, t: int) -> int:
    return int(load().bq_gemm_workspace_bytes(_fmt(fmt), n, k, t))


def bq_gemm_launches(fmt, n: int, k: int, t: int) -> int:
    return int(load().bq_gemm_launches(_fmt(fmt), n, k, t))


def bq_gemm(fmt, codes, scales, n: int, k: int, x, y=None, workspace=None, stream=None):
    """Y[t][r] = sum_k X[t][k] s q (BF16 out).  x: BF16 CUDA tensor [T][K]."""
    import torch
    f = _fmt(fmt)
    t = x.shape[0]
    if y is None:
        y = torch.empty((t, n), dtype=torch.bfloat16, device=x.device)
    need = bq_gemm_workspace_bytes(f, n, k, t)
    if need > 0 and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().bq_gemm(f, _ptr(codes), _ptr(scales), n, k, _ptr(x), t, _ptr(y),
                        _ptr(workspace), wsb, _stream(stream))
    _check(st, "bq_gemm")
    return y


# --------------------------------------------------------------- embedding
def bq_embed_rows(fmt, codes, scales, n: int, k: int, ids, out=None, stream=None):
    """BF16 rows ids (int32 CUDA tensor) of the n x k low-bit table, [count][k]."""
    import torch
    ids = ids.reshape(-1)
    if out is None:
        out = torch.empty((ids.numel(), k), dtype=torch.bfloat16, device=ids.device)
    st = load().bq_embed_rows(_fmt(fmt), _ptr(codes), _ptr(scales), n, k, _ptr(ids), ids.numel(), _ptr(out),
                              _stream(stream))
    _check(st, "bq_embed_rows")
    return out


# ------------------------------------------------------------------ chains
def bq_gemv_chain_workspace_bytes() -> int:
    return int(load().bq_gemv_chain_workspace_bytes())


def bq_gemv_chain(fmt, steps, workspace=None, stream=None):
    """Run the products of `steps` in order in one persistent launch (see bq.h).
    steps: list of dicts with keys codes, scales, n, k, x (BF16 [batch][K] CUDA
    tensor), y (output tensor: float32 for F32 output, else BF16) and optionally
    swiglu (bool).  workspace: a zero-filled CUDA uint8 tensor of >=
    bq_gemv_chain_workspace_bytes() bytes, reused across calls (a fresh zeroed
    one is made when None)."""
    import torch
    f = _fmt(fmt)
    arr = (ChainStep * len(steps))()
    batch = None
    for i, st in enumerate(steps):
        x = st["x"]
        b = x.shape[0] if x.dim() == 2 else 1
        batch = b if batch is None else batch
        ydt = BQ_F32 if st["y"].dtype == torch.float32 else BQ_BF16
        arr[i] = ChainStep(st["codes"].data_ptr(), st["scales"].data_ptr(), int(st["n"]), int(st["k"]),
                           x.data_ptr(), st["y"].data_ptr(), ydt, 1 if st.get("swiglu") else 0)
    if workspace is None:
        workspace = torch.zeros(bq_gemv_chain_workspace_bytes(), dtype=torch.uint8, device=steps[0]["x"].device)
    wsb = workspace.numel() * workspace.element_size()
    st = load().bq_gemv_chain(f, arr, len(steps), int(batch or 0), _ptr(workspace), wsb, _stream(stream))
    _check(st, "bq_gemv_chain")
    return workspace


# ------------------------------------------------------------------ errors
def bq_check(stream=None) -> int:
    return int(load().bq_check(_stream(stream)))


def bq_debug_wait_timeout(spin_limit: int, stream=None) -> int:
    return int(load().bq_debug_wait_timeout(int(spin_limit), _stream(stream)))


def bq_status_string(status: int) -> str:
    return status_string(status)


# ---------------------------------------------------------- 4-bit KV cache
def bq_kv4_codes_bytes(rows: int, d: int) -> int:
    return int(load().bq_kv4_codes_bytes(rows, d))


def bq_kv4_params_bytes(rows: int, d: int) -> int:
    return int(load().bq_kv4_params_bytes(rows, d))


def bq_kv4_quantize(x, codes=None, params=None, stream=None):
    """Quantise BF16 vectors x [..., d] (CUDA) to the 4-bit g128 cache format:
    returns (codes uint8 [..., d/2], params int32 [..., d/128]) (the given
    buffers if passed)."""
    import torch
    d = x.shape[-1]
    lead = tuple(x.shape[:-1])
    rows = x.numel() // d if d else 0
    if codes is None:
        codes = torch.empty(lead + (d // 2,), dtype=torch.uint8, device=x.device)
    if params is None:
        params = torch.empty(lead + (d // 128,), dtype=torch.int32, device=x.device)
    st = load().bq_kv4_quantize(_ptr(x), rows, d, _ptr(codes), _ptr(params), _stream(stream))
    _check(st, "bq_kv4_quantize")
    return codes, params


def bq_kv4_append(k, v, pos, k_codes, k_params, v_codes, v_params, stream=None):
    """Write the new K and V (BF16 [B][Hkv][d]) into row pos[b] (int32 CUDA
    tensor [B]) of the caches (codes uint8 [B][Hkv][L_cap][d/2], params int32
    [B][Hkv][L_cap][d/128])."""
    B, hkv, d = k.shape
    l_cap = k_codes.shape[2]
    st = load().bq_kv4_append(_ptr(k), _ptr(v), B, hkv, d, _ptr(pos), l_cap, _ptr(k_codes), _ptr(k_params),
                              _ptr(v_codes), _ptr(v_params), _stream(stream))
    _check(st, "bq_kv4_append")


def bq_kv4_attention_workspace_bytes(batch: int, hq: int, hkv: int, d: int, l_cap: int, max_len: int) -> int:
    return int(load().bq_kv4_attention_workspace_bytes(batch, hq, hkv, d, l_cap, max_len))


def bq_kv4_attention_decode(q, k_codes, k_params, v_codes, v_params, lens, max_len: int, scale: float,
                            out=None, out_dtype=None, workspace=None, stream=None):
    """Decode attention of q (BF16 [B][Hq][d]) over the 4-bit caches (see bq.h);
    lens int32 CUDA [B].  Returns (out, workspace); pass the workspace back to
    reuse it (a zero-filled one is made when None)."""
    import torch
    B, hq, d = q.shape
    hkv, l_cap = k_codes.shape[1], k_codes.shape[2]
    if out is None:
        dt = torch.float32 if out_dtype == BQ_F32 else torch.bfloat16
        out = torch.empty((B, hq, d), dtype=dt, device=q.device)
    odt = BQ_F32 if out.dtype == torch.float32 else BQ_BF16
    need = bq_kv4_attention_workspace_bytes(B, hq, hkv, d, l_cap, max_len)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=q.device)
    wsb = workspace.numel() * workspace.element_size()
    st = load().bq_kv4_attention_decode(_ptr(q), _ptr(k_codes), _ptr(k_params), _ptr(v_codes), _ptr(v_params),
                                        _ptr(lens), B, hq, hkv, d, l_cap, max_len, float(scale), _ptr(out), odt,
                                        _ptr(workspace), wsb, _stream(stream))
    _check(st, "bq_kv4_attention_decode")
    return out, workspace
