"""Host-side checks of the C ABI: the library loads without a GPU, exports
every symbol include/bq.h declares, its host helpers agree with the oracle,
and argument errors are returned before anything touches a device."""
import ctypes
import os
import re

import pytest

import oracle
import ternary_g128_weight_b200 as bq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(bq_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    from ternary_g128_weight_b200 import build
    build.build()
    return bq.load()


def test_every_declared_symbol_is_exported(lib):
    decl = declared_symbols()
    assert {"bq_pack_q1g128", "bq_pack_t2g128", "bq_pack_t5p8", "bq_gemv", "bq_gemm"} <= decl
    for name in decl:
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)
    assert set(bq.EXPORTED) == decl


def test_enums_match_oracle():
    assert (bq.BQ_Q1G128, bq.BQ_T2G128, bq.BQ_T5P8G128) == (oracle.Q1G128, oracle.T2G128, oracle.T5P8G128)
    assert (bq.BQ_OK, bq.BQ_ERR_NULL, bq.BQ_ERR_SHAPE, bq.BQ_ERR_ALIGN, bq.BQ_ERR_NONFINITE,
            bq.BQ_ERR_SCALE_RANGE, bq.BQ_ERR_FORMAT) == (
        oracle.OK, oracle.ERR_NULL, oracle.ERR_SHAPE, oracle.ERR_ALIGN, oracle.ERR_NONFINITE,
        oracle.ERR_SCALE_RANGE, oracle.ERR_FORMAT)


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("n,k", [(0, 128), (1, 128), (7, 1024), (151936, 4096), (3, 100), (-1, 128)])
def test_sizes_match_oracle(lib, fmt, n, k):
    assert bq.bq_codes_bytes(fmt, n, k) == oracle.codes_bytes(fmt, n, k)
    assert bq.bq_scales_bytes(n, k) == oracle.scales_bytes(n, k)
    assert bq.bq_effective_bits(fmt) == oracle.effective_bits(fmt)


def test_status_strings_and_version(lib):
    for s in range(10):
        assert len(bq.status_string(s)) > 0
    assert bq.status_string(99) == "unknown status"
    assert bq.bq_version() >= 100


def _gemv(lib, fmt=1, codes=16, scales=16, n=4, k=128, x=16, batch=1, y=16, ydt=0, ws=None, wsb=0):
    vp = ctypes.c_void_p
    return lib.bq_gemv(fmt, vp(codes) if codes else None, vp(scales) if scales else None, n, k,
                       vp(x) if x else None, batch, vp(y) if y else None, ydt,
                       vp(ws) if ws else None, wsb, None)


def test_argument_errors_need_no_device(lib):
    # host validation happens before any CUDA call, so these run without a GPU
    assert _gemv(lib, fmt=9) == bq.BQ_ERR_FORMAT
    assert _gemv(lib, k=100) == bq.BQ_ERR_SHAPE
    assert _gemv(lib, n=-1) == bq.BQ_ERR_SHAPE
    assert _gemv(lib, batch=0) == bq.BQ_ERR_SHAPE
    assert _gemv(lib, batch=17) == bq.BQ_ERR_SHAPE
    assert _gemv(lib, codes=0) == bq.BQ_ERR_NULL
    assert _gemv(lib, x=0) == bq.BQ_ERR_NULL
    assert _gemv(lib, y=0) == bq.BQ_ERR_NULL
    assert _gemv(lib, codes=24) == bq.BQ_ERR_ALIGN
    assert _gemv(lib, x=8) == bq.BQ_ERR_ALIGN
    assert _gemv(lib, ydt=5) == bq.BQ_ERR_FORMAT
    vp = ctypes.c_void_p
    assert lib.bq_gemm(1, vp(16), vp(16), 4, 130, vp(16), 5, vp(16), None, 0, None) == bq.BQ_ERR_SHAPE
    assert lib.bq_gemm(1, vp(16), vp(16), 4, 128, vp(16), -1, vp(16), None, 0, None) == bq.BQ_ERR_SHAPE
    assert lib.bq_gemm(4, vp(16), vp(16), 4, 128, vp(16), 5, vp(16), None, 0, None) == bq.BQ_ERR_FORMAT
    for name in ("bq_pack_q1g128", "bq_pack_t2g128", "bq_pack_t5p8"):
        f = getattr(lib, name)
        assert f(vp(16), 4, 127, None, vp(16), vp(16), None) == bq.BQ_ERR_SHAPE
        assert f(None, 4, 128, None, vp(16), vp(16), None) == bq.BQ_ERR_NULL
        assert f(vp(20), 4, 128, None, vp(16), vp(16), None) == bq.BQ_ERR_ALIGN
        assert f(vp(16), 0, 128, None, None, None, None) == bq.BQ_OK  # empty: nothing to do
    assert lib.bq_gemv_workspace_bytes(1, 4, 100, 1) == -1
    assert lib.bq_gemv_workspace_bytes(1, 4, 128, 17) == -1
    assert lib.bq_gemv_workspace_bytes(1, 4096, 4096, 1) >= 0
    # launch counts (host-side planning only)
    assert lib.bq_gemv_launches(9, 4096, 4096, 1) == -1
    assert lib.bq_gemv_launches(1, 4096, 100, 1) == -1
    assert lib.bq_gemv_launches(1, 0, 4096, 1) == 0
    assert lib.bq_gemv_launches(1, 4096, 4096, 1) == 1      # row-owning kernel
    assert lib.bq_gemv_launches(2, 4096, 4096, 4) == 1
    assert lib.bq_gemv_launches(3, 4096, 4096, 1) == 1       # 5-trit format, row-owning kernel too
    assert lib.bq_gemv_launches(3, 4096, 17408, 4) in (2, 3)  # operand too large: tcgen05 GEMM
    assert lib.bq_gemv_launches(1, 4096, 4096, 16) == 1       # wide-batch kernel
    assert lib.bq_gemv_launches(3, 4096, 4096, 16) == 1        # 5-trit format at batch 16: wide-batch kernel
    assert lib.bq_gemv_launches(3, 4096, 4096, 8) == 1         # 5-trit format at batch 8: row-owning kernel
    assert lib.bq_gemv_launches(1, 4096, 12288, 16) in (2, 3)  # FP16 x exceeds shared memory: GEMM
    assert lib.bq_gemm_launches(2, 4096, 4096, 12) == 1        # T 5..16: the wide-batch GEMV
    assert lib.bq_gemm_launches(1, 17408, 5120, 4096) == 2     # prep + GEMM, no K split
    assert lib.bq_gemm_launches(1, 4096, 4096, 1) == 1         # T <= 4: the GEMV
    assert lib.bq_gemm_launches(1, 4096, 100, 8) == -1
    assert lib.bq_gemm_workspace_bytes(2, 4096, 4096, 512) >= 0
    assert lib.bq_debug_wait_timeout(-1, None) == bq.BQ_ERR_SHAPE


def test_gemv_path_choice_host_only(lib):
    """Which kernel a bq_gemv call takes is decided on the host (shared memory
    plan at 148 SMs when no device is visible): the row-owning and wide-batch
    kernels need no workspace and one launch; split-K and the GEMM need
    workspace."""
    ws, nl = bq.bq_gemv_workspace_bytes, bq.bq_gemv_launches
    for fmt in ("q1g128", "t2g128", "t5p8"):
        for n, k, b in ((4096, 4096, 1), (151936, 4096, 1), (4096, 12288, 1), (777, 1024, 2)):
            assert ws(fmt, n, k, b) == 0 and nl(fmt, n, k, b) == 1, (fmt, n, k, b)   # row-owning
        assert ws(fmt, 4096, 1152, 1) >= 1152 * 2                                 # K % 1024 != 0: GEMM
    # 5-trit at batch 9..16: the wide-batch kernel where its FP16 x fits, else the GEMM
    assert ws("t5p8", 4096, 4096, 9) == 0 and nl("t5p8", 4096, 4096, 9) == 1
    assert ws("t5p8", 4096, 12288, 16) >= 16 * 12288 * 2
    for fmt in ("q1g128", "t2g128"):
        # batch 5..16: the wide-batch kernel while its FP16 x (2 K bytes per row,
        # rows padded to 8 or 16) fits: batch 16 at K = 4096 (128 KB), batch 8 at
        # K = 12288 (192 KB); batch 16 at K = 12288 (384 KB) goes to the GEMM
        for n, k, b in ((4096, 4096, 9), (16385, 4096, 9), (151936, 4096, 16), (4096, 12288, 8), (5, 1024, 5),
                        (6144, 4096, 6)):
            assert ws(fmt, n, k, b) == 0 and nl(fmt, n, k, b) == 1, (fmt, n, k, b)
        assert ws(fmt, 4096, 12288, 16) >= 16 * 12288 * 2
        assert ws(fmt, 4096, 17408, 4) > 0 and nl(fmt, 4096, 17408, 4) == 2  # operand too large: split-K
    # batch 4 at K = 12288: the operand takes 209 KB; two 5 KB binary slots still fit
    # beside it (row-owning), one 9 KB 2-bit slot does not (split-K)
    assert ws("q1g128", 4096, 12288, 4) == 0 and nl("q1g128", 4096, 12288, 4) == 1
    assert ws("t2g128", 4096, 12288, 4) > 0 and nl("t2g128", 4096, 12288, 4) == 2
    # 5-trit: its 32 KB digit table leaves less room -> GEMM with T = batch where the
    # operand of four n-tiles (batch 8) or of 17 stages at batch 4 does not fit
    assert ws("t5p8", 24576, 4096, 8) >= 8 * 4096 * 2
    assert ws("t5p8", 4096, 17408, 4) >= 4 * 17408 * 2


def test_binding_fails_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.import_module("ternary_g128_weight_b200")
    saved = mod._lib
    try:
        mod._lib = None
        with pytest.raises(RuntimeError, match="no CPU fallback"):
            mod.load(str(tmp_path / "missing.so"))
    finally:
        mod._lib = saved


def test_chain_argument_errors_without_device(lib):
    """bq_gemv_chain rejects bad arguments before touching a device (fake,
    aligned device addresses are never dereferenced on these paths)."""
    S = bq.ChainStep
    A = 0x100000

    def call(steps, nsteps=None, batch=1, ws=A, wsb=256, fmt=bq.BQ_Q1G128):
        arr = (S * max(1, len(steps)))(*steps)
        return lib.bq_gemv_chain(fmt, arr, len(steps) if nsteps is None else nsteps, batch,
                                 ctypes.c_void_p(ws) if ws else None, wsb, None)

    ok = S(A, A, 64, 1024, A, A, bq.BQ_BF16, 0)
    assert call([ok], nsteps=0) == bq.BQ_ERR_SHAPE
    assert call([ok] * 9) == bq.BQ_ERR_SHAPE
    assert call([ok], fmt=9) == bq.BQ_ERR_FORMAT
    assert call([ok], batch=0) == bq.BQ_ERR_SHAPE
    assert call([ok], batch=17) == bq.BQ_ERR_SHAPE
    assert call([S(A, A, 64, 1152, A, A, bq.BQ_BF16, 0)]) == bq.BQ_ERR_SHAPE      # K % 1024 != 0
    assert call([S(A, A, 64, 1000, A, A, bq.BQ_BF16, 0)]) == bq.BQ_ERR_SHAPE      # K % 128 != 0
    assert call([S(A, A, 48, 1024, A, A, bq.BQ_BF16, 1)]) == bq.BQ_ERR_SHAPE      # gate|up not in whole tiles
    assert call([S(A, A, 64, 1024, A, A, 7, 0)]) == bq.BQ_ERR_FORMAT              # output dtype
    assert call([S(A, A, 64, 1024, A, A, bq.BQ_BF16, 2)]) == bq.BQ_ERR_FORMAT     # swiglu flag
    assert call([S(A, A, 64, 1024, 0, A, bq.BQ_BF16, 0)]) == bq.BQ_ERR_NULL       # x
    assert call([S(A, A, 64, 1024, A, A + 2, bq.BQ_BF16, 0)]) == bq.BQ_ERR_ALIGN  # y
    assert call([S(A + 8, A, 64, 1024, A, A, bq.BQ_BF16, 0)]) == bq.BQ_ERR_ALIGN  # codes
    assert call([ok], ws=0) == bq.BQ_ERR_WORKSPACE
    assert call([ok], wsb=16) == bq.BQ_ERR_WORKSPACE
    assert lib.bq_gemv_chain(bq.BQ_Q1G128, None, 1, 1, ctypes.c_void_p(A), 256, None) == bq.BQ_ERR_NULL


def test_affine_sizes_match_oracle(lib):
    for n, k in [(0, 128), (7, 1024), (151936, 4096)]:
        assert bq.bq_codes_bytes("a1g128", n, k) == oracle.codes_bytes("a1g128", n, k) == n * k // 8
        assert bq.bq_group_params_bytes("a1g128", n, k) == n * (k // 128) * 4
        assert bq.bq_group_params_bytes("q1g128", n, k) == bq.bq_scales_bytes(n, k)
    assert bq.bq_effective_bits("a1g128") == oracle.effective_bits("a1g128") == 1.25
    assert bq.bq_gemm_workspace_bytes("a1g128", 64, 1024, 64) == -1


def test_kv4_argument_errors_need_no_device(lib):
    """4-bit KV-cache calls: sizes and argument errors are decided on the host
    before any launch."""
    vp = ctypes.c_void_p
    assert lib.bq_kv4_codes_bytes(10, 128) == 640 and lib.bq_kv4_params_bytes(10, 128) == 40
    assert lib.bq_kv4_codes_bytes(3, 256) == 384 and lib.bq_kv4_params_bytes(3, 256) == 24
    assert lib.bq_kv4_codes_bytes(1, 64) == -1 and lib.bq_kv4_params_bytes(-1, 128) == -1
    assert lib.bq_kv4_quantize(vp(16), 4, 64, vp(16), vp(16), None) == bq.BQ_ERR_SHAPE
    assert lib.bq_kv4_quantize(vp(16), 0, 128, None, None, None) == bq.BQ_OK
    assert lib.bq_kv4_quantize(None, 4, 128, vp(16), vp(16), None) == bq.BQ_ERR_NULL
    assert lib.bq_kv4_quantize(vp(24), 4, 128, vp(16), vp(16), None) == bq.BQ_ERR_ALIGN
    ok_append = dict(batch=2, hkv=2, d=128, l_cap=64)

    def append(**kw):
        a = dict(ok_append, **kw)
        return lib.bq_kv4_append(vp(16), vp(16), a["batch"], a["hkv"], a["d"], vp(16), a["l_cap"], vp(16),
                                 vp(16), vp(16), vp(16), None)
    assert append(l_cap=100) == bq.BQ_ERR_SHAPE
    assert append(d=64) == bq.BQ_ERR_SHAPE
    assert append(batch=0) == bq.BQ_OK
    ws = lib.bq_kv4_attention_workspace_bytes
    assert ws(1, 32, 8, 128, 65536, 65536) > 0      # one sequence: the context is split across CTAs
    assert ws(16, 32, 8, 128, 4096, 4096) == 0      # 128 (sequence, KV head) pairs: one CTA each
    assert ws(1, 36, 4, 128, 64, 64) == -1          # 9 query heads per KV head
    assert ws(1, 32, 8, 96, 64, 64) == -1           # head dimension
    assert ws(1, 32, 8, 128, 100, 64) == -1         # capacity not a multiple of 64
    assert ws(1, 32, 8, 128, 64, 65) == -1          # max_len above the capacity

    def attn(**kw):
        a = dict(q=vp(16), lens=vp(16), batch=1, hq=8, hkv=2, d=128, l_cap=64, max_len=64, scale=0.1,
                 out=vp(16), odt=bq.BQ_BF16)
        a.update(kw)
        return lib.bq_kv4_attention_decode(a["q"], vp(16), vp(16), vp(16), vp(16), a["lens"], a["batch"], a["hq"],
                                           a["hkv"], a["d"], a["l_cap"], a["max_len"], a["scale"], a["out"],
                                           a["odt"], None, 0, None)
    assert attn(d=64) == bq.BQ_ERR_SHAPE
    assert attn(hq=18) == bq.BQ_ERR_SHAPE
    assert attn(odt=9) == bq.BQ_ERR_FORMAT
    assert attn(scale=float("inf")) == bq.BQ_ERR_SHAPE
    assert attn(q=None) == bq.BQ_ERR_NULL
    assert attn(out=vp(8)) == bq.BQ_ERR_ALIGN
    assert attn(lens=vp(18)) == bq.BQ_ERR_ALIGN
    assert attn(batch=0) == bq.BQ_OK
    assert attn(l_cap=65536, max_len=65536, hq=32, hkv=8) == bq.BQ_ERR_WORKSPACE
