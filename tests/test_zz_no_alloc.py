"""The allocation-free GEMV entry point (bq_gemv_noalloc), called through the
C ABI: on two calls in a row it must give the same outputs as bq_gemv with a
caller-provided workspace, within the stated tolerance.  It serves callers
that cannot allocate device memory where they run the product, so it uses the
library's fixed scratch array instead of a workspace argument.

This file is collected last so that a run stopping at the first failure has
already run every other test; it passes alone in a fresh process and after
the other tests."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, to_dev, x_to_dev

pytestmark = pytest.mark.gpu


def _noalloc_call(fmt, c, s, n, k, x, y, ydt):
    import torch
    lib = bq.load()
    vp = ctypes.c_void_p
    st = lib.bq_gemv_noalloc(bq._fmt(fmt), vp(c.data_ptr()), vp(s.data_ptr()), n, k, vp(x.data_ptr()),
                             x.shape[0], vp(y.data_ptr()), ydt, vp(torch.cuda.current_stream().cuda_stream))
    return st


def _host_case(fmt, n, k, batch, seed):
    g = synth.rng(seed)
    if fmt == "q1g128":
        codes, scales = oracle.pack(fmt, synth.weights_normal(g, n, k))
    else:
        t = synth.trits(g, n, k)
        s = synth.scales_uniform(g, n, k // 128)
        codes, scales = oracle.pack(fmt, t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), 128, axis=1),
                                    scales_in=s)
    return codes, scales, synth.x_bf16(g, batch, k)


# Shapes on every path bq_gemv can take.  The first seven need no scratch (the
# row-owning kernel; the wide-batch kernel at batch 9 and 6, and for the 5-trit
# format at batch 9); the rest use the fixed array: the split-K kernel
# (activation operand too large for shared memory at batch 4) and the tcgen05
# GEMM with T = batch (the 5-trit format at batch 16 and K = 12288, K % 1024 !=
# 0, the 5-trit format at batch 4 and large K).
NO_SCRATCH = [("q1g128", 4096, 4096, 1), ("t2g128", 3000, 2048, 3), ("q1g128", 777, 12288, 2),
              ("t5p8", 500, 1024, 1), ("q1g128", 16385, 4096, 9), ("t2g128", 129, 8192, 6),
              ("t5p8", 4096, 4096, 9)]
SCRATCH = [("t2g128", 4096, 12288, 4), ("q1g128", 4096, 17408, 4), ("t5p8", 4096, 12288, 16),
           ("q1g128", 4096, 1152, 1), ("t5p8", 4096, 17408, 4)]


@pytest.mark.parametrize("fmt,n,k,batch", NO_SCRATCH + SCRATCH)
def test_noalloc_matches_workspace_gemv_twice(fmt, n, k, batch):
    """Two calls in a row through the C ABI, each equal to bq_gemv (with a
    caller workspace) and to the oracle.  Between them a call of another shape
    on the same scratch array leaves different contents behind, so the second
    call also shows that whatever must start at zero is cleared by the call."""
    import torch
    need = bq.bq_gemv_workspace_bytes(fmt, n, k, batch)
    if (fmt, n, k, batch) in SCRATCH:
        assert 0 < need <= bq.BQ_NOALLOC_SCRATCH_BYTES, need
    else:
        assert need == 0
    codes, scales, x = _host_case(fmt, n, k, batch, synth.SEED_BASE + 300 + n + k + batch)
    c, s_, xd = to_dev(codes), to_dev(scales.astype(np.int16)), x_to_dev(x)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    ydt = bq.BQ_F32
    y_ws = bq.bq_gemv(fmt, c, s_, n, k, xd, y_dtype=ydt)
    # another shape that uses the scratch array (split-K: counters and partials)
    on, ok_, ob = 512, 17408, 4
    oc, os_, ox = _host_case("q1g128", on, ok_, ob, synth.SEED_BASE + 399)
    oc, os_, ox = to_dev(oc), to_dev(os_.astype(np.int16)), x_to_dev(ox)
    oy = torch.empty((ob, on), dtype=torch.float32, device="cuda")
    for call in range(2):
        y = torch.full((batch, n), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_call(fmt, c, s_, n, k, xd, y, ydt) == bq.BQ_OK
        torch.cuda.synchronize()
        assert bq.bq_check() == bq.BQ_OK
        check_close(y, y_ws.cpu().numpy().astype(np.float64), bound, "f32", strict=True,
                    what=f"noalloc vs bq_gemv, call {call}")
        check_close(y, yref, bound, "f32", strict=True, what=f"noalloc vs oracle, call {call}")
        if call == 0:
            assert _noalloc_call("q1g128", oc, os_, on, ok_, ox, oy, ydt) == bq.BQ_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import torch
    n, k = 128, 256 * 1024   # prepared-activation scratch alone exceeds the fixed array
    assert bq.bq_gemv_workspace_bytes("q1g128", n, k, 4) > bq.BQ_NOALLOC_SCRATCH_BYTES
    c = torch.zeros(n * k // 8, dtype=torch.uint8, device="cuda")
    s = torch.zeros(n * k // 128, dtype=torch.int16, device="cuda")
    x = torch.zeros((4, k), dtype=torch.bfloat16, device="cuda")
    y = torch.full((4, n), 5.0, dtype=torch.float32, device="cuda")
    assert _noalloc_call("q1g128", c, s, n, k, x, y, bq.BQ_F32) == bq.BQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(y == 5.0)
