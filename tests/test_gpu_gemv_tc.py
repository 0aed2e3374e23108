"""The tensor-core decode GEMVs (binary, 2-bit and 5-trit ternary, batch 1..8,
K % 1024 == 0) against the oracle: the row-owning kernel (no workspace) and
the split-K kernel it falls back to when the activation operand does not fit
in shared memory; ragged row counts, every chunk size of the row-owning
kernel, every batch size, activations whose magnitudes span the BF16 range,
and the check that shapes take the path they should."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, y_to_f64
from test_gpu_gemv import host_weights, run_gemv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128"])
def test_path_workspace(fmt):
    # row-owning kernel: no workspace
    assert bq.bq_gemv_workspace_bytes(fmt, 4096, 4096, 1) == 0
    assert bq.bq_gemv_workspace_bytes(fmt, 151936, 4096, 4) == 0
    # batch 4 at K = 17408: the activation operand exceeds shared memory -> split-K (workspace)
    assert bq.bq_gemv_workspace_bytes(fmt, 4096, 17408, 4) > 0
    # tcgen05 GEMM with T = batch: workspace for the FP16 activations
    assert bq.bq_gemv_workspace_bytes(fmt, 4096, 1152, 1) >= 1152 * 2   # K % 1024 != 0
    assert bq.bq_gemv_workspace_bytes(fmt, 4096, 4096, 8) == 0               # batch 5..8 while x fits
    assert bq.bq_gemv_workspace_bytes(fmt, 4096, 4096, 9) == 0               # wide-batch kernel
    assert bq.bq_gemv_workspace_bytes(fmt, 4096, 12288, 16) >= 16 * 12288 * 2  # its FP16 x exceeds shared memory
    assert bq.bq_gemv_workspace_bytes("t5p8", 4096, 4096, 1) == 0       # row-owning kernel
    assert bq.bq_gemv_workspace_bytes("t5p8", 4096, 17408, 4) >= 4 * 17408 * 2   # GEMM


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("n,k", [(777, 4096), (1, 1024), (128, 2048), (129, 3072), (5000, 1024), (96, 12288),
                                 (12000, 2048), (20000, 1024), (96, 17408)])
def test_tc_parity(fmt, batch, n, k):
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 200 + n + batch)
    x = synth.x_bf16(synth.rng(n + 3 * batch + k), batch, k)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    for ydt, name in ((bq.BQ_BF16, "bf16"), (bq.BQ_F32, "f32")):
        check_close(run_gemv(fmt, codes, scales, n, k, x, ydt), yref, bound, name, strict=True,
                    what=f"tc {fmt} {n}x{k} b{batch} {name}")


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
def test_tc_activation_range(fmt):
    """Groups whose activations are all tiny (BF16 subnormals), all huge, mixed
    within a group, or all zero."""
    n, k = 200, 4096
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 210)
    g = synth.rng(211)
    xf = g.standard_normal((2, k)).astype(np.float32)
    xf[0, 0:128] *= np.float32(1e-39)       # subnormal BF16 values
    xf[0, 128:256] *= np.float32(1e30)
    xf[0, 256:384] = 0.0
    mag = 10.0 ** g.uniform(-35, 35, size=128)
    xf[0, 384:512] = (np.sign(xf[0, 384:512]) * mag).astype(np.float32)
    xf[1, :] *= np.float32(3e-36)
    x = synth.float32_to_bf16_bits(xf)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    check_close(run_gemv(fmt, codes, scales, n, k, x, bq.BQ_F32), yref, bound, "f32", strict=True,
                what=f"range {fmt}")


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128"])
def test_tc_repeat_and_workspace_reuse(fmt):
    """Back-to-back calls with one workspace (split-K counters are reset by the
    call itself) give identical bits."""
    import torch
    from gpu_util import to_dev, x_to_dev
    n, k = 1024, 4096
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 220)
    x = synth.x_bf16(synth.rng(221), 3, k)
    c, s, xd = to_dev(codes), to_dev(scales.astype(np.int16)), x_to_dev(x)
    ws = torch.empty(bq.bq_gemv_workspace_bytes(fmt, n, k, 3), dtype=torch.uint8, device="cuda")
    ys = [bq.bq_gemv(fmt, c, s, n, k, xd, workspace=ws) for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    check_close(ys[0], yref, bound, "bf16", strict=True, what="reuse")
