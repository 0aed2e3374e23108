"""The wide-batch decode GEMV (batch 5..16 for binary and 2-bit ternary, 9..16
for 5 trits per byte: FP16 effective weights s * q in the MMA fragments, x
pre-scaled per batch row) on the GPU against the FP64 oracle at the stated
tolerance."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, to_dev, x_to_dev
from test_gpu_gemv import host_weights

pytestmark = pytest.mark.gpu
FMTS = ["q1g128", "t2g128"]


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


# Shapes on the wide path, with ragged row counts, several K stages and the
# largest K each batch allows: element by element against the oracle.
WIDE_CASES = [(b, n, k) for b in (5, 6, 8, 9, 12, 16) for n, k in ((33, 1024), (300, 2048), (1000, 4096))] + \
             [(b, n, k) for b in (5, 8) for n, k in ((129, 8192), (300, 9216))] + \
             [(b, n, k) for b in (9, 16) for n, k in ((16385, 4096), (1001, 5120))]


# 5 trits per byte: batch 9..16 only (batch <= 8 stays on the row-owning
# kernel); ragged rows, one to six K stages, the 208-byte groups read as pairs
# of 16-bit halves.
T5_WIDE_CASES = [(b, n, k) for b in (9, 12, 16) for n, k in ((33, 1024), (300, 2048), (1000, 4096))] + \
                [(9, 16385, 4096), (16, 16385, 4096), (9, 1001, 5120), (16, 1001, 5120), (10, 777, 3072),
                 (13, 2047, 6144), (16, 65, 1024)]


@pytest.mark.parametrize("fmt,batch,n,k", [(f,) + c for f in FMTS for c in WIDE_CASES] +
                         [("t5p8",) + c for c in T5_WIDE_CASES])
def test_wide_shapes(fmt, batch, n, k):
    import torch
    assert bq.bq_gemv_workspace_bytes(fmt, n, k, batch) == 0 and bq.bq_gemv_launches(fmt, n, k, batch) == 1
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 800 + n + k + batch)
    x = synth.x_bf16(synth.rng(801 + batch + k), batch, k)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    c, s, xd = to_dev(codes), to_dev(scales.astype(np.int16)), x_to_dev(x)
    for ydt, name in ((bq.BQ_F32, "f32"), (bq.BQ_BF16, "bf16")):
        y = bq.bq_gemv(fmt, c, s, n, k, xd, y_dtype=ydt)
        torch.cuda.synchronize()
        assert bq.bq_check() == bq.BQ_OK
        check_close(y, yref, bound, name, strict=True, what=f"wide {fmt} {n}x{k} b{batch} {name}")


@pytest.mark.parametrize("fmt", FMTS + ["t5p8"])
def test_wide_activation_edges(fmt):
    """Per-row pre-scale at the edges: an all-zero row, magnitudes over
    1e-30 .. 1e30, a row with one huge value and the rest at and below 2^-31 of
    it, a row whose largest |x| is ~1e-36, BF16 subnormals, N(0,1) rows."""
    import torch
    n, k, batch = 16390, 4096, 12
    assert bq.bq_gemv_launches(fmt, n, k, batch) == 1 and bq.bq_gemv_workspace_bytes(fmt, n, k, batch) == 0
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 810)
    g = synth.rng(811)
    xf = np.empty((batch, k), dtype=np.float32)
    for i in range(batch):
        kind, sign = i % 6, g.choice([-1.0, 1.0], size=k)
        if kind == 0:
            xf[i] = 0.0
        elif kind == 1:
            xf[i] = sign * 10.0 ** g.uniform(-30, 30, size=k)
        elif kind == 2:
            xf[i] = sign * 2.0 ** (90 - g.uniform(20, 60, size=k))
            xf[i, g.integers(0, k)] = 2.0 ** 90
        elif kind == 3:
            xf[i] = sign * 1e-36 * g.uniform(0.0, 1.0, size=k)
        elif kind == 4:
            xf[i] = sign * 2.0 ** -133 * g.integers(0, 128, size=k)
        else:
            xf[i] = g.standard_normal(k)
    x = synth.float32_to_bf16_bits(xf)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    y = bq.bq_gemv(fmt, to_dev(codes), to_dev(scales.astype(np.int16)), n, k, x_to_dev(x), y_dtype=bq.BQ_F32)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    check_close(y, yref, bound, "f32", strict=False, what=f"wide edges {fmt}")
    assert np.all(y[0].cpu().numpy() == 0.0)


@pytest.mark.parametrize("fmt,batch", [(f, b) for f in FMTS for b in (8, 16)] + [("t5p8", 16)])
@pytest.mark.parametrize("shape", [(6144, 4096), (24576, 4096), (151936, 4096), (34816, 5120), (248320, 5120),
                                   (4096, 12288)])
def test_wide_config_shapes_sampled(fmt, shape, batch):
    """The Qwen3-8B and 27B-class decode shapes at batch 8 and 16 (those the wide
    kernel takes), sampled rows against the oracle."""
    import torch
    n, k = shape
    if bq.bq_gemv_launches(fmt, n, k, batch) != 1 or bq.bq_gemv_workspace_bytes(fmt, n, k, batch) != 0:
        pytest.skip("shape not on the wide path at this batch")
    gen = synth.device_generator(synth.SEED_BASE + 820 + batch)
    if fmt == "q1g128":
        codes, scales = bq.bq_pack(fmt, synth.device_weights_normal(gen, n, k))
    else:
        t = synth.device_trits(gen, n, k)
        s = synth.device_scales_uniform(gen, n, k // 128)
        w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(128, dim=1)
        codes, scales = bq.bq_pack(fmt, w, scales_in=s)
        del w, t
    x = synth.device_x_bf16(gen, batch, k)
    y = bq.bq_gemv(fmt, codes, scales, n, k, x)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    rows = np.unique(np.concatenate([[0, n - 1], synth.rng(821).integers(0, n, 40)]))
    sel = torch.from_numpy(rows).cuda()
    rb = bq.bq_codes_bytes(fmt, 1, k)
    c = codes.view(n, rb)[sel].cpu().numpy().reshape(-1)
    s = scales.view(n, k // 128)[sel].cpu().numpy().view(np.uint16).reshape(-1)
    yref, bound = oracle.matmul(fmt, c, s, rows.size, k, _bits(x))
    check_close(y[:, sel], yref, bound, "bf16", strict=True, what=f"wide {fmt} {n}x{k} b{batch}")


@pytest.mark.parametrize("fmt,tokens", [("q1g128", (5, 9, 16)), ("t5p8", (9, 16))])
def test_wide_gemm_tokens_match_gemv(fmt, tokens):
    """bq_gemm with the token counts the wide kernel takes runs the same kernel
    as bq_gemv: identical bits."""
    import torch
    n, k = 16390, 4096
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 830)
    c, s = to_dev(codes), to_dev(scales.astype(np.int16))
    for t in tokens:
        x = x_to_dev(synth.x_bf16(synth.rng(831 + t), t, k))
        assert bq.bq_gemm_launches(fmt, n, k, t) == 1
        y1 = bq.bq_gemm(fmt, c, s, n, k, x)
        y2 = bq.bq_gemv(fmt, c, s, n, k, x)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)
