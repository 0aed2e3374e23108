"""Prefill GEMM on the GPU against the FP64 oracle at the stated tolerance."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, to_dev, x_to_dev, y_to_f64
from test_gpu_gemv import host_weights

pytestmark = pytest.mark.gpu
G = 128


def run_gemm(fmt, codes, scales, n, k, x_bits):
    import torch
    y = bq.bq_gemm(fmt, to_dev(codes), to_dev(scales.astype(np.int16)), n, k, x_to_dev(x_bits))
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    return y


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("n,k,t", [(256, 1024, 1), (256, 1024, 8), (300, 1152, 17), (512, 2048, 64),
                                   (129, 4096, 200), (1024, 1024, 512), (384, 640, 33)])
def test_gemm_shapes(fmt, n, k, t):
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 70 + n + t)
    x = synth.x_bf16(synth.rng(synth.SEED_BASE + 71 + t), t, k)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    check_close(run_gemm(fmt, codes, scales, n, k, x), yref, bound, "bf16", strict=True,
                what=f"gemm {fmt} {n}x{k} T{t}")


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("shape", synth.PREFILL_SHAPES)
@pytest.mark.parametrize("t", [1, 8, 64, 512, 4096])
def test_gemm_prefill_config_sampled(fmt, shape, t):
    """W 17408 x 5120 and 5120 x 17408 at full size; sampled output rows."""
    import torch
    n, k = shape
    gen = synth.device_generator(synth.SEED_BASE + 80 + t)
    if fmt == "q1g128":
        codes, scales = bq.bq_pack(fmt, synth.device_weights_normal(gen, n, k))
    else:
        tr = synth.device_trits(gen, n, k)
        s = synth.device_scales_uniform(gen, n, k // G)
        w = tr.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(G, dim=1)
        codes, scales = bq.bq_pack(fmt, w, scales_in=s)
        del w
    x = synth.device_x_bf16(gen, t, k)
    y = bq.bq_gemm(fmt, codes, scales, n, k, x)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, n - 1],
                                     synth.rng(81).integers(0, n, 26)]))
    ridx = torch.from_numpy(rows).to(codes.device)
    rb = bq.bq_codes_bytes(fmt, 1, k)
    c_rows = codes.view(n, rb)[ridx].cpu().numpy().reshape(-1)
    s_rows = scales.view(n, k // G)[ridx].cpu().numpy().view(np.uint16).reshape(-1)
    tok = np.unique(np.concatenate([[0, t - 1], synth.rng(82).integers(0, t, min(t, 64))]))
    x_bits = x[torch.from_numpy(tok).to(x.device)].view(torch.int16).cpu().numpy().view(np.uint16)
    yref, bound = oracle.matmul(fmt, c_rows, s_rows, rows.size, k, x_bits)
    yg = y[torch.from_numpy(tok).to(x.device)][:, ridx]
    check_close(yg, yref, bound, "bf16", strict=True, what=f"prefill {fmt} {n}x{k} T{t}")


def test_gemm_t1_matches_gemv():
    import torch
    n, k = 512, 2048
    codes, scales = host_weights("q1g128", n, k, synth.SEED_BASE + 90)
    x = synth.x_bf16(synth.rng(91), 1, k)
    c, s, xd = to_dev(codes), to_dev(scales.astype(np.int16)), x_to_dev(x)
    y1 = bq.bq_gemm("q1g128", c, s, n, k, xd)
    y2 = bq.bq_gemv("q1g128", c, s, n, k, xd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def _edge_tokens(g, t, k):
    """T tokens of BF16 activations at the edges of the per-token FP16
    pre-scale: an all-zero token, magnitudes spread over 1e-30 .. 1e30 with
    zeros, one large value with the rest at and below 2^-31 of it (rounded or
    flushed by the pre-scale), a token whose largest magnitude is ~1e-36 (the
    pre-scale exponent past 126), BF16 subnormals only, and N(0,1) tokens."""
    x = np.empty((t, k), dtype=np.float32)
    for i in range(t):
        kind = i % 7
        sign = g.choice([-1.0, 1.0], size=k)
        if kind == 0:
            x[i] = 0.0
        elif kind == 1:
            x[i] = sign * 10.0 ** g.uniform(-30, 30, size=k)
            x[i, ::5] = 0.0
        elif kind == 2:
            x[i] = sign * 2.0 ** (100 - g.uniform(20, 60, size=k))
            x[i, g.integers(0, k)] = 2.0 ** 100
        elif kind == 3:
            x[i] = sign * 1e-36 * g.uniform(0.0, 1.0, size=k)
        elif kind == 4:
            x[i] = sign * 2.0 ** -133 * g.integers(0, 128, size=k)
        else:
            x[i] = g.standard_normal(k)
    return synth.float32_to_bf16_bits(x)


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("n,k,batch", [(300, 1152, 9), (257, 2176, 16), (200, 1152, 5), (129, 3200, 8)])
def test_gemm_path_activation_edges_f32(fmt, n, k, batch):
    """The tcgen05 GEMM (bq_gemv routes K % 1024 != 0 to it with T = batch) with
    F32 output on edge-case activations: the per-token
    FP16 pre-scale must keep every output within 2e-3 sum|s x| (plus the F32
    rounding of y)."""
    import torch
    assert bq.bq_gemv_launches(fmt, n, k, batch) in (2, 3)  # activation prep + GEMM (+ split-K reduce)
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 95 + n)
    x = _edge_tokens(synth.rng(96 + batch), batch, k)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    y = bq.bq_gemv(fmt, to_dev(codes), to_dev(scales.astype(np.int16)), n, k, x_to_dev(x), y_dtype=bq.BQ_F32)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    check_close(y, yref, bound, "f32", strict=False, what=f"gemm edges {fmt} {n}x{k} T{batch}")
    assert np.all(y_to_f64(y)[0] == 0.0)  # the all-zero token


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("t", [5, 17, 64])
def test_gemm_activation_edges_bf16(fmt, t):
    """bq_gemm (BF16 output) on the same edge-case tokens; outputs whose exact
    value is a BF16 subnormal are compared against the oracle rounded to BF16."""
    import torch
    n, k = 256, 2048
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 97)
    x = _edge_tokens(synth.rng(98 + t), t, k)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    y = run_gemm(fmt, codes, scales, n, k, x)
    yv = y_to_f64(y)
    # the BF16 output grid near zero is 2^-133: allow half of it on top of the stated bound
    err = np.abs(yv - yref)
    allow = 2e-3 * bound + 2.0 ** -8 * (np.abs(yref) + 2e-3 * bound) + 2.0 ** -134
    assert np.all(err <= allow), float((err / allow).max())
    assert np.all(yv[0] == 0.0)
