"""GEMV on the GPU against the FP64 oracle (element by element) at the stated
tolerance, on the pages' workloads: the tiny binary case, every Qwen3-8B layer
matrix, the LM head (sampled rows), ragged shapes and the degenerate cases."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, cuda, to_dev, x_to_dev, y_to_f64

pytestmark = pytest.mark.gpu
FMTS = ["q1g128", "t2g128", "t5p8"]
G = 128


def host_weights(fmt, n, k, seed):
    """Config recipe: binary = packed N(0, 0.02) floats; ternary = trits
    (0.35/0.30/0.35) with uniform FP16 scales, packed with given scales."""
    g = synth.rng(seed)
    if fmt == "q1g128":
        return oracle.pack(fmt, synth.weights_normal(g, n, k))
    t = synth.trits(g, n, k)
    s = synth.scales_uniform(g, n, k // G)
    w = t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), G, axis=1)
    return oracle.pack(fmt, w, scales_in=s)


def run_gemv(fmt, codes, scales, n, k, x_bits, y_dtype=bq.BQ_BF16):
    import torch
    c = to_dev(codes)
    s = to_dev(scales.astype(np.int16))
    x = x_to_dev(x_bits)
    y = bq.bq_gemv(fmt, c, s, n, k, x, y_dtype=y_dtype)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    return y


def test_tiny_binary_config():
    """W 256 x 1024, uniform sign bits, FP16 scales U[0.005, 0.05], x ~ N(0,1), batch 1."""
    n, k = 256, 1024
    g = synth.rng(synth.SEED_BASE + 0)
    codes = synth.code_bytes_uniform(g, oracle.codes_bytes("q1g128", n, k))
    scales = synth.scales_uniform(g, n, k // G).reshape(-1)
    x = synth.x_bf16(g, 1, k)
    yref, bound = oracle.matmul("q1g128", codes, scales, n, k, x)
    for ydt, name in ((bq.BQ_BF16, "bf16"), (bq.BQ_F32, "f32")):
        y = run_gemv("q1g128", codes, scales, n, k, x, ydt)
        check_close(y, yref, bound, name, strict=True, what=f"tiny {name}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n,k,batch", [(1, 128, 1), (3, 1152, 3), (33, 4096, 16), (257, 1024, 8),
                                       (1000, 2048, 1), (129, 12288, 2), (64, 640, 7), (300, 4096, 4)])
def test_ragged_shapes(fmt, n, k, batch):
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 10 + n + k + batch)
    x = synth.x_bf16(synth.rng(n * 7 + k), batch, k)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    for ydt, name in ((bq.BQ_BF16, "bf16"), (bq.BQ_F32, "f32")):
        y = run_gemv(fmt, codes, scales, n, k, x, ydt)
        check_close(y, yref, bound, name, strict=True, what=f"{fmt} {n}x{k} b{batch} {name}")


@pytest.mark.parametrize("fmt,batch", [("q1g128", 1), ("q1g128", 8), ("t2g128", 1), ("t2g128", 16),
                                       ("t5p8", 1), ("t5p8", 16)])
def test_qwen3_8b_layer_full(fmt, batch):
    """Every matrix of one Qwen3-8B layer, all outputs."""
    for i, (name, (n, k)) in enumerate(synth.QWEN3_8B_LAYER.items()):
        codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 20 + i)
        x = synth.x_bf16(synth.rng(synth.SEED_BASE + 40 + i), batch, k)
        yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
        y = run_gemv(fmt, codes, scales, n, k, x)
        check_close(y, yref, bound, "bf16", strict=True, what=f"{fmt} {name} b{batch}")


@pytest.mark.parametrize("fmt,batch", [("q1g128", 1), ("q1g128", 8), ("t2g128", 16), ("t5p8", 16)])
def test_qwen3_8b_lm_head_sampled(fmt, batch):
    """LM head 151936 x 4096 at full size; the oracle checks sampled rows."""
    import torch
    n, k = synth.QWEN3_8B_LM_HEAD
    gen = synth.device_generator(synth.SEED_BASE + 50)
    if fmt == "q1g128":
        w = synth.device_weights_normal(gen, n, k)
        codes, scales = bq.bq_pack(fmt, w)
    else:
        t = synth.device_trits(gen, n, k)
        s = synth.device_scales_uniform(gen, n, k // G)
        w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(G, dim=1)
        codes, scales = bq.bq_pack(fmt, w, scales_in=s)
    del w
    x = synth.device_x_bf16(gen, batch, k)
    y = bq.bq_gemv(fmt, codes, scales, n, k, x)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    rows = np.unique(np.concatenate([[0, 1, 2, 127, 128, n - 1, n - 2, n // 2],
                                     synth.rng(51).integers(0, n, 120)]))
    ridx = torch.from_numpy(rows).to(codes.device)
    rb = bq.bq_codes_bytes(fmt, 1, k)
    c_rows = codes.view(n, rb)[ridx].cpu().numpy().reshape(-1)
    s_rows = scales.view(n, k // G)[ridx].cpu().numpy().view(np.uint16).reshape(-1)
    x_bits = x.view(torch.int16).cpu().numpy().view(np.uint16)
    yref, bound = oracle.matmul(fmt, c_rows, s_rows, rows.size, k, x_bits)
    check_close(y[:, ridx], yref, bound, "bf16", strict=True, what=f"lm head {fmt} b{batch}")


@pytest.mark.parametrize("fmt", FMTS)
def test_all_ones_x_closed_form(fmt):
    """x = 1: y is a signed count times the scales; |y| can reach sum |s x|."""
    n, k = 64, 1024
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 60)
    x = np.full((1, k), 0x3F80, dtype=np.uint16)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    check_close(run_gemv(fmt, codes, scales, n, k, x, bq.BQ_F32), yref, bound, "f32", strict=True,
                what="ones f32")
    check_close(run_gemv(fmt, codes, scales, n, k, x), yref, bound, "bf16", strict=False, what="ones bf16")
    # all-plus binary row: the output equals the bound, the worst case for BF16 rounding
    if fmt == "q1g128":
        c = np.full_like(codes, 0xFF)
        yref, bound = oracle.matmul(fmt, c, scales, n, k, x)
        assert np.allclose(yref, bound)
        check_close(run_gemv(fmt, c, scales, n, k, x), yref, bound, "bf16", strict=False, what="all +")


@pytest.mark.parametrize("fmt", FMTS)
def test_small_integers_exact_in_f32(fmt):
    """Scales 1.0 and integer activations: every partial sum is an integer below
    2^24, so the F32 output must equal the oracle exactly."""
    n, k = 96, 2048
    g = synth.rng(synth.SEED_BASE + 61)
    if fmt == "q1g128":
        codes = synth.code_bytes_uniform(g, oracle.codes_bytes(fmt, n, k))
    else:
        t = synth.trits(g, n, k)
        codes, _ = oracle.pack(fmt, t.astype(np.float32), np.full((n, k // G), 0x3C00, np.uint16))
    scales = np.full(n * (k // G), 0x3C00, dtype=np.uint16)
    xi = g.integers(-16, 17, size=(3, k)).astype(np.float32)
    x = synth.float32_to_bf16_bits(xi)
    yref, _ = oracle.matmul(fmt, codes, scales, n, k, x)
    y = y_to_f64(run_gemv(fmt, codes, scales, n, k, x, bq.BQ_F32))
    assert np.array_equal(y, yref)


@pytest.mark.parametrize("fmt", FMTS)
def test_extreme_activation_magnitudes(fmt):
    """BF16 activations spanning 1e-30 .. 1e30 within one row (and zeros)."""
    n, k = 40, 1024
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 62)
    g = synth.rng(63)
    mag = 10.0 ** g.uniform(-30, 30, size=(2, k))
    xf = (g.choice([-1.0, 1.0], size=(2, k)) * mag).astype(np.float32)
    xf[0, ::7] = 0.0
    x = synth.float32_to_bf16_bits(xf)
    yref, bound = oracle.matmul(fmt, codes, scales, n, k, x)
    check_close(run_gemv(fmt, codes, scales, n, k, x, bq.BQ_F32), yref, bound, "f32", strict=False,
                what="extreme f32")


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_x_and_zero_scales(fmt):
    n, k = 17, 512
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 64)
    x0 = np.zeros((2, k), dtype=np.uint16)
    assert np.all(y_to_f64(run_gemv(fmt, codes, scales, n, k, x0, bq.BQ_F32)) == 0.0)
    x = synth.x_bf16(synth.rng(65), 2, k)
    z = np.zeros_like(scales)
    assert np.all(y_to_f64(run_gemv(fmt, codes, z, n, k, x, bq.BQ_F32)) == 0.0)


def test_empty_shapes():
    import torch
    dev = cuda()
    x = torch.zeros((1, 128), dtype=torch.bfloat16, device=dev)
    c = torch.zeros(16, dtype=torch.uint8, device=dev)
    s = torch.zeros(8, dtype=torch.int16, device=dev)
    y = bq.bq_gemv("q1g128", c, s, 0, 128, x)            # N = 0: nothing to do
    assert y.shape == (1, 0)
    y = torch.full((2, 5), 7.0, dtype=torch.float32, device=dev)
    xk0 = torch.zeros((2, 0), dtype=torch.bfloat16, device=dev)
    bq.bq_gemv("t2g128", c, s, 5, 0, xk0, y=y, y_dtype=bq.BQ_F32)  # K = 0: empty sums
    torch.cuda.synchronize()
    assert torch.all(y == 0)


@pytest.mark.parametrize("fmt", FMTS)
def test_deterministic_and_stream_ordered(fmt):
    import torch
    n, k = 4096, 4096
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 66)
    x = synth.x_bf16(synth.rng(67), 4, k)
    c, s, xd = to_dev(codes), to_dev(scales.astype(np.int16)), x_to_dev(x)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        y1 = bq.bq_gemv(fmt, c, s, n, k, xd, stream=st)
        y2 = bq.bq_gemv(fmt, c, s, n, k, xd, stream=st)
    st.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("fmt", ["t2g128", "t5p8"])
def test_invalid_codes_do_not_fault(fmt):
    import torch
    n, k = 64, 1024
    codes = np.full(oracle.codes_bytes(fmt, n, k), 0xFF, dtype=np.uint8)  # invalid everywhere
    scales = np.full(n * (k // G), 0x3C00, dtype=np.uint16)
    x = synth.x_bf16(synth.rng(68), 1, k)
    y = run_gemv(fmt, codes, scales, n, k, x, bq.BQ_F32)
    assert y.shape == (1, n)
    assert bq.bq_check() == bq.BQ_OK
