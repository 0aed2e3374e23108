"""The affine 1-bit variant (w = s b + z per group, MLX-style) on the GPU:
packing bit-exact against the oracle, the decode GEMV within
2e-3 sum_k (|s| + |z|) |x_k| of the FP64 oracle, the embedding lookup
bit-exact, and the calls that do not take the format."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, to_dev, x_to_dev

pytestmark = pytest.mark.gpu


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def host_affine(n, k, seed):
    return oracle.pack_affine(synth.weights_normal(synth.rng(seed), n, k))


@pytest.mark.parametrize("n,k", [(1, 128), (37, 1024), (256, 4096), (129, 2176)])
def test_affine_pack_bit_exact(n, k):
    import torch
    g = synth.rng(700 + n)
    w = synth.weights_normal(g, n, k)
    w[0, :5] = [0.0, -0.0, 1e-30, -1e-30, 0.5]      # zeros, tiny values, a spread
    codes_ref, params_ref = oracle.pack_affine(w)
    c, p = bq.bq_pack_a1g128(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), codes_ref)
    assert np.array_equal(p.cpu().numpy().view(np.uint16), params_ref)
    # given (scale, bias) pairs, including exact half-step ties
    pin = params_ref.copy()
    pin[0::2] = 0x3C00                              # s = 1
    pin[1::2] = 0xB800                              # z = -0.5
    wt = np.tile(np.array([0.0, 0.5, -0.5, 1e-3], dtype=np.float32), (n, k // 4))  # 0.0 is a tie
    codes_ref2, params_ref2 = oracle.pack_affine(wt, params_in=pin)
    c2, p2 = bq.bq_pack_a1g128(torch.from_numpy(wt).cuda(), params_in=torch.from_numpy(pin.view(np.int16)).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(c2.cpu().numpy(), codes_ref2)
    assert np.array_equal(p2.cpu().numpy().view(np.uint16), params_ref2)


def test_affine_pack_errors():
    import torch
    w = torch.zeros((2, 128), device="cuda")
    w[1, 3] = float("nan")
    with pytest.raises(bq.BQError) as e:
        bq.bq_pack_a1g128(w)
    assert e.value.status == bq.BQ_ERR_NONFINITE
    w = torch.zeros((1, 128), device="cuda")
    w[0, 0] = 70000.0                                # max - min overflows FP16
    with pytest.raises(bq.BQError) as e:
        bq.bq_pack_a1g128(w)
    assert e.value.status == bq.BQ_ERR_SCALE_RANGE


@pytest.mark.parametrize("n,k,batch", [(256, 1024, 1), (300, 2048, 2), (129, 4096, 3), (1000, 1024, 5),
                                       (64, 4096, 8), (64, 12288, 2), (4096, 4096, 1)])
def test_affine_gemv(n, k, batch):
    import torch
    codes, params = host_affine(n, k, 710 + n + batch)
    x = synth.x_bf16(synth.rng(711 + k), batch, k)
    yref, bound = oracle.matmul_affine(codes, params, n, k, x)
    c, p, xd = to_dev(codes), to_dev(params.astype(np.int16)), x_to_dev(x)
    for ydt, name in ((bq.BQ_F32, "f32"), (bq.BQ_BF16, "bf16")):
        y = bq.bq_gemv("a1g128", c, p, n, k, xd, y_dtype=ydt)
        torch.cuda.synchronize()
        assert bq.bq_check() == bq.BQ_OK
        check_close(y, yref, bound, name, strict=True, what=f"affine {n}x{k} b{batch} {name}")


@pytest.mark.parametrize("shape", [(151936, 4096), (24576, 4096), (4096, 12288)])
def test_affine_gemv_full_size_sampled(shape):
    import torch
    n, k = shape
    gen = synth.device_generator(synth.SEED_BASE + 720)
    codes, params = bq.bq_pack_a1g128(synth.device_weights_normal(gen, n, k))
    x = synth.device_x_bf16(gen, 1, k)
    y = bq.bq_gemv("a1g128", codes, params, n, k, x, y_dtype=bq.BQ_F32)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    rows = np.unique(np.concatenate([[0, n - 1], synth.rng(721).integers(0, n, 48)]))
    sel = torch.from_numpy(rows).cuda()
    c = codes.view(n, k // 8)[sel].cpu().numpy().reshape(-1)
    p = params.view(n, k // 128 * 2)[sel].cpu().numpy().view(np.uint16).reshape(-1)
    yref, bound = oracle.matmul_affine(c, p, rows.size, k, _bits(x))
    check_close(y[:, sel], yref, bound, "f32", strict=True, what=f"affine {n}x{k} sampled")


def test_affine_embed_rows():
    import torch
    n, k = 200, 1024
    codes, params = host_affine(n, k, 730)
    ids = np.array([0, 199, 7, 7, 100], dtype=np.int32)
    out = bq.bq_embed_rows("a1g128", to_dev(codes), to_dev(params.astype(np.int16)), n, k,
                           torch.from_numpy(ids).cuda())
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    assert np.array_equal(_bits(out), oracle.embed_rows_affine(codes, params, n, k, ids))


def test_affine_unsupported_calls():
    import torch
    n, k = 64, 1024
    c = torch.zeros(n * k // 8, dtype=torch.uint8, device="cuda")
    p = torch.zeros(n * k // 64, dtype=torch.int16, device="cuda")
    x = torch.zeros((9, k), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemm("a1g128", c, p, n, k, x)
    assert e.value.status == bq.BQ_ERR_FORMAT
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv("a1g128", c, p, n, k, x)        # batch 9: only the row-owning path takes the format
    assert e.value.status == bq.BQ_ERR_SHAPE
    x1 = torch.zeros((1, 1152), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv("a1g128", torch.zeros(n * 1152 // 8, dtype=torch.uint8, device="cuda"),
                   torch.zeros(n * 1152 // 64, dtype=torch.int16, device="cuda"), n, 1152, x1)
    assert e.value.status == bq.BQ_ERR_SHAPE
    y = torch.zeros((1, n), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv_chain("a1g128", [dict(codes=c, scales=p, n=n, k=k, x=x[:1], y=y)])
    assert e.value.status == bq.BQ_ERR_FORMAT
