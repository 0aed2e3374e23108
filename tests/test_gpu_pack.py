"""Packers on the GPU against the oracle: codes and scales must be bit-exact."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import cuda, to_dev

pytestmark = pytest.mark.gpu
FMTS = ["q1g128", "t2g128", "t5p8"]


def gpu_pack(fmt, w_np, scales_in=None):
    import torch
    w = to_dev(w_np.astype(np.float32))
    sin = None if scales_in is None else to_dev(scales_in.astype(np.int16).reshape(-1))
    codes, scales = bq.bq_pack(fmt, w, sin)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n,k", [(1, 128), (3, 1152), (257, 1024), (64, 4096)])
def test_pack_random_normal_bit_exact(fmt, n, k):
    g = synth.rng(synth.SEED_BASE + 100 + n)
    w = synth.weights_normal(g, n, k)
    c_ref, s_ref = oracle.pack(fmt, w)
    c, s = gpu_pack(fmt, w)
    assert np.array_equal(s, s_ref)
    assert np.array_equal(c, c_ref)


@pytest.mark.parametrize("fmt", ["t2g128", "t5p8"])
def test_pack_given_scales_bit_exact(fmt):
    g = synth.rng(synth.SEED_BASE + 2)
    n, k = 129, 2048
    t = synth.trits(g, n, k)
    s = synth.scales_uniform(g, n, k // 128)
    w = t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), 128, axis=1)
    c_ref, s_ref = oracle.pack(fmt, w, scales_in=s)
    c, sg = gpu_pack(fmt, w, scales_in=s)
    assert np.array_equal(sg, s_ref) and np.array_equal(c, c_ref)
    assert np.array_equal(oracle.unpack(fmt, c, n, k), t)


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_edge_values_bit_exact(fmt):
    k = 128 * 6
    w = np.zeros((8, k), dtype=np.float32)
    w[0] = 0.0                                   # all zero: scale 0
    w[1] = -0.0
    w[2, ::2] = 1e-30; w[2, 1::2] = -1e-30       # mean underflows FP16
    w[3] = np.float32(6e-8)                      # FP16 subnormal mean
    w[4] = 65504.0                               # largest FP16 mean
    w[5] = np.linspace(-1, 1, k, dtype=np.float32)
    # ties at s/2: group mean 0.5 -> threshold 0.25 exactly
    grp = np.array([0.25, -0.25, 0.75, -0.75] * 32, dtype=np.float32)
    w[6] = np.tile(grp, k // 128)
    w[7] = np.tile(np.array([1.0] + [0.0] * 127, dtype=np.float32), k // 128)
    c_ref, s_ref = oracle.pack(fmt, w)
    c, sg = gpu_pack(fmt, w)
    assert np.array_equal(sg, s_ref) and np.array_equal(c, c_ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_errors_match_oracle(fmt):
    import torch
    k = 256
    for bad, expect in [(np.nan, bq.BQ_ERR_NONFINITE), (np.inf, bq.BQ_ERR_NONFINITE),
                        (70000.0, bq.BQ_ERR_SCALE_RANGE)]:
        w = np.full((4, k), 0.01, dtype=np.float32)
        if expect == bq.BQ_ERR_SCALE_RANGE:
            w[2, 128:] = bad
        else:
            w[2, 130] = bad
            w[3, 5] = bad
        st_ref = oracle.pack_status(fmt, w)[0]
        assert st_ref == expect
        with pytest.raises(bq.BQError) as ei:
            gpu_pack(fmt, w)
        assert ei.value.status == st_ref
    # a later valid call is not affected by the earlier error
    w = np.full((2, k), 0.01, dtype=np.float32)
    c, s = gpu_pack(fmt, w)
    assert np.array_equal(c, oracle.pack(fmt, w)[0])
    # negative given scale
    neg = np.full((2, 2), 0xBC00, dtype=np.uint16)
    with pytest.raises(bq.BQError) as ei:
        gpu_pack(fmt, w, scales_in=neg)
    assert ei.value.status == bq.BQ_ERR_SCALE_RANGE == oracle.pack_status(fmt, w, neg)[0]
    assert bq.bq_check() == bq.BQ_OK


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_full_size_lm_head_sampled_rows(fmt):
    """Qwen3-8B LM head 151936 x 4096 packed on the GPU; sampled rows bit-exact."""
    import torch
    n, k = synth.QWEN3_8B_LM_HEAD
    gen = synth.device_generator(synth.SEED_BASE + 1)
    w = synth.device_weights_normal(gen, n, k)
    codes, scales = bq.bq_pack(fmt, w)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, 1, n - 1, n // 2],
                                     synth.rng(5).integers(0, n, 60)]))
    rb = bq.bq_codes_bytes(fmt, 1, k)
    G = k // 128
    w_rows = w[torch.from_numpy(rows).to(w.device)].cpu().numpy()
    c_ref, s_ref = oracle.pack(fmt, w_rows)
    c_all = codes.view(n, rb)[torch.from_numpy(rows).to(w.device)].cpu().numpy().reshape(-1)
    s_all = scales.view(n, G)[torch.from_numpy(rows).to(w.device)].cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(s_all, s_ref) and np.array_equal(c_all, c_ref)
