"""Embedding lookup on a low-bit table (bq_embed_rows) on the GPU, bit-exact
against the oracle's rows (dequantised s * q rounded once to BF16)."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import to_dev
from test_gpu_gemv import host_weights

pytestmark = pytest.mark.gpu
FMTS = ["q1g128", "t2g128", "t5p8"]


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n,k,count", [(300, 1024, 77), (1, 128, 5), (64, 4096, 64), (129, 640, 1)])
def test_embed_rows_small(fmt, n, k, count):
    import torch
    codes, scales = host_weights(fmt, n, k, synth.SEED_BASE + 600 + n + k)
    g = synth.rng(601 + count)
    ids = np.concatenate([[0, n - 1], g.integers(0, n, count)])[:count].astype(np.int32)
    ref = oracle.embed_rows(fmt, codes, scales, n, k, ids)
    out = bq.bq_embed_rows(fmt, to_dev(codes), to_dev(scales.astype(np.int16)), n, k,
                           torch.from_numpy(ids).cuda())
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    assert np.array_equal(_bits(out), ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_embed_rows_full_table_sampled(fmt):
    """The 151936 x 4096 table (the Qwen3-8B vocabulary), 64 rows looked up."""
    import torch
    n, k = synth.QWEN3_8B_LM_HEAD
    gen = synth.device_generator(synth.SEED_BASE + 610)
    if fmt == "q1g128":
        codes, scales = bq.bq_pack(fmt, synth.device_weights_normal(gen, n, k))
    else:
        t = synth.device_trits(gen, n, k)
        s = synth.device_scales_uniform(gen, n, k // 128)
        w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(128, dim=1)
        codes, scales = bq.bq_pack(fmt, w, scales_in=s)
        del w, t
    ids = np.concatenate([[0, n - 1, 7, 7], synth.rng(611).integers(0, n, 60)]).astype(np.int32)
    out = bq.bq_embed_rows(fmt, codes, scales, n, k, torch.from_numpy(ids).cuda())
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    rb = bq.bq_codes_bytes(fmt, 1, k)
    uniq, inv = np.unique(ids, return_inverse=True)
    sel = torch.from_numpy(uniq.astype(np.int64)).cuda()
    c = codes.view(n, rb)[sel].cpu().numpy().reshape(-1)
    s = scales.view(n, k // 128)[sel].cpu().numpy().view(np.uint16).reshape(-1)
    ref = oracle.embed_rows(fmt, c, s, uniq.size, k, inv.astype(np.int32))
    assert np.array_equal(_bits(out), ref)


def test_embed_rows_bad_id_gives_zero_row_and_status():
    import torch
    n, k = 40, 256
    codes, scales = host_weights("q1g128", n, k, synth.SEED_BASE + 620)
    ids = np.array([3, 40, 5, -1], dtype=np.int32)
    out = bq.bq_embed_rows("q1g128", to_dev(codes), to_dev(scales.astype(np.int16)), n, k,
                           torch.from_numpy(ids).cuda())
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_ERR_SHAPE
    assert bq.bq_check() == bq.BQ_OK          # the flag is cleared by the report
    o = _bits(out)
    ref = oracle.embed_rows("q1g128", codes, scales, n, k, ids[[0, 2]])
    assert np.array_equal(o[[0, 2]], ref)
    assert np.all(o[[1, 3]] == 0)


def test_embed_rows_empty():
    import torch
    c = torch.zeros(16, dtype=torch.uint8, device="cuda")
    s = torch.zeros(1, dtype=torch.int16, device="cuda")
    out = bq.bq_embed_rows("q1g128", c, s, 1, 128, torch.zeros(0, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert out.shape == (0, 128)
