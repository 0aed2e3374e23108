"""The 27B-class decode pass at full size, as bench.py times it (q|k|v and
gate|up as one launch each, rows concatenated), all three formats at batch 1
and 16: sampled output rows against the oracle."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close

pytestmark = pytest.mark.gpu
G = 128


def pass_shapes():
    L, head = synth.CLASS27B_LAYER, synth.CLASS27B_LM_HEAD
    return {"qkv": (L["q"][0] + L["k"][0] + L["v"][0], L["q"][1]), "o": L["o"],
            "gate_up": (L["gate"][0] + L["up"][0], L["gate"][1]), "down": L["down"], "lm_head": head}


@pytest.mark.parametrize("fmt", ["q1g128", "t2g128", "t5p8"])
@pytest.mark.parametrize("batch", [1, 16])
@pytest.mark.parametrize("name", list(pass_shapes()))
def test_class27b_pass_sampled(fmt, batch, name):
    import torch
    n, k = pass_shapes()[name]
    gen = synth.device_generator(synth.SEED_BASE + 300 + list(pass_shapes()).index(name))
    if fmt == "q1g128":
        w = synth.device_weights_normal(gen, n, k)
        codes, scales = bq.bq_pack(fmt, w)
    else:
        t = synth.device_trits(gen, n, k)
        s = synth.device_scales_uniform(gen, n, k // G)
        w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(G, dim=1)
        del t
        codes, scales = bq.bq_pack(fmt, w, scales_in=s)
    del w
    x = synth.device_x_bf16(gen, batch, k)
    y = bq.bq_gemv(fmt, codes, scales, n, k, x)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    rows = np.unique(np.concatenate([[0, 1, 15, 16, 127, 128, n // 2, n - 2, n - 1],
                                     synth.rng(301).integers(0, n, 90)]))
    ridx = torch.from_numpy(rows).to(codes.device)
    rb = bq.bq_codes_bytes(fmt, 1, k)
    c_rows = codes.view(n, rb)[ridx].cpu().numpy().reshape(-1)
    s_rows = scales.view(n, k // G)[ridx].cpu().numpy().view(np.uint16).reshape(-1)
    x_bits = x.view(torch.int16).cpu().numpy().view(np.uint16)
    yref, bound = oracle.matmul(fmt, c_rows, s_rows, rows.size, k, x_bits)
    check_close(y[:, ridx], yref, bound, "bf16", strict=True, what=f"27b {name} {fmt} b{batch}")
