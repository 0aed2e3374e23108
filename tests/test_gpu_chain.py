"""The persistent layer chain (bq_gemv_chain) on the GPU against the FP64
oracle: plain steps element by element at the stated tolerance, the SwiGLU
step against the oracle's SwiGLU of the exact gate|up product (with the
allowance the product's tolerance implies), and a step whose x is an earlier
step's output against the oracle product of that very input."""
import numpy as np
import pytest

import oracle
import synth
import ternary_g128_weight_b200 as bq
from gpu_util import check_close, to_dev, x_to_dev, y_to_f64
from test_gpu_gemv import host_weights

pytestmark = pytest.mark.gpu
FMTS = ["q1g128", "t2g128", "t5p8"]


def _dev_weights(fmt, n, k, seed):
    codes, scales = host_weights(fmt, n, k, seed)
    return codes, scales, to_dev(codes), to_dev(scales.astype(np.int16))


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check_swiglu(act_bits, fmt, gu_codes, gu_scales, inter, k, x_bits, js, what):
    """act[b][j] for j in js against BF16(silu(g) u) of the exact products g, u:
    allowance 1.1 dg (|u| + du) + (|silu(g)| + 1.1 dg) du (|silu'| <= 1.1, and
    dg, du the products' tolerance 2e-3 sum|s x|) plus one BF16 ulp."""
    rows = np.concatenate([js, inter + js])
    h, bound = oracle.matmul_rows(fmt, gu_codes, gu_scales, 2 * inter, k, x_bits, rows)
    g, u = h[:, :js.size], h[:, js.size:]
    dg, du = 2e-3 * bound[:, :js.size], 2e-3 * bound[:, js.size:]
    silu = g / (1.0 + np.exp(-g))
    a = silu * u
    allow = 1.1 * dg * (np.abs(u) + du) + (np.abs(silu) + 1.1 * dg) * du
    allow = allow + 2.0 ** -8 * (np.abs(a) + allow) + 1e-30
    got = (act_bits[:, js].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(got - a)
    bad = ~(err <= allow)
    assert not bad.any(), f"{what}: {bad.sum()} act values out of the allowance; first {np.argwhere(bad)[0]}"


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("batch", [1, 2, 3, 8])
def test_chain_mlp_block_small(fmt, batch):
    """Three chained steps: y0 = W0 x0; act = SwiGLU(Wgu y0); y2 = Wd act."""
    import torch
    hidden, inter = 1024, 2048
    c0, s0, dc0, ds0 = _dev_weights(fmt, hidden, hidden, synth.SEED_BASE + 500 + batch)
    cg, sg, dcg, dsg = _dev_weights(fmt, 2 * inter, hidden, synth.SEED_BASE + 501 + batch)
    cd, sd, dcd, dsd = _dev_weights(fmt, hidden, inter, synth.SEED_BASE + 502 + batch)
    x0 = synth.x_bf16(synth.rng(503 + batch), batch, hidden)
    x0d = x_to_dev(x0)
    y0 = torch.empty((batch, hidden), dtype=torch.bfloat16, device="cuda")
    act = torch.empty((batch, inter), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((batch, hidden), dtype=torch.float32, device="cuda")
    steps = [dict(codes=dc0, scales=ds0, n=hidden, k=hidden, x=x0d, y=y0),
             dict(codes=dcg, scales=dsg, n=2 * inter, k=hidden, x=y0, y=act, swiglu=True),
             dict(codes=dcd, scales=dsd, n=hidden, k=inter, x=act, y=y2)]
    ws = bq.bq_gemv_chain(fmt, steps)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    assert int(ws.sum()) == 0  # counters left zero
    y0ref, b0 = oracle.matmul(fmt, c0, s0, hidden, hidden, x0)
    check_close(y0, y0ref, b0, "bf16", strict=True, what=f"{fmt} b{batch} y0")
    check_swiglu(_bits(act), fmt, cg, sg, inter, hidden, _bits(y0), np.arange(inter), f"{fmt} b{batch} act")
    y2ref, b2 = oracle.matmul(fmt, cd, sd, hidden, inter, _bits(act))
    check_close(y2, y2ref, b2, "f32", strict=True, what=f"{fmt} b{batch} down of act")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("ydt", [bq.BQ_BF16, bq.BQ_F32])
def test_chain_plain_steps_and_reuse(fmt, ydt):
    """Plain steps with their own inputs, every output against the oracle; a
    second call on the same workspace gives bit-identical outputs."""
    import torch
    batch = 2
    shapes = [(384, 1024), (1000, 2048), (129, 3072), (2048, 1024)]
    steps, refs = [], []
    tdt = torch.float32 if ydt == bq.BQ_F32 else torch.bfloat16
    for i, (n, k) in enumerate(shapes):
        c, s, dc, ds = _dev_weights(fmt, n, k, synth.SEED_BASE + 520 + i)
        x = synth.x_bf16(synth.rng(530 + i), batch, k)
        steps.append(dict(codes=dc, scales=ds, n=n, k=k, x=x_to_dev(x), y=torch.empty((batch, n), dtype=tdt,
                                                                                      device="cuda")))
        refs.append(oracle.matmul(fmt, c, s, n, k, x))
    ws = bq.bq_gemv_chain(fmt, steps)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    first = [st["y"].clone() for st in steps]
    for st, (yref, bound) in zip(steps, refs):
        check_close(st["y"], yref, bound, "f32" if ydt == bq.BQ_F32 else "bf16", strict=True,
                    what=f"chain {fmt} {st['n']}x{st['k']}")
    bq.bq_gemv_chain(fmt, steps, workspace=ws)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    assert int(ws.sum()) == 0
    for a, st in zip(first, steps):
        assert torch.equal(a, st["y"])


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("batch", [1, 2])
def test_chain_qwen3_8b_layer_sampled(fmt, batch):
    """One Qwen3-8B layer as one chain: q|k|v 6144x4096, o 4096x4096, gate|up
    24576x4096 with SwiGLU, down 4096x12288 on the SwiGLU output; sampled rows
    against the oracle."""
    import torch
    L = synth.QWEN3_8B_LAYER
    H, I = L["q"][1], L["gate"][0]
    qkv = L["q"][0] + L["k"][0] + L["v"][0]
    gen = synth.device_generator(synth.SEED_BASE + 540 + batch)

    def mk(n, k):
        if fmt == "q1g128":
            return bq.bq_pack(fmt, synth.device_weights_normal(gen, n, k))
        t = synth.device_trits(gen, n, k)
        s = synth.device_scales_uniform(gen, n, k // 128)
        w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(128, dim=1)
        return bq.bq_pack(fmt, w, scales_in=s)

    mats = [mk(qkv, H), mk(H, H), mk(2 * I, H), mk(H, I)]
    xs = [synth.device_x_bf16(gen, batch, H) for _ in range(3)]
    outs = [torch.empty((batch, qkv), dtype=torch.bfloat16, device="cuda"),
            torch.empty((batch, H), dtype=torch.bfloat16, device="cuda"),
            torch.empty((batch, I), dtype=torch.bfloat16, device="cuda"),
            torch.empty((batch, H), dtype=torch.bfloat16, device="cuda")]
    steps = [dict(codes=mats[0][0], scales=mats[0][1], n=qkv, k=H, x=xs[0], y=outs[0]),
             dict(codes=mats[1][0], scales=mats[1][1], n=H, k=H, x=xs[1], y=outs[1]),
             dict(codes=mats[2][0], scales=mats[2][1], n=2 * I, k=H, x=xs[2], y=outs[2], swiglu=True),
             dict(codes=mats[3][0], scales=mats[3][1], n=H, k=I, x=outs[2], y=outs[3])]
    bq.bq_gemv_chain(fmt, steps)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    g = synth.rng(541)

    def host(i, n, k):
        rb = bq.bq_codes_bytes(fmt, 1, k)
        return mats[i][0].cpu().numpy().reshape(n, rb), mats[i][1].cpu().numpy().view(np.uint16).reshape(n, k // 128)

    for i, (n, k, xb) in enumerate([(qkv, H, xs[0]), (H, H, xs[1]), (H, I, outs[2])]):
        idx = [0, 1, 3][i]
        rows = np.unique(np.concatenate([[0, n - 1], g.integers(0, n, 40)]))
        c, s = host(idx, n, k)
        yref, bound = oracle.matmul_rows(fmt, c[rows].reshape(-1), s[rows].reshape(-1), rows.size, k, _bits(xb),
                                         np.arange(rows.size))
        check_close(outs[idx][:, torch.from_numpy(rows).cuda()], yref, bound, "bf16", strict=True,
                    what=f"layer {fmt} b{batch} step {idx}")
    js = np.unique(np.concatenate([[0, I - 1], g.integers(0, I, 60)]))
    c, s = host(2, 2 * I, H)
    check_swiglu(_bits(outs[2]), fmt, c.reshape(-1), s.reshape(-1), I, H, _bits(xs[2]), js,
                 f"layer {fmt} b{batch} act")


def test_chain_operand_too_large_is_rejected():
    """At batch 8 the activation operand of K = 12288 (418 KB) exceeds shared
    memory: the chain returns BQ_ERR_SHAPE and launches nothing."""
    import torch
    n, k, batch = 64, 12288, 8
    c = torch.zeros(n * k // 8, dtype=torch.uint8, device="cuda")
    s = torch.zeros(n * k // 128, dtype=torch.int16, device="cuda")
    x = torch.zeros((batch, k), dtype=torch.bfloat16, device="cuda")
    y = torch.full((batch, n), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv_chain("q1g128", [dict(codes=c, scales=s, n=n, k=k, x=x, y=y)])
    assert e.value.status == bq.BQ_ERR_SHAPE
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)


def test_chain_timeout_free_and_errors():
    """Argument errors come back before anything is launched."""
    import torch
    c, s = torch.zeros(4096, dtype=torch.uint8, device="cuda"), torch.zeros(256, dtype=torch.int16, device="cuda")
    x = torch.zeros((1, 1024), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    ok = dict(codes=c, scales=s, n=32, k=1024, x=x, y=y)
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv_chain("q1g128", [dict(ok, k=1152)])
    assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv_chain("q1g128", [dict(ok, n=48, swiglu=True)])
    assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv_chain("q1g128", [ok] * 9)
    assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BQError) as e:
        bq.bq_gemv_chain("q1g128", [ok], workspace=torch.zeros(8, dtype=torch.uint8, device="cuda"))
    assert e.value.status == bq.BQ_ERR_WORKSPACE
