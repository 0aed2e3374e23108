"""Benchmark of the weight-streaming g128 GEMV on B200.

Default workload (one step = one decode weight pass, batch 1): the Qwen3-8B
shapes -- 36 layers x (q 4096x4096, k 1024x4096, v 1024x4096, o 4096x4096,
gate 12288x4096, up 12288x4096, down 4096x12288) + LM head 151936x4096 -- every
layer with its own binary g128 weights (codes+scales 1.06 GB per pass, larger
than the 126 MB L2, so no flush is needed between steps).  Weights are packed
on the GPU from N(0, 0.02) floats; x ~ N(0,1) BF16.

Prints ONE JSON line (rank 0).  ``value`` = effective weight GB/s (codes +
scales bytes streamed per step / device time per step, summed over ranks);
``e2e`` = the same through the public API with the activations copied from
pinned host memory and every output copied back inside the timed region.
``--impl reference`` times the CPU oracle (the plain FP64 definition) on a
bounded sample of the same workload.

Launch: python bench.py [--gpus N --steps K --warmup W]; N > 1 under torchrun,
one independent replica per GPU (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FMT_NAMES = {"q1g128": 1, "t2g128": 2, "t5p8": 3, "a1g128": 4}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--fmt", choices=list(FMT_NAMES), default="q1g128")
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--model", choices=["qwen3-8b", "27b"], default="qwen3-8b",
                   help="layer shapes: Qwen3-8B (36 blocks, head 151936x4096) or the 27B class "
                        "(64 blocks, head 248320x5120)")
    p.add_argument("--layers", type=int, default=None, help="blocks per pass (default: the model's)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-gemm", action="store_true", help="skip the prefill GEMM legs")
    p.add_argument("--no-legs", action="store_true", help="skip the secondary configurations (the other formats, "
                   "batches and the 27B class)")
    p.add_argument("--leg-steps", type=int, default=10, help="timed steps of each secondary configuration")
    p.add_argument("--mode", choices=["calls", "chain"], default="calls",
                   help="one bq_gemv per product (calls) or one bq_gemv_chain per layer (chain)")
    p.add_argument("--gemm-only", action="store_true",
                   help="run only the prefill GEMM leg (a diagnostic line, e.g. for a profiler)")
    p.add_argument("--case", choices=["gemv", "gemm", "kv4"], default=None,
                   help="profiler case: each launch once to warm up, then once after an L2 flush, and exit "
                        "(gemv: --fmt, --batch, --shapes; gemm: --fmt, --shapes, --tokens; kv4: --batch, --ctx)")
    p.add_argument("--tokens", type=int, default=4096, help="tokens T for --case gemm")
    p.add_argument("--shapes", default="6144x4096,4096x4096,24576x4096,4096x12288,151936x4096",
                   help="NxK list for --case gemv (default: one Qwen3-8B layer's launches and the LM head)")
    p.add_argument("--ctx", type=int, default=65536, help="context tokens for --case kv4")
    return p.parse_args()


def run_case(args):
    """One launch per shape after a warm-up launch and a 256 MB L2 flush: the
    small, self-ending workloads profiler captures are taken on."""
    import math
    import torch
    import synth
    import ternary_g128_weight_b200 as bq
    dev = torch.device("cuda", 0)
    gen = synth.device_generator(synth.SEED_BASE + 9, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = []
    if args.case == "gemv":
        f = FMT_NAMES[args.fmt]
        for sh in args.shapes.split(","):
            n, k = (int(v) for v in sh.split("x"))
            codes, scales = make_weights(f, n, k, gen, dev, False)
            x = synth.device_x_bf16(gen, args.batch, k, device=dev)
            y = torch.empty((args.batch, n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(max(bq.bq_gemv_workspace_bytes(f, n, k, args.batch), 256), dtype=torch.uint8, device=dev)
            calls.append(lambda f=f, c=codes, s=scales, n=n, k=k, x=x, y=y, ws=ws:
                         bq.bq_gemv(f, c, s, n, k, x, y=y, workspace=ws))
    elif args.case == "gemm":
        f = FMT_NAMES[args.fmt]
        for sh in args.shapes.split(","):
            n, k = (int(v) for v in sh.split("x"))
            codes, scales = make_weights(f, n, k, gen, dev, False)
            x = synth.device_x_bf16(gen, args.tokens, k, device=dev)
            y = torch.empty((args.tokens, n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(max(bq.bq_gemm_workspace_bytes(f, n, k, args.tokens), 256), dtype=torch.uint8,
                             device=dev)
            calls.append(lambda f=f, c=codes, s=scales, n=n, k=k, x=x, y=y, ws=ws:
                         bq.bq_gemm(f, c, s, n, k, x, y=y, workspace=ws))
    else:
        A = synth.QWEN3_8B_ATTN
        B, ctx, hq, hkv, d = args.batch, args.ctx, A["hq"], A["hkv"], A["d"]
        cache = synth.device_kv4_cache(gen, B, hkv, ctx, d, device=dev) + \
            synth.device_kv4_cache(gen, B, hkv, ctx, d, device=dev)
        q = synth.device_x_bf16(gen, B * hq, d, device=dev).view(B, hq, d)
        lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        o = torch.empty((B, hq, d), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(bq.bq_kv4_attention_workspace_bytes(B, hq, hkv, d, ctx, ctx), 256),
                         dtype=torch.uint8, device=dev)
        calls.append(lambda: bq.bq_kv4_attention_decode(q, *cache, lens, ctx, 1.0 / math.sqrt(d), out=o,
                                                        workspace=ws))
    for c in calls:
        c()
    torch.cuda.synchronize()
    for c in calls:
        flush.fill_(1)
        c()
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    print(json.dumps({"case": args.case, "launches": len(calls)}), flush=True)
    return 0


def model_shapes(model):
    import synth
    if model == "27b":
        return synth.CLASS27B_LAYER, synth.CLASS27B_LM_HEAD, synth.CLASS27B_BLOCKS
    return synth.QWEN3_8B_LAYER, synth.QWEN3_8B_LM_HEAD, synth.QWEN3_8B_BLOCKS


def step_shapes(model, layers):
    """One decode weight pass: per layer q|k|v (one launch, rows concatenated:
    the three share x), o, gate|up (one launch), down; then the LM head."""
    L, head, _ = model_shapes(model)
    qkv = (L["q"][0] + L["k"][0] + L["v"][0], L["q"][1])
    gate_up = (L["gate"][0] + L["up"][0], L["gate"][1])
    shapes = []
    for layer in range(layers):
        shapes += [(f"L{layer}.qkv",) + qkv, (f"L{layer}.o",) + L["o"],
                   (f"L{layer}.gate_up",) + gate_up, (f"L{layer}.down",) + L["down"]]
    shapes.append(("lm_head",) + head)
    return shapes


def workload_name(model, fmt, batch, layers):
    L, head, _ = model_shapes(model)
    qkv = L["q"][0] + L["k"][0] + L["v"][0]
    return (f"{model}-shapes {fmt} GEMV batch {batch}: {layers} x (q|k|v {qkv}x{L['q'][1]} "
            f"[q {L['q'][0]}, k {L['k'][0]}, v {L['v'][0]} rows], o {L['o'][0]}x{L['o'][1]}, "
            f"gate|up {2 * L['gate'][0]}x{L['gate'][1]} [2 x {L['gate'][0]} rows], "
            f"down {L['down'][0]}x{L['down'][1]}) + LM head {head[0]}x{head[1]}, distinct weights per layer, "
            f"one CUDA graph per step")


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        loaded = [v for v in sm if smax and v > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


KERNEL_SOURCES = ("bq_gemv_rows.cu", "bq_gemv_tc.cu", "bq_gemm_tc.cu", "bq_ptx.cuh", "bq_api.cu")


def kernel_source_hash():
    """Identifies the kernel sources a recorded profiler capture belongs to
    (their code: comments and whitespace do not count)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "ternary_g128_weight_b200", "csrc", name)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(model, fmt, batch, layers):
    """DRAM bytes per step from profiles/ncu_traffic.json when it was taken on
    this workload with the current kernel sources, else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rows = json.load(fh)
    for tr in rows if isinstance(rows, list) else [rows]:
        if (tr.get("model"), tr.get("fmt"), tr.get("batch"), tr.get("layers"), tr.get("kernel_src")) == \
                (model, fmt, batch, layers, kernel_source_hash()):
            return tr.get("dram_bytes_per_step")
    return None


def measured_tensor_peak():
    """Dense 16-bit tensor peak (TFLOP/s) for a kernel timed alone: the measured
    burst cuBLAS BF16 figure (FP16 runs at the same nominal rate)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ---------------------------------------------------------------- prefill GEMM
GEMM_SHAPES = [(17408, 5120), (5120, 17408)]


def gemm_leg(fmt, dev, reps):
    """Prefill GEMM Y = X W^T on the pages' two prefill shapes at T = 1, 8, 64,
    512 and 4096 tokens; each launch timed alone with CUDA events, L2 flushed by
    a 256 MB write before every timed launch.  Reported as TFLOP/s against the
    dense 16-bit tensor peak and, for the weight-bound small T, as weight GB/s
    against HBM."""
    import torch
    import synth
    import ternary_g128_weight_b200 as bq
    peak, src = measured_tensor_peak()
    hbm, _ = measured_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = []
    for (n, k) in GEMM_SHAPES:
        gen = synth.device_generator(synth.SEED_BASE + 4, device=dev)
        codes, scales = make_weights(fmt, n, k, gen, dev, False)
        wbytes = codes.numel() + 2 * scales.numel()
        for T in synth.PREFILL_TOKENS:
            x = synth.device_x_bf16(gen, T, k, device=dev)
            y = torch.empty((T, n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(max(bq.bq_gemm_workspace_bytes(fmt, n, k, T), 256), dtype=torch.uint8, device=dev)
            for _ in range(3):
                bq.bq_gemm(fmt, codes, scales, n, k, x, y=y, workspace=ws)
            torch.cuda.synchronize()
            times = []
            for _ in range(reps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                bq.bq_gemm(fmt, codes, scales, n, k, x, y=y, workspace=ws)
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
            assert bq.bq_check() == bq.BQ_OK
            ms = statistics.median(times)
            tf = 2.0 * T * n * k / (ms / 1000.0) / 1e12
            gbs = wbytes / (ms / 1000.0) / 1e9
            out.append({"shape": f"{n}x{k}", "tokens": T, "us": round(ms * 1000, 1),
                        "tflops": round(tf, 2), "frac": round(tf / peak, 4),
                        "weight_GB_s": round(gbs, 1), "hbm_frac": round(gbs / hbm, 4),
                        "launches": bq.bq_gemm_launches(fmt, n, k, T)})
            del x, y, ws
        del codes, scales
    return {"bound": "tensor (T >= 64), hbm (T <= 8)", "peak": peak, "unit": "TFLOP/s",
            "peak_source": f"{src} (MEASURED_PEAKS.json bf16_tflops, burst; FP16 operands at the same rate)",
            "kernel": "xprep_f16_kernel + gemm_tc_kernel (tcgen05 kind::f16, TMEM accumulators); T <= 4: the GEMV",
            "dtype": "f16 operands (exact s*q and pre-scaled x), f32 accumulate", "cases": out}


def embed_leg(dev, reps):
    """The 1-bit embedding lookup (bq_embed_rows) on the Qwen3-8B table
    (151936 x 4096, binary g128) for 1, 16 and 4096 token ids: 20 lookups of
    fresh random ids per CUDA graph, bytes = table rows read + BF16 rows written."""
    import torch
    import synth
    import ternary_g128_weight_b200 as bq
    hbm, _ = measured_peaks()
    n, k = synth.QWEN3_8B_LM_HEAD
    gen = synth.device_generator(synth.SEED_BASE + 8, device=dev)
    codes, scales = make_weights("q1g128", n, k, gen, dev, True)
    out = []
    for count in (1, 16, 4096):
        ids = [torch.randint(0, n, (count,), generator=gen, device=dev, dtype=torch.int32) for _ in range(20)]
        o = torch.empty((count, k), dtype=torch.bfloat16, device=dev)
        for i in ids[:3]:
            bq.bq_embed_rows("q1g128", codes, scales, n, k, i, out=o)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in ids:
                bq.bq_embed_rows("q1g128", codes, scales, n, k, i, out=o)
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / len(ids))
        assert bq.bq_check() == bq.BQ_OK
        ms = statistics.median(times)
        byts = count * (bq.bq_codes_bytes("q1g128", 1, k) + bq.bq_scales_bytes(1, k) + 2 * k + 4)
        out.append({"tokens": count, "us": round(1000.0 * ms, 2), "bytes": byts,
                    "GB_s": round(byts / (ms / 1000.0) / 1e9, 1), "frac": round(byts / (ms / 1000.0) / 1e9 / hbm, 4)})
        del g
    return {"workload": "qwen3-8b embedding table 151936x4096 q1g128, random token ids, one launch per lookup",
            "kernel": "embed_rows_kernel", "bound": "hbm", "peak": hbm, "cases": out}


def attention_leg(dev, reps):
    """4-bit KV-cache decode attention of Qwen3-8B (32 query / 8 KV heads, head
    dimension 128): a step is one decode token through 36 layers, each layer
    appending the token's K and V to its own cache (bq_kv4_append) and attending
    over the whole context (bq_kv4_attention_decode), in one CUDA graph.  The
    36 caches together exceed L2.  Reported as cache GB/s against HBM, plus one
    attention launch timed alone (L2 flushed before it)."""
    import math
    import torch
    import synth
    import ternary_g128_weight_b200 as bq
    A = synth.QWEN3_8B_ATTN
    hq, hkv, d, layers = A["hq"], A["hkv"], A["d"], synth.QWEN3_8B_BLOCKS
    hbm, _ = measured_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = []
    for B, ctx in ((1, 65536), (16, 4096)):
        gen = synth.device_generator(synth.SEED_BASE + 7, device=dev)
        caches = [synth.device_kv4_cache(gen, B, hkv, ctx, d, device=dev) +
                  synth.device_kv4_cache(gen, B, hkv, ctx, d, device=dev) for _ in range(layers)]
        q = synth.device_x_bf16(gen, B * hq, d, device=dev).view(B, hq, d)
        kn = synth.device_x_bf16(gen, B * hkv, d, device=dev).view(B, hkv, d)
        vn = synth.device_x_bf16(gen, B * hkv, d, device=dev).view(B, hkv, d)
        lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        pos = lens - 1
        o = torch.empty((B, hq, d), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(bq.bq_kv4_attention_workspace_bytes(B, hq, hkv, d, ctx, ctx), 256), dtype=torch.uint8,
                         device=dev)
        scale = 1.0 / math.sqrt(d)

        def layer(c):
            bq.bq_kv4_append(kn, vn, pos, c[0], c[1], c[2], c[3])
            bq.bq_kv4_attention_decode(q, c[0], c[1], c[2], c[3], lens, ctx, scale, out=o, workspace=ws)

        for c in caches:
            layer(c)
        torch.cuda.synchronize()
        st = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for c in caches:
                layer(c)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            # (replay() launches on the current stream: time it there)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        # one attention launch alone, L2 flushed, events on its stream
        a_times = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            bq.bq_kv4_attention_decode(q, *caches[0], lens, ctx, scale, out=o, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            a_times.append(e0.elapsed_time(e1))
        assert bq.bq_check() == bq.BQ_OK
        cache_bytes = B * hkv * ctx * (bq.bq_kv4_codes_bytes(1, d) + bq.bq_kv4_params_bytes(1, d)) * 2
        algo = cache_bytes + B * hq * d * 2 * 2 + B * 4  # + q in, out, lens
        a_ms = statistics.median(a_times)
        out.append({"workload": f"qwen3-8b decode attention, 4-bit g128 KV cache, batch {B} x {ctx} tokens, "
                                f"{layers} layers (append + attention per layer)",
                    "batch": B, "context": ctx, "ms_per_step": round(ms, 4),
                    "value": round(layers * algo / (ms / 1000.0) / 1e9, 1), "unit": "GB/s",
                    "frac": round(layers * algo / (ms / 1000.0) / 1e9 / hbm, 4),
                    "us_per_layer": round(1000.0 * ms / layers, 2),
                    "tokens_per_s": round(1000.0 / ms, 1),
                    "attention_launch": {"us": round(1000.0 * a_ms, 2), "bytes": algo,
                                         "GB_s": round(algo / (a_ms / 1000.0) / 1e9, 1),
                                         "frac": round(algo / (a_ms / 1000.0) / 1e9 / hbm, 4)},
                    "launches_per_step": 2 * layers})
        del caches, g
        torch.cuda.empty_cache()
    return {"bound": "hbm", "peak": hbm, "kernel": "attn_kernel (bq_kv4_attention_decode) + append_kernel",
            "dtype": "f16 operands (q pre-scaled, codes c - 8, P s_V 2^sigma), f32 accumulate", "cases": out}


# ------------------------------------------------------------------ reference
def run_reference(args):
    """The CPU oracle as it stands, on a bounded sample of the workload."""
    if world_info()[1] != 0:
        return 0
    import numpy as np
    import oracle
    import synth
    fmt = args.fmt
    n, k = synth.QWEN3_8B_LAYER["q"]
    g = synth.rng(synth.SEED_BASE + 1)
    codes = synth.code_bytes_uniform(g, oracle.codes_bytes(fmt, n, k)) if fmt == "q1g128" else None
    if codes is None:
        t = synth.trits(g, n, k)
        s = synth.scales_uniform(g, n, k // 128)
        w = t.astype(np.float32) * np.repeat(synth.fp16_bits_to_float32(s), 128, axis=1)
        codes, scales = oracle.pack(fmt, w, scales_in=s)
    else:
        scales = synth.scales_uniform(g, n, k // 128).reshape(-1)
    x = synth.x_bf16(g, args.batch, k)
    wbytes = codes.nbytes + scales.nbytes
    for _ in range(args.warmup):
        oracle.matmul(fmt, codes, scales, n, k, x)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.matmul(fmt, codes, scales, n, k, x)
        times.append(time.perf_counter() - t0)
    ms = 1000.0 * sum(times) / len(times)
    value = wbytes / (ms / 1000.0) / 1e9
    sample = f"one q matrix 4096x4096 ({fmt}, batch {args.batch}) per step"
    line = {
        "impl": "reference", "metric": "effective weight GB/s (g128 GEMV weight stream)",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(args.model, fmt, args.batch, args.layers), "fmt": fmt,
                   "batch": args.batch, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.max_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(fmt, mats, batch):
    """Oracle on a bounded sample (the LM head plus the first layer), host cores."""
    import numpy as np
    import torch
    import oracle
    sample = [mats[-1]] + mats[:4]  # LM head + the first layer's four launches
    host = []
    for m in sample:
        host.append((m["n"], m["k"], m["codes"].cpu().numpy(), m["scales"].cpu().numpy().view(np.uint16),
                     m["x"].view(torch.int16).cpu().numpy().view(np.uint16)))
    # repeat the sample until about 10 s of host work is done (bounded: 200 passes)
    total_bytes, passes, t0 = 0, 0, time.perf_counter()
    while passes < 200 and (passes == 0 or time.perf_counter() - t0 < 10.0):
        for (n, k, c, s, x) in host:
            oracle.matmul(fmt, c, s, n, k, x)
            total_bytes += c.nbytes + s.nbytes
        passes += 1
    dt = time.perf_counter() - t0
    # the same oracle on one core: the first layer's o matrix, about 3 s
    n1, k1, c1, s1, x1 = host[2]
    one_bytes, one_passes, t1 = 0, 0, time.perf_counter()
    while one_passes < 200 and (one_passes == 0 or time.perf_counter() - t1 < 3.0):
        oracle.matmul(fmt, c1, s1, n1, k1, x1, nthreads=1)
        one_bytes += c1.nbytes + s1.nbytes
        one_passes += 1
    dt1 = time.perf_counter() - t1
    return {"value": round(total_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.max_threads(),
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"LM head + one layer's q|k|v, o, gate|up, down ({fmt}, batch {batch}) x {passes} passes, "
                      f"{total_bytes / 1e6:.1f} MB of weights, {dt:.1f} s",
            "single_core": {"value": round(one_bytes / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "sample": f"o {n1}x{k1} x {one_passes} passes, {dt1:.1f} s"}}


def cpu_model():
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------ ranks (host side)
def world_info():
    """(WORLD_SIZE, RANK, LOCAL_RANK) as torchrun sets them; one process alone is rank 0 of 1."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, dist, device):
    """Element-wise maximum of each rank's timings (every rank calls it, in
    the same order); without a process group the values themselves."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_value(bytes_per_rank_step, world, ms_per_step):
    """Whole-job GB/s: the bytes all ranks processed in one step over the
    slowest rank's step time (replicas: each rank runs the full step)."""
    return bytes_per_rank_step * world / (ms_per_step / 1000.0) / 1e9


# --------------------------------------------------------------- the passes
def make_weights(fmt, n, k, gen, dev, direct_codes):
    """Weights of one matrix: binary by packing N(0, 0.02) floats (or, for the
    27B class, uniform code bytes with uniform FP16 scales, no float pass);
    ternary by packing trits (P(-1) = P(+1) = 0.35) times uniform FP16 scales
    with the scales given."""
    import torch
    import synth
    import ternary_g128_weight_b200 as bq
    if fmt == "q1g128" and direct_codes:
        return (synth.device_code_bytes(gen, bq.bq_codes_bytes(fmt, n, k), device=dev),
                synth.device_scales_uniform(gen, n, k // 128, device=dev).view(-1))
    if fmt in ("q1g128", "a1g128"):
        return bq.bq_pack(fmt, synth.device_weights_normal(gen, n, k, device=dev))
    t = synth.device_trits(gen, n, k, device=dev)
    s = synth.device_scales_uniform(gen, n, k // 128, device=dev)
    w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(128, dim=1)
    del t
    return bq.bq_pack(fmt, w, scales_in=s)


class Pass:
    """One decode weight pass on the device: per layer q|k|v, o, gate|up, down,
    then the LM head, each with its own weights; every activation and output
    in one contiguous buffer (one copy per step for the end-to-end timing).
    mode "calls": one bq_gemv per product, each a programmatic dependent of the
    previous one; mode "chain": one bq_gemv_chain per layer (q|k|v, o,
    gate|up with the SwiGLU epilogue, down on that output), then the head."""

    def __init__(self, model, fmt, batch, layers, seed, dev, mode="calls"):
        import torch
        import synth
        import ternary_g128_weight_b200 as bq
        self.model, self.fmt, self.batch, self.layers, self.mode = model, fmt, batch, layers, mode
        self.f = FMT_NAMES[fmt]
        gen = synth.device_generator(seed, device=dev)
        shapes = step_shapes(model, layers)
        direct = model == "27b"

        def offsets(sizes):
            offs, tot = [], 0
            for sz in sizes:
                offs.append(tot)
                tot += (sz + 127) // 128 * 128
            return offs, tot
        L = model_shapes(model)[0]
        inter = L["gate"][0]
        x_sizes, y_sizes = [], []
        for name, n, k in shapes:
            x_sizes.append(batch * k)
            y_sizes.append(batch * (inter if (mode == "chain" and name.endswith("gate_up")) else n))
        x_offs, x_tot = offsets(x_sizes)
        y_offs, y_tot = offsets(y_sizes)
        self.X = synth.device_x_bf16(gen, 1, x_tot, device=dev).view(-1)
        self.Y = torch.zeros(y_tot, dtype=torch.bfloat16, device=dev)
        self.mats = []
        for i, (name, n, k) in enumerate(shapes):
            codes, scales = make_weights(fmt, n, k, gen, dev, direct)
            yn = y_sizes[i] // batch
            self.mats.append({"name": name, "n": n, "k": k, "codes": codes, "scales": scales,
                              "x": self.X[x_offs[i]:x_offs[i] + batch * k].view(batch, k),
                              "y": self.Y[y_offs[i]:y_offs[i] + batch * yn].view(batch, yn)})
        torch.cuda.synchronize()
        self.weight_bytes = sum(m["codes"].numel() + 2 * m["scales"].numel() for m in self.mats)
        self.algo_bytes = self.weight_bytes + sum(2 * m["k"] * batch + 2 * m["y"].shape[1] * batch
                                                  for m in self.mats)
        ws_need = max(bq.bq_gemv_workspace_bytes(self.f, m["n"], m["k"], batch) for m in self.mats)
        self.workspace = torch.empty(max(ws_need, 256), dtype=torch.uint8, device=dev)
        self.chains = []
        if mode == "chain":
            for l in range(layers):
                q, o, gu, dn = self.mats[4 * l:4 * l + 4]
                steps = [dict(codes=q["codes"], scales=q["scales"], n=q["n"], k=q["k"], x=q["x"], y=q["y"]),
                         dict(codes=o["codes"], scales=o["scales"], n=o["n"], k=o["k"], x=o["x"], y=o["y"]),
                         dict(codes=gu["codes"], scales=gu["scales"], n=gu["n"], k=gu["k"], x=gu["x"], y=gu["y"],
                              swiglu=True),
                         dict(codes=dn["codes"], scales=dn["scales"], n=dn["n"], k=dn["k"], x=gu["y"], y=dn["y"])]
                self.chains.append((steps, torch.zeros(bq.bq_gemv_chain_workspace_bytes(), dtype=torch.uint8,
                                                       device=dev)))
        self.launches = (sum(bq.bq_gemv_launches(self.f, m["n"], m["k"], batch) for m in self.mats)
                         if mode == "calls" else layers + bq.bq_gemv_launches(self.f, *shapes[-1][1:], batch))
        self.graph = None

    def step(self):
        import ternary_g128_weight_b200 as bq
        if self.mode == "chain":
            for steps, ws in self.chains:
                bq.bq_gemv_chain(self.f, steps, workspace=ws)
            m = self.mats[-1]
            bq.bq_gemv(self.f, m["codes"], m["scales"], m["n"], m["k"], m["x"], y=m["y"], workspace=self.workspace)
            return
        for m in self.mats:
            bq.bq_gemv(self.f, m["codes"], m["scales"], m["n"], m["k"], m["x"], y=m["y"], workspace=self.workspace)

    def capture(self):
        """Warm up eagerly (lazy initialisation), then capture one step in a CUDA graph."""
        import torch
        import ternary_g128_weight_b200 as bq
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step()
            self.step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        assert bq.bq_check() == bq.BQ_OK
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()

    def time_steps(self, steps, warmup, barrier):
        """Device time of `steps` graph replays (ms per step), CUDA events on the
        replaying stream, barrier + synchronize on both sides."""
        import torch
        import ternary_g128_weight_b200 as bq
        for _ in range(warmup):
            self.graph.replay()
        barrier()
        stream = torch.cuda.current_stream()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            self.graph.replay()
        t1.record(stream)
        barrier()
        assert bq.bq_check() == bq.BQ_OK
        return t0.elapsed_time(t1) / steps

    def time_e2e(self, steps, barrier):
        """The same step through the public API with the step's activations
        copied from pinned host memory and every output copied back, inside the
        timed region."""
        import torch
        x_host = torch.empty_like(self.X, device="cpu").pin_memory()
        x_host.copy_(self.X)
        y_host = torch.empty_like(self.Y, device="cpu").pin_memory()
        stream = torch.cuda.current_stream()

        def e2e_step():
            self.X.copy_(x_host, non_blocking=True)
            self.graph.replay()
            y_host.copy_(self.Y, non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        barrier()
        return {"ms_per_step": e0.elapsed_time(e1) / steps, "h2d": self.X.numel() * 2, "d2h": self.Y.numel() * 2}

    def free(self):
        import torch
        self.graph = None
        self.mats.clear()
        self.chains.clear()
        self.X = self.Y = self.workspace = None
        torch.cuda.empty_cache()


def leg(model, fmt, batch, mode, dev, steps, warmup, peak, seed):
    """One secondary configuration: a whole pass, its GB/s, roofline fraction,
    tokens/s-equivalent and end-to-end figure."""
    layers = model_shapes(model)[2]
    ps = Pass(model, fmt, batch, layers, seed, dev, mode)
    ps.capture()
    import torch
    ms = ps.time_steps(steps, warmup, torch.cuda.synchronize)
    e2e = ps.time_e2e(max(2, steps // 2), torch.cuda.synchronize)
    out = {"workload": workload_name(model, fmt, batch, layers) + ("" if mode == "calls" else ", one chain per layer"),
           "model": model, "fmt": fmt, "batch": batch, "mode": mode, "steps": steps,
           "ms_per_step": round(ms, 4), "value": round(ps.weight_bytes / (ms / 1000.0) / 1e9, 2), "unit": "GB/s",
           "roofline_frac": round(ps.algo_bytes / (ms / 1000.0) / 1e9 / peak, 4),
           "tokens_per_s_equiv": round(1000.0 / ms, 2),
           "e2e": {"value": round(ps.weight_bytes / (e2e["ms_per_step"] / 1000.0) / 1e9, 2), "unit": "GB/s",
                   "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
           "launches_per_step": ps.launches}
    ps.free()
    return out


# The secondary configurations: the Qwen3-8B shapes in both ternary formats
# at batch 1 and 16 and in binary at batch 8, the 27B class in all three
# formats at batch 1 and 16, the binary Qwen3-8B pass as per-layer chains, and
# the affine 1-bit variant (scale and bias per group) at batch 1.
LEGS = [("qwen3-8b", "t2g128", 1, "calls"), ("qwen3-8b", "t5p8", 1, "calls"), ("qwen3-8b", "q1g128", 8, "calls"),
        ("qwen3-8b", "t2g128", 16, "calls"), ("qwen3-8b", "t5p8", 16, "calls"),
        ("27b", "q1g128", 1, "calls"), ("27b", "t2g128", 1, "calls"), ("27b", "t5p8", 1, "calls"),
        ("27b", "q1g128", 16, "calls"), ("27b", "t2g128", 16, "calls"), ("27b", "t5p8", 16, "calls"),
        ("qwen3-8b", "q1g128", 1, "chain"), ("qwen3-8b", "a1g128", 1, "calls")]


# ----------------------------------------------------------------------- ours
def main():
    args = parse()
    if args.layers is None:
        args.layers = model_shapes(args.model)[2]
    if args.impl == "reference":
        return run_reference(args)
    if args.case:
        return run_case(args)

    import torch
    import ternary_g128_weight_b200 as bq

    world, rank, local = world_info()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    fmt, batch = args.fmt, args.batch
    f = FMT_NAMES[fmt]
    if args.gemm_only:
        if rank == 0:
            print(json.dumps({"metric": "prefill GEMM TFLOP/s", "fmt": fmt,
                              "prefill_gemm": gemm_leg(fmt, dev, max(args.steps, 1))}), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    ps = Pass(args.model, fmt, batch, args.layers, synth_seed(rank), dev, args.mode)
    mats = ps.mats
    ps.capture()
    calls_per_step = len(mats)
    # the arithmetic of the path bq_gemv takes for this format and batch
    int8_path = batch <= 8 and all(bq.bq_gemv_workspace_bytes(f, m["n"], m["k"], batch) == 0 for m in mats)
    path_dtype = "s8xu8->s32 (warp MMA), f32 recombine" if int8_path else "f16 (tcgen05) -> f32"
    path_kernel = (("gemv_rows_kernel (row-owning tensor-core GEMV)" if args.mode == "calls" else
                    "gemv_chain_kernel (persistent layer chain) + gemv_rows_kernel (head)") if int8_path
                   else "xprep_f16_kernel + gemm_tc_kernel (tcgen05 GEMM with T = batch)")

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        ps.graph.replay()
    barrier()
    assert bq.bq_check() == bq.BQ_OK

    # ---- device-timed region
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    elapsed_ms = ps.time_steps(args.steps, 0, barrier) * args.steps
    clocks = sampler.stop()

    # ---- LM head alone (largest launch): per-launch time with events around it
    head = mats[-1]
    stream = torch.cuda.current_stream()
    hg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(hg):
        bq.bq_gemv(f, head["codes"], head["scales"], head["n"], head["k"], head["x"], y=head["y"],
                   workspace=ps.workspace)
    hg.replay()
    torch.cuda.synchronize()
    h_times = []
    for _ in range(max(3, args.steps)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ps.graph.replay()  # evicts the head's weights from L2 (1 GB streamed)
        e0.record(stream)
        hg.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        h_times.append(e0.elapsed_time(e1))
    head_bytes = head["codes"].numel() + 2 * head["scales"].numel() + 2 * head["k"] * batch + 2 * head["n"] * batch
    head_ms = statistics.median(h_times)

    # ---- end-to-end through the public API: pinned host inputs in, outputs out
    e2e = None if args.no_e2e else ps.time_e2e(args.steps, barrier)

    # ---- max over ranks
    ms_per_step, e2e_ms = max_over_ranks([elapsed_ms / args.steps, e2e["ms_per_step"] if e2e else 0.0], dist, dev)
    if e2e:
        e2e["ms_per_step"] = e2e_ms

    peak, peak_src = measured_peaks()
    weight_bytes, algo_bytes = ps.weight_bytes, ps.algo_bytes
    value = job_value(weight_bytes, world, ms_per_step)
    achieved = algo_bytes / (ms_per_step / 1000.0) / 1e9
    traffic = recorded_traffic(args.model, fmt, batch, args.layers)
    launches_per_step = ps.launches

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(fmt, mats, batch)
    del hg
    ps.free()
    legs, prefill = [], None
    if rank == 0 and not args.no_legs:
        for i, (model, lf, lb, mode) in enumerate(LEGS):
            legs.append(leg(model, lf, lb, mode, dev, args.leg_steps, 3, peak, synth_seed(rank) + 100 + i))
    if rank == 0 and not args.no_gemm:
        prefill = {lf: gemm_leg(lf, dev, 5) for lf in (["q1g128", "t2g128", "t5p8"] if not args.no_legs else [fmt])}
    attention = attention_leg(dev, 5) if rank == 0 and not args.no_legs else None
    embedding = embed_leg(dev, 5) if rank == 0 and not args.no_legs else None

    if rank == 0:
        line = {
            "metric": "effective weight GB/s (g128 GEMV weight stream)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": path_dtype, "data": "synthetic",
            "config": {"workload": workload_name(args.model, fmt, batch, args.layers)
                       + ("" if args.mode == "calls" else ", one chain per layer"),
                       "fmt": fmt, "batch": batch, "mode": args.mode,
                       "weight_bytes_per_step": weight_bytes, "gemv_calls_per_step": calls_per_step,
                       "l2": f"inputs larger than L2 ({weight_bytes / 1e9:.2f} GB of weights per step, L2 126 MB), no flush",
                       "parallelism": f"replicas x{world}"},
            "hbm_roofline_pct": round(100.0 * value / world / peak, 2),
            "tokens_per_s_equiv": round(1000.0 / ms_per_step, 2),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
                         "kernel": path_kernel + ", every launch of a step back to back",
                         "algorithmic_bytes_per_step": algo_bytes},
            "lm_head_launch": {"us": round(head_ms * 1000, 2), "bytes": head_bytes,
                               "GB_s": round(head_bytes / (head_ms / 1000.0) / 1e9, 2),
                               "frac": round(head_bytes / (head_ms / 1000.0) / 1e9 / peak, 4)},
            "clocks": clocks,
            "gpu_launches": launches_per_step * args.steps,
        }
        if e2e:
            line["e2e"] = {"value": round(job_value(weight_bytes, world, e2e["ms_per_step"]), 2),
                           "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                           "d2h_bytes_per_step": e2e["d2h"]}
        if cpu:
            line["cpu_baseline"] = cpu
        if legs:
            line["configs"] = legs
        if prefill:
            line["prefill_gemm"] = prefill
        if attention:
            line["kv4_attention"] = attention
        if embedding:
            line["embedding"] = embedding
        print(json.dumps(line), flush=True)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def synth_seed(rank):
    import synth
    return synth.SEED_BASE + 1 + 1000 * rank


if __name__ == "__main__":
    sys.exit(main())
