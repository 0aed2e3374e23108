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

FMT_NAMES = {"q1g128": 1, "t2g128": 2, "t5p8": 3}


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
    p.add_argument("--no-gemm", action="store_true", help="skip the prefill GEMM leg")
    p.add_argument("--gemm-only", action="store_true",
                   help="run only the prefill GEMM leg (a diagnostic line, e.g. for a profiler)")
    return p.parse_args()


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
GEMM_TOKENS = 4096


def gemm_leg(fmt, dev, reps):
    """Prefill GEMM Y = X W^T at T = 4096 on the pages' two prefill shapes
    (tensor-bound); each launch timed alone with CUDA events, L2 flushed by a
    256 MB write before every timed launch."""
    import torch
    import synth
    import ternary_g128_weight_b200 as bq
    peak, src = measured_tensor_peak()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    out = []
    for (n, k) in GEMM_SHAPES:
        gen = synth.device_generator(synth.SEED_BASE + 4, device=dev)
        if fmt == "q1g128":
            codes, scales = bq.bq_pack(fmt, synth.device_weights_normal(gen, n, k, device=dev))
        else:
            t = synth.device_trits(gen, n, k, device=dev)
            s = synth.device_scales_uniform(gen, n, k // 128, device=dev)
            w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(128, dim=1)
            codes, scales = bq.bq_pack(fmt, w, scales_in=s)
            del w
        x = synth.device_x_bf16(gen, GEMM_TOKENS, k, device=dev)
        y = torch.empty((GEMM_TOKENS, n), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(bq.bq_gemm_workspace_bytes(fmt, n, k, GEMM_TOKENS), 256), dtype=torch.uint8, device=dev)
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
        tf = 2.0 * GEMM_TOKENS * n * k / (ms / 1000.0) / 1e12
        out.append({"shape": f"{n}x{k}", "tokens": GEMM_TOKENS, "us": round(ms * 1000, 1),
                    "tflops": round(tf, 1), "frac": round(tf / peak, 4),
                    "launches": bq.bq_gemm_launches(fmt, n, k, GEMM_TOKENS)})
        del codes, scales, x, y, ws
    return {"bound": "tensor", "peak": peak, "unit": "TFLOP/s",
            "peak_source": f"{src} (MEASURED_PEAKS.json bf16_tflops, burst; FP16 operands at the same rate)",
            "kernel": "xprep_f16_kernel + gemm_tc_kernel (tcgen05 kind::f16, TMEM accumulators)",
            "dtype": "f16 operands (exact s*q and pre-scaled x), f32 accumulate", "cases": out}


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
    return {"value": round(total_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"LM head + one layer's q|k|v, o, gate|up, down ({fmt}, batch {batch}) x {passes} passes, "
                      f"{total_bytes / 1e6:.1f} MB of weights, {dt:.1f} s"}


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


# ----------------------------------------------------------------------- ours
def main():
    args = parse()
    if args.layers is None:
        args.layers = model_shapes(args.model)[2]
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import synth
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
    gen = synth.device_generator(synth.SEED_BASE + 1 + 1000 * rank, device=dev)
    shapes = step_shapes(args.model, args.layers)

    # ---- activations and outputs: one contiguous buffer each (one copy per step for e2e)
    def offsets(sizes):
        offs, tot = [], 0
        for sz in sizes:
            offs.append(tot)
            tot += (sz + 127) // 128 * 128
        return offs, tot
    x_offs, x_tot = offsets([batch * k for _, _, k in shapes])
    y_offs, y_tot = offsets([batch * n for _, n, _ in shapes])
    X_all = synth.device_x_bf16(gen, 1, x_tot, device=dev).view(-1)
    Y_all = torch.zeros(y_tot, dtype=torch.bfloat16, device=dev)

    # ---- weights: distinct per launch, packed on the GPU
    mats = []
    for i, (name, n, k) in enumerate(shapes):
        if fmt == "q1g128":
            w = synth.device_weights_normal(gen, n, k, device=dev)
            codes, scales = bq.bq_pack(fmt, w)
        else:
            t = synth.device_trits(gen, n, k, device=dev)
            s = synth.device_scales_uniform(gen, n, k // 128, device=dev)
            w = t.to(torch.float32) * s.view(torch.float16).to(torch.float32).repeat_interleave(128, dim=1)
            codes, scales = bq.bq_pack(fmt, w, scales_in=s)
        del w
        mats.append({"name": name, "n": n, "k": k, "codes": codes, "scales": scales,
                     "x": X_all[x_offs[i]:x_offs[i] + batch * k].view(batch, k),
                     "y": Y_all[y_offs[i]:y_offs[i] + batch * n].view(batch, n)})
    torch.cuda.synchronize()
    ws_need = max(bq.bq_gemv_workspace_bytes(f, m["n"], m["k"], batch) for m in mats)
    workspace = torch.empty(max(ws_need, 256), dtype=torch.uint8, device=dev)
    weight_bytes = sum(m["codes"].numel() + 2 * m["scales"].numel() for m in mats)
    algo_bytes = weight_bytes + sum(2 * m["k"] * batch + 2 * m["n"] * batch for m in mats)
    launches_per_step = sum(bq.bq_gemv_launches(f, m["n"], m["k"], batch) for m in mats)
    calls_per_step = len(mats)
    # the arithmetic of the path bq_gemv takes for this format and batch
    int8_path = batch <= 4 and all(bq.bq_gemv_workspace_bytes(f, m["n"], m["k"], batch) == 0 for m in mats)
    path_dtype = "s8xu8->s32 (warp MMA), f32 recombine" if int8_path else "f16 (tcgen05) -> f32"
    path_kernel = ("gemv_rows_kernel (row-owning tensor-core GEMV)" if int8_path
                   else "xprep_f16_kernel + gemm_tc_kernel (tcgen05 GEMM with T = batch)")

    def step():
        for m in mats:
            bq.bq_gemv(f, m["codes"], m["scales"], m["n"], m["k"], m["x"], y=m["y"], workspace=workspace)

    # warm up eagerly (lazy initialisation), then capture one step in a CUDA graph
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert bq.bq_check() == bq.BQ_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        graph.replay()
    barrier()
    assert bq.bq_check() == bq.BQ_OK

    # ---- device-timed region
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        graph.replay()
    t_end.record(stream)
    barrier()
    clocks = sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    assert bq.bq_check() == bq.BQ_OK

    # ---- LM head alone (largest launch): per-launch time with events around it
    head = mats[-1]
    hg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(hg):
        bq.bq_gemv(f, head["codes"], head["scales"], head["n"], head["k"], head["x"], y=head["y"],
                   workspace=workspace)
    hg.replay()
    torch.cuda.synchronize()
    h_times = []
    for _ in range(max(3, args.steps)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        graph.replay()  # evicts the head's weights from L2 (1 GB streamed)
        e0.record(stream)
        hg.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        h_times.append(e0.elapsed_time(e1))
    head_bytes = head["codes"].numel() + 2 * head["scales"].numel() + 2 * head["k"] * batch + 2 * head["n"] * batch
    head_ms = statistics.median(h_times)

    # ---- end-to-end through the public API: pinned host inputs in, outputs out
    e2e = None
    if not args.no_e2e:
        x_host = torch.empty_like(X_all, device="cpu").pin_memory()
        x_host.copy_(X_all)
        y_host = torch.empty_like(Y_all, device="cpu").pin_memory()

        def e2e_step():
            X_all.copy_(x_host, non_blocking=True)
            graph.replay()
            y_host.copy_(Y_all, non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        barrier()
        e2e = {"ms_per_step": e0.elapsed_time(e1) / args.steps,
               "h2d": sum(2 * batch * m["k"] for m in mats), "d2h": sum(2 * batch * m["n"] for m in mats)}

    # ---- max over ranks
    ms_per_step, e2e_ms = max_over_ranks([elapsed_ms / args.steps, e2e["ms_per_step"] if e2e else 0.0], dist, dev)
    if e2e:
        e2e["ms_per_step"] = e2e_ms

    peak, peak_src = measured_peaks()
    value = job_value(weight_bytes, world, ms_per_step)
    achieved = algo_bytes / (ms_per_step / 1000.0) / 1e9
    traffic = recorded_traffic(args.model, fmt, batch, args.layers)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(fmt, mats, batch)
    prefill = None
    if rank == 0 and not args.no_gemm:
        del graph, hg
        graph = hg = None
        mats.clear()
        torch.cuda.empty_cache()
        prefill = gemm_leg(fmt, dev, 5)

    if rank == 0:
        line = {
            "metric": "effective weight GB/s (g128 GEMV weight stream)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": path_dtype, "data": "synthetic",
            "config": {"workload": workload_name(args.model, fmt, batch, args.layers), "fmt": fmt, "batch": batch,
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
        if prefill:
            line["prefill_gemm"] = prefill
        print(json.dumps(line), flush=True)

    del graph, hg
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
