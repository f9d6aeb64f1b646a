#!/usr/bin/env python
"""Benchmark of the NVFP4 ScaleSearch hot path on B200.

One step = one pass of the whole path over one synthetic batch resident in HBM:
  tensor amax -> [all-reduce(max) across ranks] -> tensor scale g -> ScaleSearch quantize (f in [-2,6])
  -> dequantize to FP32.
Default workload: the 4 GiB FP32 stream (2^30 elements, mixture 0.9 N(0,1) + 0.1 N(0,16), seed 3), the
configuration the throughput target is stated on.  Every step's input (4 GiB) is larger than the
126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Workloads: stream_f32 (default), act_f32, act_bf16, kv_bf16, bev_f16, and gemm_nvfp4 -- the tensor-core
consumer: ScaleSearch-quantized BF16 activations [8192, 8192] times NVFP4 weights [8192, 8192] on the
tensor cores, reported in TFLOP/s against the FP4 tensor roofline; and msda_nvfp4 -- deformable attention
over the BEVFormer value maps with ScaleSearch NVFP4 values, reported in queries/s; and attn_nvfp4 --
causal attention with NVFP4 Q K^T and P V^T on the tensor cores, reported in TFLOP/s.

Prints ONE JSON line on rank 0.  Times are CUDA events on the launching stream, max over ranks.
`--impl reference` times the CPU oracle (the plain C definition) on a bounded sample of the same
workload on the host cores.
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

METRIC = "NVFP4 ScaleSearch quantize GB/s (input) and fraction of 8 TB/s HBM roofline"
OVERLAP_CHUNKS = 4            # round trip: search chunk i+1 while chunk i is dequantized on a second stream
OVERLAP_DEQ_CTAS_PER_SM = 2   # measured: 4 chunks x 2 CTAs/SM beat 8 or 16 chunks and 1 CTA/SM
FALLBACK_HBM_GBS = 6650.0
SOURCE_NOTE = "synthetic (seeded generators; stand-in for LLM activations / KV keys / BEV value maps)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="stream_f32")
    ap.add_argument("--scale", type=float, default=1.0, help="fraction of the workload size (profiling runs)")
    ap.add_argument("--f-lo", type=int, default=-2)
    ap.add_argument("--f-hi", type=int, default=6)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time the eager step only (no CUDA graph replay)")
    ap.add_argument("--kv-layers", type=int, default=32, help="kv_decode_layers: layers flushed per step (K and V each)")
    ap.add_argument("--no-configs", action="store_true",
                    help="default workload: skip the per-configuration lines of the other four workloads")
    ap.add_argument("--config-steps", type=int, default=50, help="timed steps of each per-configuration run")
    ap.add_argument("--with-configs", action="store_true", help="add the per-configuration lines at any --scale")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def captured_traffic(kernel_key: str, elements: int):
    """DRAM bytes per launch from the committed ncu record, scaled to `elements`; None when the kernel
    sources changed since the capture (the counters then no longer describe the compiled kernel)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
            rec = json.load(fh)[kernel_key]
        h = hashlib.sha256()
        for f in rec["source_files"]:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        per = (rec["dram_bytes_read"] + rec["dram_bytes_write"]) / rec["captured_elements"]
        return per * elements
    except Exception:
        return None


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampler unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        with open(self.path) as fh:
            for line in fh:
                parts = [s.strip() for s in line.split(",")]
                if len(parts) < 4:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx.append(float(parts[1]))
                    bits = int(parts[3], 16)
                except ValueError:
                    continue
                for b, name in REASON_BITS.items():
                    if bits & b and name != "gpu_idle":
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU oracle arm
# ------------------------------------------------------------------------------------------------
def oracle_sample(name: str, elems: int):
    """A bounded CPU sample of the workload's recipe (same generator recipe, CPU stream)."""
    from nvfp4_block_scaled_11_b200 import workloads as W
    if name == "stream_f32":
        x = W.stream_f32("cpu", elems / float(1 << 30))
    elif name == "kv_bf16":
        import numpy as np
        import torch
        T = max(64, elems // 128)
        k = W.kv_bf16("cpu", scale=T / 32768, heads=1)
        return k.view(torch.int16).numpy().view(np.uint16), "kv", k.numel()
    else:
        w = W.make(name, "cpu")
        x = w.x.reshape(-1)[:elems].contiguous()
    import numpy as np
    import torch
    if x.dtype == torch.float32:
        return x.numpy().reshape(-1), 0, x.numel()
    code = 1 if x.dtype == torch.bfloat16 else 2
    return x.view(torch.int16).numpy().view(np.uint16).reshape(-1), code, x.numel()


def oracle_step(xs, code, f_lo, f_hi):
    from oracle import oracle as O
    if code == "kv":
        _, _, c, s, g = O.kv_mixed(xs, 16, 16, 1, f_lo, f_hi)
        O.dequantize(c.reshape(-1), s.reshape(-1), g, 1)
        return
    c, s, g, _, _ = O.quantize(xs, f_lo, f_hi, dtype=code)
    O.dequantize(c, s, g, 0)


def time_oracle(name, f_lo, f_hi, budget_s, max_elems=1 << 25):
    """Pick a sample size whose oracle step takes about budget_s, then time one step."""
    probe = 1 << 16
    xs, code, n = oracle_sample(name, probe)
    t = time.perf_counter()
    oracle_step(xs, code, f_lo, f_hi)
    dt = time.perf_counter() - t
    elems = int(min(max_elems, max(probe, probe * budget_s / max(dt, 1e-6))))
    elems -= elems % 16
    xs, code, n = oracle_sample(name, elems)
    return xs, code, n


def quant_stats(nv, x, g, deq, f_lo, f_hi, elements_per_s):
    """Secondary statistics of the timed input, computed once after the timed region: the histogram of
    the chosen offsets f*, the total block SSE against max-scaling (window {0}) under the same g, and
    the normalised absolute error of the dequantized tensor (sums in float64, in chunks)."""
    import torch
    _, _, _, f, sse = nv.quantize_ex(x, f_lo, f_hi, gscale_in=g)
    _, _, _, _, sse0 = nv.quantize_ex(x, 0, 0, gscale_in=g, want_f=False)
    counts = torch.bincount(f.to(torch.int64) + 128, minlength=256).cpu().tolist()
    s, s0 = sse.double().sum().item(), sse0.double().sum().item()
    num = den = 0.0
    xf, df = x.reshape(-1), deq.reshape(-1)
    for i in range(0, xf.numel(), 1 << 26):
        a, b = xf[i:i + (1 << 26)].double(), df[i:i + (1 << 26)].double()
        num += (a - b).abs().sum().item()
        den += a.abs().sum().item()
    return {"elements_per_s": elements_per_s, "blocks": f.numel(),
            "f_star_hist": {str(i - 128): c for i, c in enumerate(counts) if c},
            "sse_total": s, "sse_max_scaling": s0, "mse_reduction_pct": 100.0 * (1.0 - s / s0) if s0 > 0 else None,
            "nae_dequant": num / den if den > 0 else None}


def run_reference(args, rank, world):
    if rank != 0:
        return
    budget = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    xs, code, n = time_oracle(args.workload, args.f_lo, args.f_hi, budget)
    for _ in range(args.warmup):
        oracle_step(xs, code, args.f_lo, args.f_hi)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(xs, code, args.f_lo, args.f_hi)
    el = time.perf_counter() - t
    bytes_in = n * xs.dtype.itemsize
    val = bytes_in * args.steps / el / 1e9
    sample = f"first {n} elements of the {args.workload} recipe per step (CPU generator), oracle quantize + dequantize"
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": workload_dtype(args.workload), "data": SOURCE_NOTE,
        "config": workload_config(args),
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


WORKLOAD_DTYPE = {"stream_f32": "f32", "act_f32": "f32", "act_bf16": "bf16", "kv_bf16": "bf16", "bev_f16": "f16"}


def workload_dtype(name: str) -> str:
    """The element type the quantize path reads and computes its dequantized values in (the search itself
    runs in FP32 on the widened values)."""
    return WORKLOAD_DTYPE.get(name, "f32")


def workload_config(args):
    from nvfp4_block_scaled_11_b200 import workloads as W
    notes = {
        "stream_f32": "FP32 2^30 = 4 GiB, 0.9 N(0,1) + 0.1 N(0,16), seed 3",
        "act_f32": "FP32 [1024,4096] N(0,1), seed 0",
        "act_bf16": "BF16 [8192,8192] 0.5*t(3), 1% outlier columns x20, seed 1",
        "kv_bf16": "BF16 K [1,8,32768,128], N(0,1) + N(0,2) bias on 4 channels, seed 2",
        "bev_f16": "FP16 [6,30825,8,32] N(0,1) x level gain 1,2,4,8, seed 5",
    }
    big = args.workload == "stream_f32" and args.scale >= 0.125   # 512 MiB and more: no flush needed
    name = f"{args.workload} ({notes.get(args.workload, '')})"
    if args.scale != 1.0:
        name += f" scaled by {args.scale}"
    return {
        "workload": name,
        "window": [args.f_lo, args.f_hi],
        "step": ("kv_mixed (sink/recent copy + FWHT-16 + amax + ScaleSearch) + dequantize BF16"
                 if args.workload == "kv_bf16" else
                 "amax + [allreduce max] + g + ScaleSearch quantize + dequantize"),
        "l2": ("inputs larger than L2 (at least 512 MiB per step per GPU), no flush" if big else
               "L2 flushed between steps by a 256 MiB write (not timed)"),
        "block": 16,
    }


# ------------------------------------------------------------------------------------------------
# Tensor-core consumer workload: an NVFP4 linear layer
# ------------------------------------------------------------------------------------------------
GEMM_METRIC = "NVFP4 linear layer TFLOP/s (ScaleSearch-quantized activations x NVFP4 weights, tensor cores)"
FP4_PER_BF16 = 4.0   # nominal dense FP4 / BF16 tensor throughput ratio of B200 (9 / 2.25 PFLOP/s)


def gemm_shape(args):
    return max(128, int(8192 * args.scale)), 8192, 8192     # M (tokens), N (outputs), K (inputs)


def gemm_config(args):
    M, N, K = gemm_shape(args)
    return {
        "workload": f"gemm_nvfp4 (activations BF16 [{M},{K}] 0.5*t(3) with 1% outlier columns x20, seed 1; "
                    f"weights BF16 [{N},{K}] N(0,1/{K}), seed 11)",
        "window": [args.f_lo, args.f_hi],
        "step": "activations: amax + g + ScaleSearch quantize with tile-layout scales; "
                "then D = g_a g_w A W^T on the tensor cores (NVFP4 x NVFP4, FP32 accumulate) -> BF16",
        "weights": "quantized once before timing (ScaleSearch [-2,6], tile-layout scales)",
        "l2": "L2 flushed between steps by a 256 MiB write (not timed)",
        "M": M, "N": N, "K": K, "block": 16,
    }


def oracle_gemm_sample(args, rows=64, w_rows=1024):
    """Oracle work for the CPU baseline: quantize `rows` activation rows and multiply them (fp64, exact
    products) by `w_rows` weight rows quantized beforehand.  Returns (step function, flops per step)."""
    import numpy as np
    import torch
    from nvfp4_block_scaled_11_b200 import workloads as W
    from oracle import oracle as O
    K = gemm_shape(args)[2]
    xa = W.act_bf16("cpu", rows / 8192.0)[:rows].contiguous()
    xw = W.weight_bf16("cpu", w_rows, K)
    a16 = xa.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    w16 = xw.view(torch.int16).numpy().view(np.uint16).reshape(-1)
    wc, ws, wg, _, _ = O.quantize(w16, args.f_lo, args.f_hi, dtype=O.BF16)

    def step():
        ac, as_, ag, _, _ = O.quantize(a16, args.f_lo, args.f_hi, dtype=O.BF16)
        O.gemm_nt(ac, as_, ag, wc, ws, wg, rows, w_rows, K)

    return step, 2.0 * rows * w_rows * K, f"{rows} activation rows x {w_rows} weight rows, K = {K}"


def run_gemm_reference(args, rank, world):
    if rank != 0:
        return
    step, flops, desc = oracle_gemm_sample(args)
    for _ in range(min(args.warmup, 3)):
        step()
    steps = max(1, min(args.steps, 20))
    t = time.perf_counter()
    for _ in range(steps):
        step()
    el = time.perf_counter() - t
    val = flops * steps / el / 1e12
    line = {
        "impl": "reference", "metric": GEMM_METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": min(args.warmup, 3), "ms_per_step": el / steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp4 x fp4 -> f64 (oracle)", "data": SOURCE_NOTE,
        "config": gemm_config(args),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": torch_threads(), "kind": "oracle",
                         "sample": desc + ": oracle quantize (C, 1 thread) + fp64 numpy product"},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def torch_threads():
    try:
        import numpy as np  # noqa: F401
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def run_gemm(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import workloads as W

    M, N, K = gemm_shape(args)
    x = W.act_bf16(dev, M / 8192.0)[:M].contiguous()
    w = W.weight_bf16(dev, N, K)
    wc, wsf, wg = nv.quantize_mma(w, args.f_lo, args.f_hi)
    del w
    ac = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    asf = torch.empty(nv.sf_mma_bytes(M, K), dtype=torch.uint8, device=dev)
    ag = torch.empty(1, dtype=torch.float32, device=dev)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    aw = torch.empty(1, dtype=torch.float32, device=dev)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        nv.quantize_mma(x, args.f_lo, args.f_hi, codes=ac, sf=asf, gscale=ag)
        if evs:
            evs[1].record(stream)
        nv.gemm_nt(ac, asf, ag, wc, wsf, wg, out=d, alpha_work=aw)
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    for k in range(args.steps):
        flush.fill_(float(k))
        step(evs[k])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    eager_ms = elapsed_ms
    graph_used = False
    if world == 1 and not args.no_graph:
        cg = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        torch.cuda.synchronize()
        with torch.cuda.graph(cg, stream=side):
            step()
        for _ in range(max(1, args.warmup)):
            cg.replay()
        torch.cuda.synchronize()
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for k in range(args.steps):
            flush.fill_(float(-k))
            gev[k][0].record(stream)
            cg.replay()
            gev[k][1].record(stream)
        torch.cuda.synchronize()
        graph_ms = sum(a.elapsed_time(b) for a, b in gev)
        del cg
        if graph_ms < elapsed_ms:
            elapsed_ms, graph_used = graph_ms, True
    q_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    g_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = t.item()
    flops = 2.0 * M * N * K
    bf16_peak, src = tensor_peak()
    fp4_peak = bf16_peak * FP4_PER_BF16
    achieved = flops / (g_ms * 1e-3) / 1e12
    line = {
        "metric": GEMM_METRIC, "value": world * flops * args.steps / (elapsed_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4 (e2m1 x e2m1, e4m3 block scales)",
        "data": SOURCE_NOTE, "config": gemm_config(args),
        "roofline": {"bound": "tensor", "kernel": "NVFP4 block-scaled GEMM (tcgen05, 128x128x256 tile)",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "traffic": None, "peak_source": f"{src} bf16 burst x {FP4_PER_BF16:g} (nominal fp4/bf16 ratio)",
                     "flops_per_launch": flops},
        "breakdown_ms": {"quantize_activations": q_ms, "gemm": g_ms},
        "quantize_activations": {"gbs_input": M * K * 2 / (q_ms * 1e-3) / 1e9},
        "gpu_launches": 5 * args.steps,
        "clocks": clocks,
        "cuda_graph": {"used_for_value": graph_used, "eager_ms_per_step": eager_ms / args.steps},
    }
    if not args.no_e2e and args.e2e_steps > 0:
        hx = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        hx.copy_(x)
        hd = torch.empty(d.shape, dtype=d.dtype, pin_memory=True)
        xin = torch.empty_like(x)

        def e2e_step():
            xin.copy_(hx, non_blocking=True)
            nv.quantize_mma(xin, args.f_lo, args.f_hi, codes=ac, sf=asf, gscale=ag)
            nv.gemm_nt(ac, asf, ag, wc, wsf, wg, out=d, alpha_work=aw)
            hd.copy_(d, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        line["e2e"] = {"value": world * flops * args.e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": hx.numel() * hx.element_size(),
                       "d2h_bytes_per_step": hd.numel() * hd.element_size()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        step_o, fl, desc = oracle_gemm_sample(args)
        step_o()
        t = time.perf_counter()
        step_o()
        el = time.perf_counter() - t
        line["cpu_baseline"] = {"value": fl / el / 1e12, "unit": "TFLOP/s", "cores": torch_threads(), "kind": "oracle",
                                "sample": desc + f": oracle quantize (C, 1 thread) + fp64 numpy product, {el:.2f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# Deformable attention on NVFP4 values (BEVFormer value maps)
# ------------------------------------------------------------------------------------------------
MSDA_METRIC = "deformable attention forward queries/s (ScaleSearch NVFP4 values, BEVFormer value maps)"


def msda_config(args):
    from nvfp4_block_scaled_11_b200 import workloads as W
    bs, nq, heads, L, P = 6, max(1, int(10000 * args.scale)), 8, len(W.LEVELS), 4   # as W.msda_inputs draws them
    return {
        "workload": f"msda_nvfp4 (value FP16 [6,30825,8,32] = bev_f16, levels {list(W.LEVELS)}; {nq} queries per "
                    f"camera, {L} levels x {P} points, loc ~ U(-0.05,1.05), softmax weights; seeds 5, 13)",
        "window": [args.f_lo, args.f_hi],
        "step": "value: amax + g + ScaleSearch quantize (blocks of 16 channels); deformable attention forward "
                "gathering NVFP4 values, FP32 interpolation and accumulation",
        "l2": "L2 flushed between steps by a 256 MiB write (not timed)",
        "bs": bs, "nq": nq, "heads": heads, "levels": L, "points": P, "channels": 32,
    }


def oracle_msda_sample(args, per_camera=10000):
    import numpy as np
    import torch
    from nvfp4_block_scaled_11_b200 import workloads as W
    from oracle import oracle as O
    value = W.bev_f16("cpu")
    bs, nk, heads, ch = value.shape
    loc, w = W.msda_inputs("cpu", scale=args.scale)
    vh = value.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    c, sc, g, _, _ = O.quantize(vh, args.f_lo, args.f_hi, dtype=O.F16)
    vq = O.dequantize(c, sc, g).reshape(bs, nk, heads, ch)
    per_camera = min(per_camera, loc.shape[1])
    ls, ws = loc[:, :per_camera].contiguous().numpy(), w[:, :per_camera].contiguous().numpy()

    def step():
        O.msda_forward(vq, W.LEVELS, ls, ws)

    return step, bs * per_camera, f"{per_camera} queries per camera x {bs} cameras, fp64 oracle forward on " \
                                  f"oracle-quantized values (value quantization not timed)"


def run_msda(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import workloads as W

    value = W.bev_f16(dev)
    bs, nk, heads, ch = value.shape
    loc, w = W.msda_inputs(dev, scale=args.scale)
    nq, L, P = loc.shape[1], loc.shape[3], loc.shape[4]
    n = value.numel()
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    scales = torch.empty(n // 16, dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    out = torch.empty((bs, nq, heads, ch), dtype=torch.float32, device=dev)
    trip = (codes.view(bs, nk, heads, ch // 2), scales.view(bs, nk, heads, ch // 16), g)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        nv.quantize(value.reshape(-1), args.f_lo, args.f_hi, codes=codes, scales=scales, gscale=g)
        if evs:
            evs[1].record(stream)
        nv.msda_forward(trip, W.LEVELS, loc, w, out=out)
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    for k in range(args.steps):
        flush.fill_(float(k))
        step(evs[k])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    q_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    m_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    def twin_ms(v):
        ts = []
        for k in range(max(3, args.steps // 10) + 3):
            flush.fill_(float(k))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            nv.msda_forward(v, W.LEVELS, loc, w, out=out)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.mean(ts[3:])

    f16_ms = twin_ms(value)
    v32 = value.float()
    f32_ms = twin_ms(v32)
    # accuracy of the NVFP4 path against the FP32-value forward (normalised absolute error)
    o4 = nv.msda_forward(trip, W.LEVELS, loc, w).double()
    o32 = nv.msda_forward(v32, W.LEVELS, loc, w).double()
    nae = float((o4 - o32).abs().mean() / o32.abs().mean())
    del v32, o4, o32
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = t.item()
    peak, src = peaks()
    msda_bytes = n // 2 + n // 16 + loc.numel() * 4 + w.numel() * 4 + out.numel() * 4
    achieved = msda_bytes / (m_ms * 1e-3) / 1e9
    line = {
        "metric": MSDA_METRIC, "value": world * bs * nq * args.steps / (elapsed_ms * 1e-3), "unit": "queries/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 values, f32 math",
        "data": SOURCE_NOTE, "config": msda_config(args),
        "roofline": {"bound": "hbm", "kernel": "msda_forward_kernel<NVFP4, 32> (gather-latency bound; value map "
                     "resident in L2)", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": src, "bytes_per_launch": msda_bytes},
        "breakdown_ms": {"quantize_value": q_ms, "msda_nvfp4": m_ms, "msda_f16_twin": f16_ms, "msda_f32_twin": f32_ms},
        "value_bytes": {"nvfp4": n // 2 + n // 16, "f16": n * 2, "f32": n * 4},
        "normalised_abs_error_vs_f32_values": nae,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    if not args.no_e2e and args.e2e_steps > 0:
        hv = torch.empty(value.shape, dtype=value.dtype, pin_memory=True)
        hv.copy_(value)
        hl = torch.empty(loc.shape, dtype=loc.dtype, pin_memory=True)
        hl.copy_(loc)
        hw = torch.empty(w.shape, dtype=w.dtype, pin_memory=True)
        hw.copy_(w)
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dv, dl, dw = torch.empty_like(value), torch.empty_like(loc), torch.empty_like(w)

        def e2e_step():
            dv.copy_(hv, non_blocking=True)
            dl.copy_(hl, non_blocking=True)
            dw.copy_(hw, non_blocking=True)
            nv.quantize(dv.reshape(-1), args.f_lo, args.f_hi, codes=codes, scales=scales, gscale=g)
            nv.msda_forward(trip, W.LEVELS, dl, dw, out=out)
            ho.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        line["e2e"] = {"value": world * bs * nq * args.e2e_steps / (e2e_ms * 1e-3), "unit": "queries/s",
                       "h2d_bytes_per_step": (hv.numel() * 2 + hl.numel() * 4 + hw.numel() * 4),
                       "d2h_bytes_per_step": ho.numel() * 4}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        step_o, nqs, desc = oracle_msda_sample(args)
        t = time.perf_counter()
        step_o()
        el = time.perf_counter() - t
        line["cpu_baseline"] = {"value": nqs / el, "unit": "queries/s", "cores": 1, "kind": "oracle",
                                "sample": desc + f", {el:.2f} s single-threaded C"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_msda_reference(args, rank, world):
    if rank != 0:
        return
    step, nqs, desc = oracle_msda_sample(args)
    steps = max(1, min(args.steps, 5))
    step()
    t = time.perf_counter()
    for _ in range(steps):
        step()
    el = time.perf_counter() - t
    val = nqs * steps / el
    print(json.dumps({
        "impl": "reference", "metric": MSDA_METRIC, "value": val, "unit": "queries/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": 1, "ms_per_step": el / steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 oracle", "data": SOURCE_NOTE, "config": msda_config(args),
        "cpu_baseline": {"value": val, "unit": "queries/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": val, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------------------------------------
# FP4 attention (ScaleSearchAttention numerics, unfused)
# ------------------------------------------------------------------------------------------------
KVD_METRIC = ("KV-cache decode: tokens appended per second (16-token groups of new keys quantized into the "
              "NVFP4 middle of the cache, 8 heads x 128)")


def kvd_config(args, n_new):
    return {
        "workload": f"kv_decode (cache = kv_bf16 keys [1,8,32768,128] with the prefill's tensor scale; {n_new} newly "
                    f"decoded keys [8,{n_new},128] BF16, N(0,1) + the same channel bias, seed 4)",
        "window": [args.f_lo, args.f_hi],
        "step": "one 16-token group of new keys, Hadamard-rotated and ScaleSearch-quantized with the prefill's "
                "tensor scale into the next 16 rows of the NVFP4 middle (nvfp4_kv_append)",
        "l2": "each group's 32 KB of keys is read once; latency-bound (1024 blocks per launch)",
        "heads": 8, "head_dim": 128, "group": 16,
    }


def run_kv_decode(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import workloads as W

    k = W.kv_bf16(dev)
    B, H, T, D = k.shape
    steps, warmup = max(1, args.steps), max(0, args.warmup)
    e2e_steps = max(0, args.e2e_steps) if not args.no_e2e else 0
    n_new = 16 * (steps + warmup + e2e_steps + 9)
    cap = (T - 32) + n_new
    g = nv.kv_gscale(k)                                   # the prefill's tensor scale (rotated middle)
    codes = torch.empty((H, cap, D // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((H, cap, D // 16), dtype=torch.uint8, device=dev)
    nv.kv_append(k[0], 16, T - 32, g, codes, scales, 0)   # prefill of the middle (not timed)
    new = W.kv_decode_keys(dev, n_new)
    stream = torch.cuda.current_stream(dev)
    group = [0]

    def step():
        i = group[0]
        nv.kv_append(new, 16 * i, 16, g, codes, scales, (T - 32) + 16 * i, f_lo=args.f_lo, f_hi=args.f_hi)
        group[0] += 1

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = t0.elapsed_time(t1)
    call_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    eager_ms = elapsed_ms
    graph_used = False
    if world == 1 and not args.no_graph and steps >= 8:
        # a decode loop runs as a CUDA graph: 8 consecutive group appends captured once and replayed, every
        # replay quantizing the same 8 groups into the same rows again (the same work per group)
        base = group[0]
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)

        def eight():
            for j in range(8):
                nv.kv_append(new, 16 * (base + j), 16, g, codes, scales, (T - 32) + 16 * (base + j),
                             f_lo=args.f_lo, f_hi=args.f_hi)

        with torch.cuda.stream(side):
            eight()
        torch.cuda.synchronize()
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=side):
            eight()
        cg.replay()
        torch.cuda.synchronize()
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ga.record(stream)
        for _ in range(steps // 8):
            cg.replay()
        gb.record(stream)
        torch.cuda.synchronize()
        graph_ms = ga.elapsed_time(gb) * steps / (8 * (steps // 8))   # per `steps` groups
        del cg
        group[0] += 8
        if graph_ms < elapsed_ms:
            elapsed_ms, graph_used = graph_ms, True
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = t.item()
    peak, psrc = peaks()
    nbytes = 16 * H * D * 2 + 16 * H * (D // 2) + 16 * H * (D // 16)
    launch_ms = elapsed_ms / steps if graph_used else call_ms     # one launch per group
    line = {
        "metric": KVD_METRIC, "value": world * 16 * steps / (elapsed_ms * 1e-3), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": elapsed_ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, nvfp4 out",
        "data": SOURCE_NOTE, "config": kvd_config(args, n_new),
        "roofline": {"bound": "hbm", "kernel": "quantize_lanes_kernel (KV append, 1024 blocks per launch)",
                     "achieved": nbytes / (launch_ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": nbytes / (launch_ms * 1e-3) / 1e9 / peak, "traffic": None, "peak_source": psrc,
                     "bytes_per_launch": nbytes,
                     "note": "latency-bound: a half warp per block (one offset per lane) on 64 CTAs, one "
                             "block's load-search-store chain per launch; the bytes are far below HBM's"},
        "gpu_launches": steps,
        "clocks": clocks,
        "cuda_graph": {"used_for_value": graph_used, "eager_ms_per_step": eager_ms / steps},
    }
    if e2e_steps > 0:
        # every step: the group's new keys from pinned host memory, the append, and the group's codes and
        # scales read back
        hk = torch.empty((H, 16 * e2e_steps, D), dtype=torch.bfloat16, pin_memory=True)
        hk.copy_(new[:, 16 * group[0]:16 * (group[0] + e2e_steps)])
        dk = torch.empty((H, 16, D), dtype=torch.bfloat16, device=dev)
        hc = torch.empty((H, 16, D // 2), dtype=torch.uint8, pin_memory=True)
        hs = torch.empty((H, 16, D // 16), dtype=torch.uint8, pin_memory=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for j in range(e2e_steps):
            row = (T - 32) + 16 * group[0]
            dk.copy_(hk[:, 16 * j:16 * (j + 1)], non_blocking=True)
            nv.kv_append(dk, 0, 16, g, codes, scales, row, f_lo=args.f_lo, f_hi=args.f_hi)
            hc.copy_(codes[:, row:row + 16], non_blocking=True)
            hs.copy_(scales[:, row:row + 16], non_blocking=True)
            group[0] += 1
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        line["e2e"] = {"value": world * 16 * e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": 16 * H * D * 2, "d2h_bytes_per_step": 16 * H * (D // 2 + D // 16)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = kvd_oracle_baseline(args)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def kvd_oracle_baseline(args, groups=20):
    """The oracle's append of `groups` 16-token groups (single-threaded C), as tokens/s."""
    import numpy as np
    import torch
    from nvfp4_block_scaled_11_b200 import workloads as W
    from oracle import oracle as O
    new = W.kv_decode_keys("cpu", 16 * groups).view(torch.int16).numpy().view(np.uint16)
    H, _, D = new.shape
    codes = np.zeros((H, 16 * groups, D // 2), np.uint8)
    scales = np.zeros((H, 16 * groups, D // 16), np.uint8)
    g = 0.0015   # a tensor scale of the prefill's magnitude (the oracle's cost does not depend on its value)
    t = time.perf_counter()
    for i in range(groups):
        O.kv_append(new, 16 * i, 16, g, codes, scales, 16 * i, 1, args.f_lo, args.f_hi)
    el = time.perf_counter() - t
    return {"value": 16 * groups / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{groups} groups of 16 new keys x 8 heads, oracle kv_append (C, 1 thread), {el:.2f} s"}


def run_kvd_reference(args, rank, world):
    if rank != 0:
        return
    for _ in range(args.warmup):
        kvd_oracle_baseline(args, groups=4)
    cb = kvd_oracle_baseline(args, groups=max(4, min(200, 4 * max(1, args.steps))))
    line = {
        "impl": "reference", "metric": KVD_METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 16e3 / cb["value"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, nvfp4 out", "data": SOURCE_NOTE,
        "config": kvd_config(args, 16 * max(1, args.steps)), "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


KVDL_METRIC = ("KV-cache decode, whole model: tokens appended per second (every step one 16-token group of new "
               "keys and values leaves the BF16 window of each of L layers' K and V caches, 8 heads x 128 each, "
               "quantized in one batched launch)")


def kvdl_config(args, n_new):
    L = args.kv_layers
    return {
        "workload": f"kv_decode_layers ({2 * L} caches = K and V of {L} layers, each 8 heads x 128 with the kv_bf16 "
                    f"prefill's tensor scale; per cache {n_new} new rows [8,{n_new},128] BF16 = kv_decode_keys x "
                    f"(1 + 0.01 j) for cache j)",
        "window": [args.f_lo, args.f_hi], "layers": L, "caches": 2 * L,
        "step": f"one decode flush: {2 * L} 16-token groups (Hadamard-rotated, ScaleSearch with the tensor scale) "
                f"into the next 16 rows of each cache's NVFP4 middle, one nvfp4_kv_append_batch launch",
        "l2": f"{2 * L} x 32 KB of window keys read once per step; latency-bound",
    }


def run_kv_decode_layers(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import workloads as W

    L = max(1, min(args.kv_layers, nv.KV_APPEND_BATCH_MAX // 2))
    args.kv_layers = L
    C = 2 * L
    k = W.kv_bf16(dev)
    _, H, _, D = k.shape
    g = nv.kv_gscale(k)
    del k
    steps, warmup = max(1, args.steps), max(0, args.warmup)
    e2e_steps = max(0, args.e2e_steps) if not args.no_e2e else 0
    n_new = 16 * (steps + warmup + e2e_steps + 9)
    base = W.kv_decode_keys(dev, n_new)
    srcs = [(base.float() * (1.0 + 0.01 * j)).to(torch.bfloat16) for j in range(C)]
    codes_all = torch.empty((C, H, n_new, D // 2), dtype=torch.uint8, device=dev)
    scales_all = torch.empty((C, H, n_new, D // 16), dtype=torch.uint8, device=dev)
    codes, scales = list(codes_all), list(scales_all)
    stream = torch.cuda.current_stream(dev)
    group = [0]
    # the caches' descriptors are prepared once; each flush sets only the rows
    batch = nv.KvAppendBatch([(srcs[j], g, codes[j], scales[j], True, False) for j in range(C)], args.f_lo, args.f_hi)

    def step():
        batch(16 * group[0], 16, 16 * group[0])
        group[0] += 1

    def separate(i):
        for j in range(C):
            nv.kv_append(srcs[j], 16 * i, 16, g, codes[j], scales[j], 16 * i, f_lo=args.f_lo, f_hi=args.f_hi)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = eager_ms = t0.elapsed_time(t1)
    graph_used, sep_ms = False, None
    if world == 1 and not args.no_graph and steps >= 8:
        # the decode loop as a CUDA graph: 8 consecutive flushes captured once and replayed (the same rows
        # rewritten, the same work per flush); the same 8 flushes as 2L launches each, timed beside it
        g0 = group[0]
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)

        def graph_ms(fn):
            with torch.cuda.stream(side):
                fn()
            torch.cuda.synchronize()
            cg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(cg, stream=side):
                fn()
            cg.replay()
            torch.cuda.synchronize()
            ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ga.record(stream)
            for _ in range(steps // 8):
                cg.replay()
            gb.record(stream)
            torch.cuda.synchronize()
            del cg
            return ga.elapsed_time(gb) * steps / (8 * (steps // 8))

        batched = graph_ms(lambda: [batch(16 * (g0 + j), 16, 16 * (g0 + j)) for j in range(8)])
        sep_ms = graph_ms(lambda: [separate(g0 + j) for j in range(8)]) / steps
        group[0] += 8
        if batched < elapsed_ms:
            elapsed_ms, graph_used = batched, True
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = t.item()
    peak, psrc = peaks()
    nbytes = C * (16 * H * D * 2 + 16 * H * (D // 2) + 16 * H * (D // 16))
    launch_ms = elapsed_ms / steps
    line = {
        "metric": KVDL_METRIC, "value": world * 16 * steps / (elapsed_ms * 1e-3), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": elapsed_ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, nvfp4 out",
        "data": SOURCE_NOTE, "config": kvdl_config(args, n_new),
        "roofline": {"bound": "hbm", "kernel": f"kv_append_batch_kernel ({C} items, {C * 1024} blocks per launch)",
                     "achieved": nbytes / (launch_ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": nbytes / (launch_ms * 1e-3) / 1e9 / peak, "traffic": None, "peak_source": psrc,
                     "bytes_per_launch": nbytes,
                     "note": "latency-bound: one launch per step; lane groups (16 lanes per block while the "
                             "batch has at most 4096 blocks, then 4 lanes x 3 offsets)"},
        "gpu_launches": steps,
        "clocks": clocks,
        "cuda_graph": {"used_for_value": graph_used, "eager_ms_per_step": eager_ms / steps,
                       "separate_launches_ms_per_step": sep_ms},
    }
    if e2e_steps > 0:
        # every step: the C windows' 16 new rows from pinned host memory (one copy), one batched flush,
        # and the C groups' codes and scales read back (one copy each)
        hk = torch.empty((C, H, 16 * e2e_steps, D), dtype=torch.bfloat16, pin_memory=True)
        for j in range(C):
            hk[j].copy_(srcs[j][:, 16 * group[0]:16 * (group[0] + e2e_steps)])
        dk = torch.empty((C, H, 16, D), dtype=torch.bfloat16, device=dev)
        hc = torch.empty((C, H, 16, D // 2), dtype=torch.uint8, pin_memory=True)
        hs = torch.empty((C, H, 16, D // 16), dtype=torch.uint8, pin_memory=True)
        ebatch = nv.KvAppendBatch([(dk[j], g, codes[j], scales[j], True, False) for j in range(C)],
                                  args.f_lo, args.f_hi)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(e2e_steps):
            row = 16 * group[0]
            dk.copy_(hk[:, :, 16 * i:16 * (i + 1)], non_blocking=True)
            ebatch(0, 16, row)
            hc.copy_(codes_all[:, :, row:row + 16], non_blocking=True)
            hs.copy_(scales_all[:, :, row:row + 16], non_blocking=True)
            group[0] += 1
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        line["e2e"] = {"value": world * 16 * e2e_steps / (e2e_ms * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": C * 16 * H * D * 2, "d2h_bytes_per_step": C * 16 * H * (D // 2 + D // 16)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = kvdl_oracle_baseline(args)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def kvdl_oracle_baseline(args, steps=4):
    """The oracle appending `steps` flushes of 2L 16-token groups (single-threaded C), as tokens/s."""
    cb = kvd_oracle_baseline(args, groups=steps * 2 * args.kv_layers)
    value = cb["value"] / (2 * args.kv_layers)      # one sequence token = a row in each of the 2L caches
    return {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{steps} flushes of {2 * args.kv_layers} groups of 16 new keys x 8 heads, oracle kv_append "
                      f"(C, 1 thread)"}


def run_kvdl_reference(args, rank, world):
    if rank != 0:
        return
    args.kv_layers = max(1, min(args.kv_layers, 32))
    for _ in range(args.warmup):
        kvdl_oracle_baseline(args, steps=1)
    cb = kvdl_oracle_baseline(args, steps=max(1, min(8, args.steps)))
    line = {
        "impl": "reference", "metric": KVDL_METRIC, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 16e3 / cb["value"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, nvfp4 out", "data": SOURCE_NOTE,
        "config": kvdl_config(args, 16 * max(1, args.steps)), "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


ATTN_METRIC = "FP4 attention TFLOP/s (4*H*Tq*Tk*D per step; NVFP4 Q K^T and P V^T on the tensor cores)"


def attn_config(args, shape):
    H, Tq, Tk, D = shape
    return {
        "workload": f"attn_nvfp4 (q [{H},{Tq},{D}] N(0,1) seed 21; k = KV-cache keys [{H},{Tk},{D}] (N(0,1) + channel "
                    f"bias, seed 2); v [{H},{Tk},{D}] N(0,1) seed 22; BF16; causal, queries at the end)",
        "window": [args.f_lo, args.f_hi],
        "step": "ScaleSearch NVFP4 quantize of Hadamard-16-rotated q, k (rotation fused into amax and search; "
                "tile layout) and of v along tokens; "
                "S = Q K^T (FP4 tensor cores); softmax numerators quantized with ScaleSearch; O = P~ V^T "
                "(FP4 tensor cores) / rowsum",
        "l2": "inputs and scores larger than L2 (S is 2.1 GB), no flush",
        "H": H, "Tq": Tq, "Tk": Tk, "D": D,
    }


def run_attn(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import workloads as W

    q, k, v = W.attn_inputs(dev, scale=args.scale)
    H, Tq, D = q.shape
    Tk = k.shape[1]
    stream = torch.cuda.current_stream(dev)
    scale = D ** -0.5
    # every intermediate preallocated, so the step launches kernels only (no allocator calls)
    f32, u8 = torch.float32, torch.uint8
    E = lambda *shape, dt=f32: torch.empty(shape, dtype=dt, device=dev)
    qc, qsf, qg = E(H, Tq, D // 2, dt=u8), E(nv.sf_mma_bytes(Tq, D, H), dt=u8), E(1)
    kc, ksf, kg = E(H, Tk, D // 2, dt=u8), E(nv.sf_mma_bytes(Tk, D, H), dt=u8), E(1)
    q4, k4, qc4, kc4 = q[None], k[None], qc[None], kc[None]   # [1, H, T, D] views for the fused prologue
    vc, vsf, vg = E(H, D, Tk // 2, dt=u8), E(nv.sf_mma_bytes(D, Tk, H), dt=u8), E(1)
    s_buf = E(H, Tq, Tk)
    pc, psf, pg = E(H, Tq, Tk // 2, dt=u8), E(nv.sf_mma_bytes(Tq, Tk, H), dt=u8), E(1)
    m_buf, l_buf, o, aw1, aw2 = E(H * Tq), E(H * Tq), E(H, Tq, D), E(1), E(1)

    def step(evs=None):
        def mark(i):
            if evs:
                evs[i].record(stream)
        mark(0)
        # Hadamard-16 fused into the amax and search kernels of q and k (no FP32 copy)
        nv.kv_mixed_mma(q4, 0, 0, True, args.f_lo, args.f_hi, codes=qc4, sf=qsf, gscale=qg)
        nv.kv_mixed_mma(k4, 0, 0, True, args.f_lo, args.f_hi, codes=kc4, sf=ksf, gscale=kg)
        nv.quantize_mma_t(v, args.f_lo, args.f_hi, codes=vc, sf=vsf, gscale=vg)
        mark(1)
        nv.gemm_nt(qc, qsf, qg, kc, ksf, kg, alpha=scale, out=s_buf, alpha_work=aw1)
        mark(2)
        nv.softmax_quantize_mma(s_buf, True, Tk - Tq, args.f_lo, args.f_hi, codes=pc, sf=psf, g=pg, m=m_buf, l=l_buf)
        mark(3)
        nv.gemm_nt(pc, psf, pg, vc, vsf, vg, out=o, alpha_work=aw2)
        mark(4)
        nv.rows_divide(o, l_buf)
        mark(5)
        return o

    vside = torch.cuda.Stream(dev)

    def step_overlap():
        # V's quantization depends on neither Q nor K: it runs on a second stream beside the Q/K
        # prologue, the Q K^T product and the softmax, and joins before the P V^T product
        cur = torch.cuda.current_stream(dev)
        fork = torch.cuda.Event()
        fork.record(cur)
        vside.wait_event(fork)
        with torch.cuda.stream(vside):
            nv.quantize_mma_t(v, args.f_lo, args.f_hi, codes=vc, sf=vsf, gscale=vg)
        vdone = torch.cuda.Event()
        vdone.record(vside)
        nv.kv_mixed_mma(q4, 0, 0, True, args.f_lo, args.f_hi, codes=qc4, sf=qsf, gscale=qg)
        nv.kv_mixed_mma(k4, 0, 0, True, args.f_lo, args.f_hi, codes=kc4, sf=ksf, gscale=kg)
        nv.gemm_nt(qc, qsf, qg, kc, ksf, kg, alpha=scale, out=s_buf, alpha_work=aw1)
        nv.softmax_quantize_mma(s_buf, True, Tk - Tq, args.f_lo, args.f_hi, codes=pc, sf=psf, g=pg, m=m_buf, l=l_buf)
        cur.wait_event(vdone)
        nv.gemm_nt(pc, psf, pg, vc, vsf, vg, out=o, alpha_work=aw2)
        nv.rows_divide(o, l_buf)
        return o

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    steps = max(1, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = t0.elapsed_time(t1)
    eager_ms = elapsed_ms
    graph_used = False
    v_overlap_used = False
    if world == 1 and not args.no_graph:
        cg = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        torch.cuda.synchronize()
        with torch.cuda.graph(cg, stream=side):
            step()
        cgo = torch.cuda.CUDAGraph()      # the same step with V's quantization on a second stream
        with torch.cuda.stream(side):
            step_overlap()
        torch.cuda.synchronize()
        with torch.cuda.graph(cgo, stream=side):
            step_overlap()
        graph_times = []
        for g_ in (cg, cgo):
            for _ in range(max(1, args.warmup)):
                g_.replay()
            torch.cuda.synchronize()
            ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ga.record(stream)
            for _ in range(steps):
                g_.replay()
            gb.record(stream)
            torch.cuda.synchronize()
            graph_times.append(ga.elapsed_time(gb))
        del cg, cgo
        graph_ms = min(graph_times)
        v_overlap_used = graph_times[1] < graph_times[0]
        if graph_ms < elapsed_ms:
            elapsed_ms, graph_used = graph_ms, True
    stage = [statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j in range(5)]
    chain_o = o.clone()

    # The same attention with the scores kept on chip: the prologue, then nvfp4_attention_fused (Q K^T,
    # row maxima, numerators, their ScaleSearch and P~ V^T in one kernel).  Timed eagerly (per-stage events)
    # and as a CUDA graph; the faster of the chain and this schedule sets `value`.
    fo, fm, fl, fst = E(H, Tq, D), E(H * Tq), E(H * Tq), torch.zeros(1, dtype=torch.int32, device=dev)
    fused_ok = world == 1 and Tq % 128 == 0 and Tk % 64 == 0 and D == 128
    f_splits = nv.attention_fused_splits(H, Tq, Tk) if fused_ok else 1
    f_ws = nv.attention_fused_workspace(H, Tq, Tk, f_splits, dev) if fused_ok else None

    def step_fused(evs=None):
        # V's quantization runs on a second stream beside Q's and K's and joins before the attention call
        cur = torch.cuda.current_stream(dev)
        if evs:
            evs[0].record(cur)
        fork = torch.cuda.Event()
        fork.record(cur)
        vside.wait_event(fork)
        with torch.cuda.stream(vside):
            nv.quantize_mma_t(v, args.f_lo, args.f_hi, codes=vc, sf=vsf, gscale=vg)
        vdone = torch.cuda.Event()
        vdone.record(vside)
        nv.kv_mixed_mma(q4, 0, 0, True, args.f_lo, args.f_hi, codes=qc4, sf=qsf, gscale=qg)
        nv.kv_mixed_mma(k4, 0, 0, True, args.f_lo, args.f_hi, codes=kc4, sf=ksf, gscale=kg)
        cur.wait_event(vdone)
        if evs:
            evs[1].record(cur)
        nv.attention_fused(qc, qsf, qg, kc, ksf, kg, vc, vsf, vg, True, Tk - Tq, scale, args.f_lo, args.f_hi,
                           out=fo, m=fm, l=fl, status=fst, splits=f_splits, workspace=f_ws)
        if evs:
            evs[2].record(cur)
        return fo

    fused = None
    if fused_ok:
        for _ in range(args.warmup):
            step_fused()
        torch.cuda.synchronize()
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        fa, fb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fa.record(stream)
        for i in range(steps):
            step_fused(fev[i])
        fb.record(stream)
        torch.cuda.synchronize()
        fused_ms = fa.elapsed_time(fb)
        fused_graph_ms = None
        if not args.no_graph:
            cgf = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step_fused()
            torch.cuda.synchronize()
            with torch.cuda.graph(cgf, stream=side):
                step_fused()
            for _ in range(max(1, args.warmup)):
                cgf.replay()
            torch.cuda.synchronize()
            fa.record(stream)
            for _ in range(steps):
                cgf.replay()
            fb.record(stream)
            torch.cuda.synchronize()
            fused_graph_ms = fa.elapsed_time(fb)
            del cgf
        best_f = min(fused_ms, fused_graph_ms) if fused_graph_ms is not None else fused_ms
        fused = {"ms_per_step": fused_ms / steps,
                 "graph_ms_per_step": fused_graph_ms / steps if fused_graph_ms is not None else None,
                 "prologue_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in fev),
                 "kernel_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in fev),
                 "splits": f_splits,
                 "status": int(fst.item()),
                 "max_abs_diff_vs_chain": float((fo - chain_o).abs().max().item()),
                 "used_for_value": best_f < elapsed_ms and fst.item() == 0}
        if fused["used_for_value"]:
            elapsed_ms = best_f
            graph_used = fused_graph_ms is not None and fused_graph_ms <= fused_ms
            o = fo
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = t.item()
    flops = 4.0 * H * Tq * Tk * D
    bf16_peak, src = tensor_peak()
    fp4_peak = bf16_peak * FP4_PER_BF16
    hbm_peak, hsrc = peaks()
    sm_bytes = H * Tq * Tk * 4 + H * Tq * Tk // 2 + H * Tq * Tk // 16 + 2 * H * Tq * 4
    # the fused kernel's arithmetic roofline: the certified fast score costs 3 FP32-pipe operations per
    # candidate and element (multiply, mixed-precision subtract, square-accumulate); P~ has one element per
    # allowed (query, key) pair and args.f_hi - args.f_lo + 1 candidates per block
    allowed = sum(min(Tk, q_ + (Tk - Tq) + 1) for q_ in range(Tq)) * H
    fused_fp32_ops = 3.0 * (args.f_hi - args.f_lo + 1) * allowed / 1e12 * 1e12
    fp32_peak = 128 * 148 * 1.965e9 / 1e12
    # accuracy against full-precision attention on the last 64 queries of head 0
    qf, kf, vf = q[0, -64:].double(), k[0].double(), v[0].double()
    sref = (qf @ kf.T) * scale
    mask = torch.arange(Tk, device=dev)[None, :] > torch.arange(Tq - 64, Tq, device=dev)[:, None] + (Tk - Tq)
    oref = torch.softmax(sref.masked_fill(mask, float("-inf")), -1) @ vf
    nae = float((o[0, -64:].double() - oref).abs().mean() / oref.abs().mean())
    line = {
        "metric": ATTN_METRIC, "value": world * flops * steps / (elapsed_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 operands, f32 accumulation", "data": SOURCE_NOTE, "config": attn_config(args, (H, Tq, Tk, D)),
        "roofline": ({"bound": "alu", "kernel": "nvfp4_attention_fused (row maxima, numerators with their "
                      "ScaleSearch and P~ V^T, combine; timed together)",
                      "achieved": fused_fp32_ops / (fused["kernel_ms"] * 1e-3) / 1e12,
                      "peak": fp32_peak, "unit": "TFLOP/s", "frac": fused_fp32_ops / (fused["kernel_ms"] * 1e-3) / 1e12 / fp32_peak,
                      "traffic": None, "peak_source": "FP32 pipes: 128 lanes x 148 SMs x 1.965 GHz (one operation per lane per cycle)",
                      "ops_per_launch": fused_fp32_ops,
                      "ops": "3 FP32-pipe operations per scored candidate and element of P~ (9 candidates, allowed keys)"}
                     if fused and fused["used_for_value"] else
                     {"bound": "hbm", "kernel": "softmax_quantize_kernel (reads the FP32 scores, writes NVFP4 P)",
                      "achieved": sm_bytes / (stage[2] * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                      "frac": sm_bytes / (stage[2] * 1e-3) / 1e9 / hbm_peak, "traffic": None, "peak_source": hsrc,
                      "bytes_per_launch": sm_bytes}),
        "fused": fused,
        "products": {"qk_tflops": 2.0 * H * Tq * Tk * D / (stage[1] * 1e-3) / 1e12,
                     "pv_tflops": 2.0 * H * Tq * Tk * D / (stage[3] * 1e-3) / 1e12,
                     "fp4_peak": fp4_peak, "peak_source": f"{src} bf16 burst x {FP4_PER_BF16:g}"},
        "breakdown_ms": {"rotate_and_quantize_qkv": stage[0], "qk_product": stage[1], "softmax_quantize": stage[2],
                         "pv_product": stage[3], "rows_divide": stage[4]},
        "normalised_abs_error_vs_fp64_attention": nae,
        # kernels + tensor-scale memsets: 9 in the prologue, then the row maxima, the numerators and (with
        # more than one key range) the combine; the chain: 18
        "gpu_launches": ((11 + (f_splits > 1)) if fused and fused["used_for_value"] else 18) * steps,
        "clocks": clocks,
        "cuda_graph": {"used_for_value": graph_used, "eager_ms_per_step": eager_ms / steps,
                       "v_quantize_on_second_stream": v_overlap_used},
    }
    if not args.no_e2e and args.e2e_steps > 0:
        # the schedule that set `value`, with every step's q, k, v copied in from pinned host memory and O
        # read back: inputs and outputs double-buffered on a copy stream, so that step k + 1's input copy
        # runs while step k computes (PCIe is the bound: 138 MB in per step)
        hq, hk, hv = (torch.empty(t_.shape, dtype=t_.dtype, pin_memory=True) for t_ in (q, k, v))
        hq.copy_(q), hk.copy_(k), hv.copy_(v)
        ho = [torch.empty((H, Tq, D), dtype=torch.float32, pin_memory=True) for _ in range(2)]
        dq = [torch.empty_like(q) for _ in range(2)]
        dk = [torch.empty_like(k) for _ in range(2)]
        dv = [torch.empty_like(v) for _ in range(2)]
        do = [E(H, Tq, D) for _ in range(2)]
        use_fused = bool(fused and fused["used_for_value"])
        cstream = torch.cuda.Stream(dev)

        def compute(i):
            b = i % 2
            if use_fused:
                nv.kv_mixed_mma(dq[b][None], 0, 0, True, args.f_lo, args.f_hi, codes=qc4, sf=qsf, gscale=qg)
                nv.kv_mixed_mma(dk[b][None], 0, 0, True, args.f_lo, args.f_hi, codes=kc4, sf=ksf, gscale=kg)
                nv.quantize_mma_t(dv[b], args.f_lo, args.f_hi, codes=vc, sf=vsf, gscale=vg)
                nv.attention_fused(qc, qsf, qg, kc, ksf, kg, vc, vsf, vg, True, Tk - Tq, scale, args.f_lo, args.f_hi,
                                   out=do[b], m=fm, l=fl, status=fst, splits=f_splits, workspace=f_ws)
            else:
                q.copy_(dq[b]), k.copy_(dk[b]), v.copy_(dv[b])
                do[b].copy_(step())

        def e2e_run(n):
            ready = [torch.cuda.Event() for _ in range(n)]
            done = [torch.cuda.Event() for _ in range(n)]

            def h2d(i):   # step i's inputs, enqueued one step ahead of its compute
                b = i % 2
                with torch.cuda.stream(cstream):
                    if i >= 2:
                        cstream.wait_event(done[i - 2])        # step i - 2 has finished with buffer b
                    dq[b].copy_(hq, non_blocking=True)
                    dk[b].copy_(hk, non_blocking=True)
                    dv[b].copy_(hv, non_blocking=True)
                    ready[i].record(cstream)

            h2d(0)
            for i in range(n):
                b = i % 2
                if i + 1 < n:
                    h2d(i + 1)
                stream.wait_event(ready[i])
                compute(i)
                done[i].record(stream)
                with torch.cuda.stream(cstream):   # after step i + 1's input copy on the copy stream
                    cstream.wait_event(done[i])
                    ho[b].copy_(do[b], non_blocking=True)

        e2e_run(2)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        a.record(cstream)
        stream.wait_event(a)
        e2e_run(args.e2e_steps)
        cstream.wait_stream(stream)
        b_.record(cstream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b_)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        line["e2e"] = {"value": world * flops * args.e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": sum(t_.numel() * t_.element_size() for t_ in (hq, hk, hv)),
                       "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size(),
                       "schedule": ("fused" if use_fused else "chain") +
                                   ", inputs and outputs double-buffered on a copy stream"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = attn_oracle_baseline(args)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def attn_oracle_baseline(args, Tq=64, Tk=1024):
    """The oracle pipeline on one head, Tq x Tk, timed on one host core."""
    import numpy as np
    import torch
    from nvfp4_block_scaled_11_b200 import workloads as W
    from oracle import oracle as O
    q, k, v = W.attn_inputs("cpu", scale=Tk / 32768)
    D = q.shape[2]
    u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    qh, kh, vh = u16(q[0, -Tq:]), u16(k[0, :Tk]), u16(v[0, :Tk])
    t = time.perf_counter()
    qc, qs, qg, _, _ = O.quantize(O.hadamard16(qh.reshape(-1), dtype=O.BF16, out_dtype=O.F32))
    kc, ks, kg, _, _ = O.quantize(O.hadamard16(kh.reshape(-1), dtype=O.BF16, out_dtype=O.F32))
    s = O.gemm_nt(qc, qs, qg, kc, ks, kg, Tq, Tk, D, D ** -0.5).astype(np.float32)
    pc, ps, _, pl, pg = O.softmax_quantize(s, True, Tk - Tq)
    vc, vs, vg, _, _ = O.quantize(np.ascontiguousarray(vh.T).reshape(-1), dtype=O.BF16)
    O.gemm_nt(pc, ps, pg, vc, vs, vg, Tq, D, Tk) / pl[..., None]
    el = time.perf_counter() - t
    return {"value": 4.0 * Tq * Tk * D / el / 1e12, "unit": "TFLOP/s", "cores": torch_threads(), "kind": "oracle",
            "sample": f"one head, {Tq} queries x {Tk} keys, D = {D}: the oracle pipeline (C quantize and softmax, "
                      f"fp64 numpy products), {el:.2f} s"}


def run_attn_reference(args, rank, world):
    if rank != 0:
        return
    base = attn_oracle_baseline(args)
    print(json.dumps({
        "impl": "reference", "metric": ATTN_METRIC, "value": base["value"], "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": 1, "warmup": 0, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4 operands, f64 oracle", "data": SOURCE_NOTE,
        "config": attn_config(args, (8, 2048, 32768, 128)), "cpu_baseline": base,
        "e2e": {"value": base["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if args.workload == "gemm_nvfp4":
            run_gemm_reference(args, rank, world)
        elif args.workload == "msda_nvfp4":
            run_msda_reference(args, rank, world)
        elif args.workload == "attn_nvfp4":
            run_attn_reference(args, rank, world)
        elif args.workload == "kv_decode":
            run_kvd_reference(args, rank, world)
        elif args.workload == "kv_decode_layers":
            run_kvdl_reference(args, rank, world)
        else:
            run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import nvfp4_block_scaled_11_b200 as nv
    from nvfp4_block_scaled_11_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if args.workload == "gemm_nvfp4":
        run_gemm(args, rank, world, dev)
        return
    if args.workload == "msda_nvfp4":
        run_msda(args, rank, world, dev)
        return
    if args.workload == "attn_nvfp4":
        run_attn(args, rank, world, dev)
        return
    if args.workload == "kv_decode":
        run_kv_decode(args, rank, world, dev)
        return
    if args.workload == "kv_decode_layers":
        run_kv_decode_layers(args, rank, world, dev)
        return
    w = W.make(args.workload, dev, args.scale, shard=rank)
    x = w.x.contiguous()
    n = x.numel()
    esz = x.element_size()
    kv = w.kind == "kv"
    torch.cuda.synchronize()

    amax = torch.empty(1, dtype=torch.float32, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    if kv:
        B, H, T, D = x.shape
        n_q = B * H * (T - 32) * D          # quantized middle tokens
        deq = torch.empty(n_q, dtype=torch.bfloat16, device=dev)
    else:
        x = x.reshape(-1)
        n_q = n
        codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(n // 16, dtype=torch.uint8, device=dev)
        deq = torch.empty(n, dtype=x.dtype, device=dev)
    stream = torch.cuda.current_stream(dev)
    # inputs that fit in L2 are evicted between timed steps by writing a 256 MiB buffer (not timed)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev) if n * esz < (512 << 20) else None

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        if kv:
            _, _, kc, ks, kg = nv.kv_mixed(x, 16, 16, True, args.f_lo, args.f_hi)
            if evs:
                evs[1].record(stream)
                evs[2].record(stream)
            nv.dequantize(kc.reshape(-1), ks.reshape(-1), kg, torch.bfloat16, out=deq)
        else:
            nv.tensor_amax(x, out=amax)
            if world > 1:
                dist.all_reduce(amax, op=dist.ReduceOp.MAX)
            nv.global_scale(amax, out=g)
            if evs:
                evs[1].record(stream)
            nv.quantize_ex(x, args.f_lo, args.f_hi, gscale_in=g, want_f=False, want_sse=False, codes=codes,
                           scales=scales, gscale=None)
            if evs:
                evs[2].record(stream)
            nv.dequantize(codes, scales, g, deq.dtype, out=deq)
        if evs:
            evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0.record(stream)
    for k in range(args.steps):
        if flush is not None:
            flush.fill_(float(k))
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if flush is None:
        elapsed_ms = t0.elapsed_time(t1)
    else:  # the flushes are not part of the step
        elapsed_ms = sum(e[0].elapsed_time(e[3]) for e in evs)

    def rmax(ms):
        """A time as the maximum over ranks, so that every rank compares the same numbers."""
        if world == 1:
            return ms
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.item()

    elapsed_ms = rmax(elapsed_ms)
    eager_ms = elapsed_ms
    graph_used = False
    if world == 1 and not args.no_graph:
        # the same step captured once as a CUDA graph and replayed: removes the host launch latency
        # that dominates the small configurations (the per-stage breakdown stays the eager one)
        cg = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()  # warm the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(cg, stream=side):
            step()
        for _ in range(max(1, args.warmup)):
            cg.replay()
        torch.cuda.synchronize()
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        ga = torch.cuda.Event(enable_timing=True)
        gb = torch.cuda.Event(enable_timing=True)
        ga.record(stream)
        for k in range(args.steps):
            if flush is not None:
                flush.fill_(float(-k))
            gev[k][0].record(stream)
            cg.replay()
            gev[k][1].record(stream)
        gb.record(stream)
        torch.cuda.synchronize()
        graph_ms = ga.elapsed_time(gb) if flush is None else sum(a.elapsed_time(b) for a, b in gev)
        del cg
        if graph_ms < elapsed_ms:
            elapsed_ms = graph_ms
            graph_used = True
    # The same step with the dequantize of finished chunks overlapped with the search of the next ones
    # (a second stream; the dequantize launched at 2 CTAs per SM so that it fits beside the 2 resident
    # search CTAs): same kernels, same outputs, for inputs larger than L2.
    overlap = None
    if not kv and flush is None and n % (OVERLAP_CHUNKS * 32) == 0:
        aux = torch.cuda.Stream(dev)
        c = n // OVERLAP_CHUNKS

        def step_overlap():
            nv.tensor_amax(x, out=amax)
            if world > 1:
                dist.all_reduce(amax, op=dist.ReduceOp.MAX)
            nv.global_scale(amax, out=g)
            for i in range(OVERLAP_CHUNKS):
                nv.quantize_ex(x[i * c:(i + 1) * c], args.f_lo, args.f_hi, gscale_in=g, want_f=False, want_sse=False,
                               codes=codes[i * c // 2:(i + 1) * c // 2], scales=scales[i * c // 16:(i + 1) * c // 16],
                               gscale=None)
                done = torch.cuda.Event()
                done.record(stream)
                aux.wait_event(done)
                with torch.cuda.stream(aux):
                    nv.dequantize(codes[i * c // 2:(i + 1) * c // 2], scales[i * c // 16:(i + 1) * c // 16], g,
                                  deq.dtype, out=deq[i * c:(i + 1) * c], ctas_per_sm=OVERLAP_DEQ_CTAS_PER_SM)
            joined = torch.cuda.Event()
            joined.record(aux)
            stream.wait_event(joined)

        for _ in range(args.warmup):
            step_overlap()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        oa, ob = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        oa.record(stream)
        for _ in range(args.steps):
            step_overlap()
        ob.record(stream)
        torch.cuda.synchronize()
        overlap_ms = rmax(oa.elapsed_time(ob))
        overlap = {"chunks": OVERLAP_CHUNKS, "dequant_ctas_per_sm": OVERLAP_DEQ_CTAS_PER_SM,
                   "ms_per_step": overlap_ms / args.steps, "used_for_value": overlap_ms < elapsed_ms}
        if overlap_ms < elapsed_ms:
            elapsed_ms = overlap_ms
            graph_used = False
    # The same step with the quantize and the dequantize fused (nvfp4_quantize_dequantize: the search
    # kernel writes each block's dequantized values as soon as its scale is chosen, so the codes are not
    # read back): same outputs (tested), one pass fewer over HBM.
    fused = None
    if True:
        def step_fused(ev=None):
            if kv:   # one call: copies + rotated amax + rotated search writing codes, scales and values
                if ev:
                    ev[0].record(stream)
                nv.kv_mixed_dequantize(x, 16, 16, True, args.f_lo, args.f_hi, mid_out=deq)
                if ev:
                    ev[1].record(stream)
                return
            nv.tensor_amax(x, out=amax)
            if world > 1:
                dist.all_reduce(amax, op=dist.ReduceOp.MAX)
            nv.global_scale(amax, out=g)
            if ev:
                ev[0].record(stream)
            nv.quantize_dequantize(x, args.f_lo, args.f_hi, gscale_in=g, codes=codes, scales=scales, gscale=None,
                                   out=deq)
            if ev:
                ev[1].record(stream)

        for _ in range(args.warmup):
            step_fused()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        fa, fb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fa.record(stream)
        for k in range(args.steps):
            if flush is not None:
                flush.fill_(float(k + 0.5))
            fev[k][2].record(stream)
            step_fused(fev[k])
            fev[k][3].record(stream)
        fb.record(stream)
        torch.cuda.synchronize()
        fused_ms = fa.elapsed_time(fb) if flush is None else sum(e[2].elapsed_time(e[3]) for e in fev)
        fused_ms = rmax(fused_ms)
        fused_graph_ms = None
        if world == 1 and not args.no_graph:
            # the fused step replayed as a CUDA graph (the small configurations are launch-bound)
            cgf = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                step_fused()
            torch.cuda.synchronize()
            with torch.cuda.graph(cgf, stream=side):
                step_fused()
            for _ in range(max(1, args.warmup)):
                cgf.replay()
            torch.cuda.synchronize()
            gfe = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
            fa.record(stream)
            for k in range(args.steps):
                if flush is not None:
                    flush.fill_(float(k + 0.25))
                gfe[k][0].record(stream)
                cgf.replay()
                gfe[k][1].record(stream)
            fb.record(stream)
            torch.cuda.synchronize()
            fused_graph_ms = fa.elapsed_time(fb) if flush is None else sum(a.elapsed_time(b) for a, b in gfe)
            del cgf
        fused = {"ms_per_step": fused_ms / args.steps,
                 "graph_ms_per_step": fused_graph_ms / args.steps if fused_graph_ms is not None else None,
                 "kernel_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in fev)}
        fused["graph_used"] = fused_graph_ms is not None and fused_graph_ms < fused_ms
        if fused["graph_used"]:
            fused_ms = fused_graph_ms
        fused["used_for_value"] = fused_ms < elapsed_ms
        if fused_ms < elapsed_ms:
            elapsed_ms = fused_ms
            graph_used = False
            if overlap:
                overlap["used_for_value"] = False
    # Steady-state stream of tensors: the amax pass of step k+1 (HBM-bound) runs on a second stream beside the
    # fused search of step k (bound by the FP32 pipes), each step with its own g word.  Every step still
    # computes its own amax before its own search; only consecutive steps overlap.
    pipelined = None
    if not kv and world == 1 and flush is None and fused is not None:
        aux = torch.cuda.Stream(dev)
        amax2 = torch.empty(2, dtype=torch.float32, device=dev)
        g2 = torch.empty(2, dtype=torch.float32, device=dev)

        def run_pipelined(nsteps):
            done = [None, None]
            nv.tensor_amax(x, out=amax2[0:1])
            nv.global_scale(amax2[0:1], out=g2[0:1])
            ready = torch.cuda.Event()
            ready.record(stream)
            for k in range(nsteps):
                nxt = None
                if k + 1 < nsteps:
                    j = (k + 1) % 2
                    if done[j] is not None:
                        aux.wait_event(done[j])      # step k-1's search has read g2[j]
                    with torch.cuda.stream(aux):
                        nv.tensor_amax(x, out=amax2[j:j + 1])
                        nv.global_scale(amax2[j:j + 1], out=g2[j:j + 1])
                    nxt = torch.cuda.Event()
                    nxt.record(aux)
                stream.wait_event(ready)
                i = k % 2
                nv.quantize_dequantize(x, args.f_lo, args.f_hi, gscale_in=g2[i:i + 1], codes=codes, scales=scales,
                                       gscale=None, out=deq)
                d = torch.cuda.Event()
                d.record(stream)
                done[i] = d
                ready = nxt

        run_pipelined(max(2, args.warmup))
        torch.cuda.synchronize()
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pa.record(stream)
        run_pipelined(args.steps)
        pb.record(stream)
        torch.cuda.synchronize()
        pipe_ms = pa.elapsed_time(pb)
        pipelined = {"ms_per_step": pipe_ms / args.steps, "streams": 2,
                     "schedule": "amax of step k+1 beside the fused search of step k (separate g words)",
                     "used_for_value": pipe_ms < elapsed_ms}
        if pipe_ms < elapsed_ms:
            elapsed_ms = pipe_ms
            graph_used = False
            fused["used_for_value"] = False
            if overlap:
                overlap["used_for_value"] = False
    # the window sweep of the streaming configuration: the search pass alone for {0}, the default window
    # and [-8,8], with the same g (CUDA events, mean of a few launches)
    sweep = None
    if not kv and world == 1:
        sweep = {}
        for lo, hi in ((0, 0), (args.f_lo, args.f_hi), (-8, 8)):
            nv.quantize_ex(x, lo, hi, gscale_in=g, want_f=False, want_sse=False, codes=codes, scales=scales, gscale=None)
            evs_s = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
            for a_, b_ in evs_s:
                if flush is not None:
                    flush.fill_(1.0)
                a_.record(stream)
                nv.quantize_ex(x, lo, hi, gscale_in=g, want_f=False, want_sse=False, codes=codes, scales=scales,
                               gscale=None)
                b_.record(stream)
            torch.cuda.synchronize()
            sweep[f"[{lo},{hi}]"] = statistics.mean(a_.elapsed_time(b_) for a_, b_ in evs_s)
    clocks = sampler.stop()   # sampled over the eager, graph, overlapped, fused and pipelined timings
    amax_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    q_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    dq_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)

    bytes_in = n * esz
    value = world * bytes_in * args.steps / (elapsed_ms * 1e-3) / 1e9
    peak, peak_src = peaks()
    q_bytes = n_q * esz + n_q // 2 + n_q // 16          # search pass: read x, write codes + scales
    two_pass_bytes = 2 * n_q * esz + n_q // 2 + n_q // 16
    dq_bytes = n_q // 2 + n_q // 16 + deq.element_size() * n_q
    if kv:
        # one fused call: copies + rotated amax + rotated search; report the call against its bytes
        q_ms = amax_ms + q_ms
        amax_ms = 0.0
    q_gbs = (two_pass_bytes if kv else q_bytes) / (q_ms * 1e-3) / 1e9
    f32_default = not kv and x.dtype == torch.float32 and (args.f_lo, args.f_hi) == (-2, 6)
    search_roofline = {"bound": "hbm",
                       "kernel": "kv_mixed (amax + search passes)" if kv else "quantize (ScaleSearch search + encode pass)",
                       "achieved": q_gbs, "peak": peak, "unit": "GB/s", "frac": q_gbs / peak,
                       "traffic": captured_traffic("quantize_search_kernel<0,0,0,9,0>", n) if f32_default else None,
                       "peak_source": peak_src, "bytes_per_launch": two_pass_bytes if kv else q_bytes}
    roofline = search_roofline
    if kv and fused and fused["used_for_value"]:
        launches = 4
        f_bytes = two_pass_bytes + deq.element_size() * n_q
        f_gbs = f_bytes / (fused["kernel_ms"] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": "kv_mixed_dequantize (copies + rotated amax + rotated search writing "
                    "codes, scales and values)", "achieved": f_gbs, "peak": peak, "unit": "GB/s", "frac": f_gbs / peak,
                    "traffic": None, "peak_source": peak_src, "bytes_per_launch": f_bytes}
    elif kv:
        launches = 5
    elif (fused and fused["used_for_value"]) or (pipelined and pipelined["used_for_value"]):
        # the step's dominant kernel is then the fused one: read x, write codes, scales and the values
        launches = 3
        f_bytes = n_q * esz + n_q // 2 + n_q // 16 + deq.element_size() * n_q
        f_gbs = f_bytes / (fused["kernel_ms"] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": "quantize_dequantize (ScaleSearch search + encode + dequantized values)",
                    "achieved": f_gbs, "peak": peak, "unit": "GB/s", "frac": f_gbs / peak,
                    "traffic": captured_traffic("quantize_search_kernel<0,0,0,9,0,0>", n) if f32_default else None,
                    "peak_source": peak_src, "bytes_per_launch": f_bytes}
    elif overlap and overlap["used_for_value"]:
        launches = 2 + 2 * OVERLAP_CHUNKS
    else:
        launches = 4

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": workload_dtype(args.workload), "data": SOURCE_NOTE,
        "config": workload_config(args),
        "roofline": roofline,
        "roofline_search_pass": search_roofline,
        "breakdown_ms": {"amax_and_g": amax_ms, "quantize": q_ms, "dequantize": dq_ms,
                         "fused_quantize_dequantize": fused["kernel_ms"] if fused else None},
        "quantize_two_pass": {"gbs_input": n_q * esz / ((amax_ms + q_ms) * 1e-3) / 1e9,
                              "gbs_moved": two_pass_bytes / ((amax_ms + q_ms) * 1e-3) / 1e9,
                              "frac_of_8TBs": two_pass_bytes / ((amax_ms + q_ms) * 1e-3) / 8e12},
        "dequantize": {"gbs_moved": dq_bytes / (dq_ms * 1e-3) / 1e9},
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
        "cuda_graph": {"used_for_value": graph_used, "eager_ms_per_step": eager_ms / args.steps},
        "overlap": overlap,
        "fused": fused,
        "pipelined": pipelined,
    }
    if sweep:
        base = amax_ms + sweep["[0,0]"]
        line["window_sweep_ms"] = {"amax_and_g": amax_ms, "search": sweep,
                                   "two_pass_over_max_scaling": {w: (amax_ms + t) / base for w, t in sweep.items()}}
    if not kv:
        line["stats"] = quant_stats(nv, x, g, deq, args.f_lo, args.f_hi, value / esz * 1e9)
        if world > 1:
            line["stats"]["scope"] = "rank 0's shard"
    if kv:
        args.no_e2e = True
    # end to end through the public API with host buffers: every step copies its whole input in from
    # pinned host memory, runs the step, and reads its quantized result (codes, scales, g) back.  The
    # buffers are doubled and the copies run on their own streams, so step k's read-back overlaps step
    # k+1's input copy (PCIe carries both directions at once); a buffer is reused only after the step
    # that last used it has been computed and read back.
    if not args.no_e2e and args.e2e_steps > 0:
        NB = 2
        hx = torch.empty(n, dtype=x.dtype, pin_memory=True)
        hx.copy_(x)
        xin = [torch.empty_like(x) for _ in range(NB)]
        cb = [codes] + [torch.empty_like(codes) for _ in range(NB - 1)]
        sb = [scales] + [torch.empty_like(scales) for _ in range(NB - 1)]
        gb = [g] + [torch.empty_like(g) for _ in range(NB - 1)]
        hc = [torch.empty(n // 2, dtype=torch.uint8, pin_memory=True) for _ in range(NB)]
        hs = [torch.empty(n // 16, dtype=torch.uint8, pin_memory=True) for _ in range(NB)]
        hg = [torch.empty(1, dtype=torch.float32, pin_memory=True) for _ in range(NB)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        fused_step = bool((fused and fused["used_for_value"]) or (pipelined and pipelined["used_for_value"]))
        computed, read_back = [None] * NB, [None] * NB

        def e2e_step(k):
            i = k % NB
            if computed[i] is not None:
                s_in.wait_event(computed[i])          # xin[i] was read by step k - NB
            with torch.cuda.stream(s_in):
                xin[i].copy_(hx, non_blocking=True)
            arrived = torch.cuda.Event()
            arrived.record(s_in)
            stream.wait_event(arrived)
            if read_back[i] is not None:
                stream.wait_event(read_back[i])       # cb[i], sb[i], gb[i] were read back by step k - NB
            nv.tensor_amax(xin[i], out=amax)
            if world > 1:
                dist.all_reduce(amax, op=dist.ReduceOp.MAX)
            nv.global_scale(amax, out=gb[i])
            if fused_step:   # the schedule that set `value`
                nv.quantize_dequantize(xin[i], args.f_lo, args.f_hi, gscale_in=gb[i], codes=cb[i], scales=sb[i],
                                       gscale=None, out=deq)
            else:
                nv.quantize_ex(xin[i], args.f_lo, args.f_hi, gscale_in=gb[i], want_f=False, want_sse=False,
                               codes=cb[i], scales=sb[i], gscale=None)
                nv.dequantize(cb[i], sb[i], gb[i], torch.float32, out=deq)
            done = torch.cuda.Event()
            done.record(stream)
            computed[i] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                hc[i].copy_(cb[i], non_blocking=True)
                hs[i].copy_(sb[i], non_blocking=True)
                hg[i].copy_(gb[i], non_blocking=True)
            back = torch.cuda.Event()
            back.record(s_out)
            read_back[i] = back

        e2e_step(0)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_event(a)
        for k in range(1, args.e2e_steps + 1):
            e2e_step(k)
        for ev in read_back:
            stream.wait_event(ev)
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = t.item()
        line["e2e"] = {"value": world * bytes_in * args.e2e_steps / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                       "h2d_bytes_per_step": bytes_in, "d2h_bytes_per_step": n // 2 + n // 16 + 4,
                       "schedule": ("fused round trip" if fused_step else "quantize + dequantize")
                       + ", input copy of step k+1 overlapping the read-back of step k"}
        del hx, hc, hs, hg, xin, cb, sb, gb

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xs, code, ns = time_oracle(args.workload, args.f_lo, args.f_hi, args.cpu_seconds)
        t = time.perf_counter()
        oracle_step(xs, code, args.f_lo, args.f_hi)
        el = time.perf_counter() - t
        line["cpu_baseline"] = {
            "value": ns * xs.dtype.itemsize / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{ns} elements of the {args.workload} recipe (CPU generator), one quantize + dequantize, "
                      f"{el:.1f} s single-threaded C",
        }
    if (rank == 0 and world == 1 and args.workload == "stream_f32" and (args.scale == 1.0 or args.with_configs)
            and not args.no_configs):
        line["configs"] = config_lines(args)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


CONFIG_KEYS = ("value", "unit", "ms_per_step", "dtype", "roofline", "cpu_baseline", "quantize_two_pass", "breakdown_ms",
               "clocks", "gpu_launches", "stats")


def config_lines(args):
    """The other four workloads (C1 act_f32, C2 act_bf16, C3 kv_bf16, C5 bev_f16), each measured by its own
    run of this script (same metric: input GB/s of amax + g + ScaleSearch + dequantize), so that one default
    run reports every configuration with its roofline and CPU baseline.  Each entry keeps the sub-run's
    keys that describe its number; a failed sub-run is recorded as such."""
    out = {}
    for name in ("act_f32", "act_bf16", "kv_bf16", "bev_f16"):
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", name, "--steps", str(args.config_steps),
               "--warmup", str(max(3, args.warmup)), "--no-e2e", "--cpu-seconds", "2", "--no-configs",
               "--f-lo", str(args.f_lo), "--f-hi", str(args.f_hi)]
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=600,
                               env={k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")})
            rows = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
            d = json.loads(rows[-1]) if r.returncode == 0 and rows else None
        except (subprocess.TimeoutExpired, ValueError):
            d = None
        if d is None:
            out[name] = {"error": "sub-run failed"}
            continue
        e = {k: d[k] for k in CONFIG_KEYS if k in d}
        e["workload"] = d["config"]["workload"]
        e["steps"] = d["steps"]
        if "roofline" in e and "quantize_two_pass" in d:
            e["frac_of_8TBs_two_pass_quantize"] = d["quantize_two_pass"]["frac_of_8TBs"]
        out[name] = e
    return out


if __name__ == "__main__":
    main()
