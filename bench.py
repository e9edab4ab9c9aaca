#!/usr/bin/env python
"""Benchmark of the Step-5 routed-MoE layer forward on B200. Prints one JSON line.

Headline workload: the Step-5 MoE layer prefill with FP8 experts, T = 8192
tokens (hidden 4096, 352 routed experts, top-8, one shared expert,
intermediate 1536; 128x128 E4M3 weight blocks, 1x128 E4M3 activations).
A step is one whole layer forward (router, top-k, histogram/scan/permute,
gather+quantise, gate/up GEMM + SwiGLU, down GEMM, combine) through the C ABI
on inputs already resident in HBM. The line also carries the FP8 decode
workload (T = 64) that the metric quotes, measured the same way.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (one per GPU; the layer does not shard on
one node in this design) under torchrun; the value is the tokens of all ranks
over the slowest rank's time. --impl reference times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Step-5 MoE layer tokens/s (FP8, T=8192 / T=64) and % of FP8 / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 256 << 20
KERNELS = ["router_gemm", "router_topk", "histogram", "scan", "scatter", "gather", "gemm1_gate_up_swiglu",
           "gemm2_down", "combine"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill-fp8", "decode-bf16", "long-skew-fp8", "dense-ffn-fp8",
                                           "nvfp4"],
                    default="prefill-fp8")
    ap.add_argument("--no-decode", action="store_true", help="skip the T=64 FP8 decode line")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the Zipf-skewed T=32768 long prefill, FP8 decode-sweep, NVFP4 and dense-FFN lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--residual", action="store_true",
                    help="also time the residual-stream kernels (RMSNorm in, residual combine out)")
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling cases)")
    ap.add_argument("--experts", type=int, default=None, help="override E (profiling cases)")
    return ap.parse_args()


def workload(name, tokens=None, experts=None):
    import dataclasses
    import synth
    s = {"prefill-fp8": synth.PREFILL_FP8, "decode-bf16": synth.DECODE_BF16,
         "long-skew-fp8": synth.LONG_SKEW_FP8, "dense-ffn-fp8": synth.DENSE_FFN_FP8, "nvfp4": synth.STEP5_NVFP4}[name]
    if experts is not None:
        s = dataclasses.replace(s, n_experts=experts, name=f"{s.name}-E{experts}")
    if tokens is not None:
        s = s.with_tokens(tokens)
    return s


STORAGE = {0: "BF16", 1: "FP8 E4M3 128x128 weights, 1x128 activations",
           2: "NVFP4 weights (E2M1, E4M3 per 16, fp32 global), bf16 activations"}


def describe(shape) -> dict:
    return {"workload": f"{shape.name}: T={shape.T} H={shape.hidden} E={shape.n_experts} top-{shape.top_k} "
                        f"shared={shape.n_shared} I={shape.inter} "
                        f"{STORAGE[shape.wdtype]}"
                        f"{', Zipf-skewed routing' if shape.skew else ', uniform routing'}",
            "tokens": shape.T, "hidden": shape.hidden, "experts": shape.n_experts, "top_k": shape.top_k,
            "shared_experts": shape.n_shared, "inter": shape.inter, "seed": shape.seed,
            "l2": "flushed between timed steps (256 MB write)"}


def peaks():
    p = dict(FALLBACK_PEAKS)
    src = "fallback"
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            d = json.load(open(path))
            p["hbm_gbs"] = float(d["hbm_gbs"])
            p["bf16_tflops"] = float(d["bf16_tflops"])
            src = "measured"
        except Exception:
            pass
    p["fp8_tflops"] = 2.0 * p["bf16_tflops"]  # nominal FP8:BF16 dense ratio 2
    p["source"] = src
    return p


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi clock/throttle sampling while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"moe_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        loaded = [s for s, p in zip(sm, power) if p > 250.0] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded)}


# ------------------------------------------------------------ replicas ----

def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's value (device time of the same timed region).

    Every rank calls this the same number of times, in the same order; with one
    rank it returns `value` unchanged.
    """
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, world: int, steps: int, max_total_ms: float) -> float:
    """Whole-job tokens/s of `world` independent replicas: all ranks' tokens over
    the slowest rank's time for the same `steps`."""
    return world * tokens_per_rank * steps / (max_total_ms / 1e3)


# --------------------------------------------------------------- our arm ----

def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    import synth
    import mixture_experts_histogram_b200 as m
    from mixture_experts_histogram_b200 import build as mbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        mbuild.build()
    if world > 1:
        dist.barrier()
    m.load()
    shape = workload(args.workload, args.tokens, args.experts)
    x_np = synth.make_x(shape)
    w_np = synth.make_weights(shape)
    wd = m.upload_weights(w_np, f"cuda:{local}")
    wts = m.make_weights(wd)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=f"cuda:{local}")
    stream = torch.cuda.current_stream()

    def measure(T, x_host, profile=True, shape=shape, wts=wts):
        cfg = m.make_config(shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
        x = m.to_device(x_host, f"cuda:{local}")
        out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device=f"cuda:{local}")
        idx = torch.empty((T, shape.top_k), dtype=torch.int32, device=f"cuda:{local}")
        gate = torch.empty((T, shape.top_k), dtype=torch.float32, device=f"cuda:{local}")
        ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device=f"cuda:{local}")

        def step():
            m.moe_forward(cfg, T, x, wts, out, ws, topk_idx=idx, topk_w=gate, stream=stream)

        for _ in range(args.warmup):
            flush.fill_(1)
            step()
        st = m.moe_read_status(ws)
        if st != 0:
            raise RuntimeError(f"device status after warm-up: {m.moe_status_string(st)}")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        per_kernel = {k: 0.0 for k in KERNELS}
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        launches0 = m.moe_launch_count()
        # Timed steps: no per-kernel events inside. Before each step ~1 ms of GPU
        # sleep (outside ev0..ev1) lets the host queue the whole step, so the
        # device time is not stretched by host launch gaps.
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            torch.cuda._sleep(2000000)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        launches = m.moe_launch_count() - launches0
        if world > 1:
            dist.barrier()
        total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, f"cuda:{local}")
        if profile:
            # Per-kernel split from a separate pass with an event between kernels.
            m.moe_profile_enable(True)
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                torch.cuda._sleep(2000000)
                step()
                for k, v in m.moe_profile_read().items():
                    per_kernel[k] += v
            torch.cuda.synchronize()
            m.moe_profile_enable(False)
        st = m.moe_read_status(ws)
        if st != 0:
            raise RuntimeError(f"device status after timing: {m.moe_status_string(st)}")
        res = {"ms_per_step": total_ms / args.steps, "tokens_per_s": replica_throughput(T, world, args.steps, total_ms),
               "kernel_ms": {k: v / args.steps for k, v in per_kernel.items()},
               "idx": idx.cpu().numpy(), "launches": launches}
        return res

    def end_to_end(T, x_host, shape=shape, wts=wts):
        """The e2e figure: the layer through the host-buffer entry points. It runs
        after the T = 64 line that shares its weights: measured before it, its
        seconds of back-to-back T = 8192 steps left that line about 7% slow (0.966
        against 0.901 ms per layer, the kernels' own times unchanged)."""
        cfg = m.make_config(shape.hidden, shape.n_experts, shape.top_k, shape.n_shared, shape.inter, shape.wdtype)
        ws = torch.empty(m.moe_workspace_bytes(cfg, T), dtype=torch.uint8, device=f"cuda:{local}")
        res = {}
        # End to end through the host-buffer entry points: every step copies
        # its x in from pinned host memory and its output back out.
        xh = torch.from_numpy(np.ascontiguousarray(x_host).view(np.int16)).pin_memory()
        oh = [torch.empty((T, shape.hidden), dtype=torch.int16).pin_memory() for _ in range(2)]
        for _ in range(2):
            m.moe_forward_host(cfg, T, xh, wts, oh[0], ws, stream=stream)
        # (a) one step at a time (moe_forward_host: copy in, layer, copy out, sync).
        ms = []
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            m.moe_forward_host(cfg, T, xh, wts, oh[0], ws, stream=stream)
            ms.append((time.perf_counter() - t0) * 1e3)
        serial_ms = max_over_ranks(sum(ms), world, f"cuda:{local}")
        # (b) steps pipelined over two streams and two workspaces
        # (moe_forward_host_async): one step's copies overlap the other's kernels.
        ws2 = torch.empty_like(ws)
        streams = [stream, torch.cuda.Stream(device=f"cuda:{local}")]
        wss = [ws, ws2]
        for i in range(4):
            m.moe_forward_host_async(cfg, T, xh, wts, oh[i % 2], wss[i % 2], stream=streams[i % 2])
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for i in range(args.steps):
            m.moe_forward_host_async(cfg, T, xh, wts, oh[i % 2], wss[i % 2], stream=streams[i % 2])
        torch.cuda.synchronize()
        pipe_ms = max_over_ranks((time.perf_counter() - t0) * 1e3, world, f"cuda:{local}")
        for wsx in wss:
            st = m.moe_read_status(wsx)
            if st != 0:
                raise RuntimeError(f"device status after the host-buffer steps: {m.moe_status_string(st)}")
        del ws2
        res["e2e"] = {"value": replica_throughput(T, world, args.steps, pipe_ms), "unit": "tokens/s",
                      "h2d_bytes_per_step": T * shape.hidden * 2, "d2h_bytes_per_step": T * shape.hidden * 2,
                      "how": "moe_forward_host_async, steps alternating two streams and workspaces, "
                             "host wall clock from the first copy in to the last copy out",
                      "serial_value": replica_throughput(T, world, args.steps, serial_ms),
                      "serial_how": "moe_forward_host, one synchronous step at a time, L2 flushed between"}
        return res

    pk = peaks()
    with ClockSampler(local) as clk:
        main = measure(shape.T, x_np)
        decode = None
        if not args.no_decode and shape.wdtype == synth.WDTYPE_FP8 and shape.T != 64:
            dshape = shape.with_tokens(64)
            decode = measure(64, synth.make_x(dshape))
        if not args.no_e2e:
            main.update(end_to_end(shape.T, x_np))
    decode_bf16 = None
    if not args.no_decode and shape.wdtype == synth.WDTYPE_FP8 and args.workload == "prefill-fp8":
        # The BF16 decode workload (its own seed and BF16 weights).
        wd = wts = None
        torch.cuda.empty_cache()
        bshape = synth.DECODE_BF16
        bw = m.upload_weights(synth.make_weights(bshape), f"cuda:{local}")
        with ClockSampler(local):
            decode_bf16 = (bshape, measure(bshape.T, synth.make_x(bshape), shape=bshape,
                                           wts=m.make_weights(bw)))
        del bw
    extra = {}
    if not args.no_extra and args.workload == "prefill-fp8" and args.tokens is None and args.experts is None:
        # The long skewed prefill and the FP8 decode sweep, each on its own
        # seeded weights (freed between workloads).
        for key, wshape, tokens in (("long_skew_t32768", synth.LONG_SKEW_FP8, [synth.LONG_SKEW_FP8.T]),
                                    ("decode_sweep_fp8", synth.SWEEP_FP8, list(synth.SWEEP_TOKENS)),
                                    ("nvfp4_w4a16", synth.STEP5_NVFP4, [64, 8192]),
                                    ("dense_ffn_fp8", synth.DENSE_FFN_FP8, [64, 8192])):
            wd = wts = None
            torch.cuda.empty_cache()
            ew = m.upload_weights(synth.make_weights(wshape), f"cuda:{local}")
            ewts = m.make_weights(ew)
            with ClockSampler(local) as eclk:
                runs = [(T, measure(T, synth.make_x(wshape.with_tokens(T)), shape=wshape.with_tokens(T),
                                    wts=ewts)) for T in tokens]
            extra[key] = (wshape, runs, eclk.summary())
            del ew, ewts
    clocks = clk.summary()

    def roofline(res, T, shape=shape):
        """The dominant kernel against its bound (HBM bytes or tensor FLOPs)."""
        idx = res["idx"]
        touched = int(np.unique(idx).size)
        fp8 = shape.wdtype == synth.WDTYPE_FP8
        es = 1 if fp8 else 2  # activation bytes (x, h); NVFP4 keeps bf16 activations
        H, I, E, k, S = shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared
        R = (k + S) * T
        groups = touched + S

        def wbytes(rows, cols):
            """Stored bytes of one expert matrix [rows, cols], scales included."""
            if fp8:
                return rows * cols + (rows // 128) * (cols // 128) * 4
            if shape.wdtype == synth.WDTYPE_NVFP4:
                return rows * cols // 2 + rows * cols // 16 + 4
            return rows * cols * 2

        kern = {
            "gemm1_gate_up_swiglu": {
                "bytes": groups * 2 * wbytes(I, H) + T * H * es + R * I * es,
                "flops": 2.0 * R * H * 2 * I},
            "gemm2_down": {"bytes": groups * wbytes(H, I) + R * I * es + R * H * 2,
                           "flops": 2.0 * R * I * H},
        }
        for kk, v in kern.items():
            kms = res["kernel_ms"].get(kk, 0.0)
            if kms > 0:
                v["ms"] = round(kms, 4)
                v["hbm_gbs"] = round(v["bytes"] / (kms / 1e3) / 1e9, 1)
                v["hbm_frac"] = round(v["hbm_gbs"] / pk["hbm_gbs"], 4)
                v["tflops"] = round(v["flops"] / (kms / 1e3) / 1e12, 1)
                v["tensor_frac"] = round(v["tflops"] / (pk["fp8_tflops"] if fp8 else pk["bf16_tflops"]), 4)
        dom = max(kern, key=lambda kk: res["kernel_ms"].get(kk, 0.0))
        ms = res["kernel_ms"][dom]
        t_hbm = kern[dom]["bytes"] / (pk["hbm_gbs"] * 1e9)
        peak_tf = pk["fp8_tflops"] if fp8 else pk["bf16_tflops"]  # NVFP4 runs bf16 MMAs
        t_tc = kern[dom]["flops"] / (peak_tf * 1e12)
        traffic = traffic_for(dom, shape.name if T == shape.T else f"{shape.name}@T={T}")
        if t_hbm >= t_tc:
            ach = kern[dom]["bytes"] / (ms / 1e3) / 1e9
            r = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s"}
        else:
            ach = kern[dom]["flops"] / (ms / 1e3) / 1e12
            r = {"bound": "tensor", "achieved": round(ach, 1), "peak": peak_tf, "unit": "TFLOP/s"}
        r.update({"frac": round(ach / r["peak"], 4), "traffic": traffic, "kernel": dom,
                  "kernel_ms": round(ms, 4), "algorithmic_bytes": kern[dom]["bytes"],
                  "algorithmic_flops": kern[dom]["flops"], "touched_experts": touched,
                  "peak_source": f"{pk['source']} (MEASURED_PEAKS.json; FP8 = 2 x measured BF16)"})
        # Whole layer against max(compute, bytes): weights of touched experts + router + x + out.
        lay_bytes = groups * (2 * wbytes(I, H) + wbytes(H, I)) + E * H * 2 + 2 * T * H * 2
        lay_flops = 2.0 * T * H * E + 2.0 * 3 * H * I * R
        t_roof = max(lay_bytes / (pk["hbm_gbs"] * 1e9), lay_flops / (peak_tf * 1e12))
        layer = {"ms": round(res["ms_per_step"], 4), "roofline_ms": round(t_roof * 1e3, 4),
                 "expert_gemms": {kk: {q: v[q] for q in ("ms", "hbm_gbs", "hbm_frac", "tflops", "tensor_frac")
                                       if q in v} for kk, v in kern.items()},
                 "frac": round(t_roof * 1e3 / res["ms_per_step"], 4),
                 "tflops": round(lay_flops / (res["ms_per_step"] / 1e3) / 1e12, 1),
                 "hbm_gbs_of_algorithmic_bytes": round(lay_bytes / (res["ms_per_step"] / 1e3) / 1e9, 1)}
        return r, layer

    roof, layer = roofline(main, shape.T)
    line = {
        "metric": METRIC, "value": round(main["tokens_per_s"], 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(main["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {0: "bf16", 1: "e4m3", 2: "nvfp4 weights, bf16 activations"}[shape.wdtype],
        "data": "synthetic (seeded, counter-based generator)",
        "config": dict(describe(shape), parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        "roofline": roof, "layer_roofline": layer,
        "kernel_ms": {k: round(v, 4) for k, v in main["kernel_ms"].items()},
        "e2e": main.get("e2e"), "gpu_launches": main["launches"], "clocks": clocks,
    }
    if decode is not None:
        droof, dlayer = roofline(decode, 64)
        line["decode_t64"] = {"value": round(decode["tokens_per_s"], 1), "unit": "tokens/s",
                              "ms_per_step": round(decode["ms_per_step"], 4), "roofline": droof,
                              "layer_roofline": dlayer,
                              "kernel_ms": {k: round(v, 4) for k, v in decode["kernel_ms"].items()},
                              "config": "T=64, same layer and weights as the headline workload"}
    if decode_bf16 is not None:
        bshape, bres = decode_bf16
        broof, blayer = roofline(bres, bshape.T, shape=bshape)
        line["decode_bf16_t64"] = {"value": round(bres["tokens_per_s"], 1), "unit": "tokens/s",
                                   "ms_per_step": round(bres["ms_per_step"], 4), "roofline": broof,
                                   "layer_roofline": blayer,
                                   "kernel_ms": {k: round(v, 4) for k, v in bres["kernel_ms"].items()},
                                   "config": describe(bshape)}
    for key, (wshape, runs, eclk) in extra.items():
        sub = {}
        for T, res in runs:
            r_, l_ = roofline(res, T, shape=wshape.with_tokens(T))
            counts = np.bincount(res["idx"].reshape(-1), minlength=wshape.n_experts)
            sub[f"T={T}"] = {"value": round(res["tokens_per_s"], 1), "unit": "tokens/s",
                             "ms_per_step": round(res["ms_per_step"], 4), "roofline": r_, "layer_roofline": l_,
                             "kernel_ms": {k: round(v, 4) for k, v in res["kernel_ms"].items()},
                             "routed_rows_per_expert": {"hottest": int(counts.max()),
                                                        "mean": round(float(counts.mean()), 1),
                                                        "hottest_over_mean": round(float(counts.max() / counts.mean()), 2)},
                             "gpu_launches": res["launches"]}
        line[key] = {"config": describe(wshape), "tokens": [T for T, _ in runs], "clocks": eclk, **sub}
    if args.residual:
        line["residual_stream"] = time_residual(m, shape, args, pk, local, flush)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape, x_np, w_np)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def time_residual(m, shape, args, pk, local, flush):
    """moe_rmsnorm and moe_combine_residual at the workload's T, against measured HBM.

    Algorithmic bytes: RMSNorm reads r (4TH) and w (4H), writes x (2TH); the
    residual combine reads the (k+S)T expert rows (2H each) and r, writes r_out.
    """
    import numpy as np
    import torch
    T, H, k, S = shape.T, shape.hidden, shape.top_k, shape.n_shared
    dev = f"cuda:{local}"
    g = torch.Generator(device=dev).manual_seed(shape.seed)
    r = torch.randn((T, H), generator=g, device=dev, dtype=torch.float32)
    w = torch.ones(H, device=dev, dtype=torch.float32)
    x = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    rows = (k + S) * T
    y = torch.randn((rows, H), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    pos = torch.randperm(rows, generator=g, device=dev).to(torch.int32).view(T, k + S)
    r_out = torch.empty_like(r)
    cfg = m.make_config(H, shape.n_experts, k, S, shape.inter, shape.wdtype)
    res = {}
    for name, fn, nbytes in (
            ("rmsnorm", lambda: m.moe_rmsnorm(T, H, r, w, 1e-6, x), 4 * T * H + 4 * H + 2 * T * H),
            ("combine_residual", lambda: m.moe_combine_residual(cfg, T, y, pos, r, r_out),
             2 * rows * H + 4 * T * H + 4 * T * H)):
        for _ in range(max(args.warmup, 3)):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
        gbs = nbytes / (ms / 1e3) / 1e9
        res[name] = {"ms": round(ms, 4), "algorithmic_bytes": nbytes, "achieved_gbs": round(gbs, 1),
                     "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4)}
    return res


def traffic_for(kernel: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        d = json.load(open(path))
        ent = d.get(kernel, {}).get(workload_name)
        if not ent or ent.get("source_sha") != kernel_source_sha():
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


# Sources that build the grouped expert GEMMs and their launch (tensor maps,
# variant choice): the files a traffic figure for those kernels depends on.
GEMM_SOURCES = ("grouped_gemm.cu", "grouped_gemm_swap.cu", "nvfp4_gemm.cu", "nvfp4_gemm_swap.cu", "gemm_common.cuh",
                "ptx.cuh", "common.cuh", "abi.cu")


def kernel_source_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixture_experts_histogram_b200", "csrc")
    for f in GEMM_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


# --------------------------------------------------------- CPU oracle arm ----

def _oracle_sample(shape, x_np, w_np, n_tok):
    import oracle
    t0 = time.perf_counter()
    xs = x_np[:n_tok]
    idx, gate, _ = oracle.route(xs, w_np["router_w"], w_np["router_bias"], shape.top_k)
    oracle.moe_tokens(shape.with_tokens(n_tok), w_np, xs, idx, gate)
    return time.perf_counter() - t0


def _pick_sample(shape, x_np, w_np, target_s):
    t1 = _oracle_sample(shape, x_np, w_np, 2)
    per_tok = max(t1 / 2, 1e-4)
    return int(min(max(2, target_s / per_tok), 512, shape.T))


def cpu_baseline(shape, x_np, w_np, target_s=12.0):
    """The oracle, as it stands, on all host cores, on a bounded token sample."""
    n = _pick_sample(shape, x_np, w_np, target_s)
    dt = _oracle_sample(shape, x_np, w_np, n)
    import oracle
    return {"value": round(n / dt, 3), "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {n} tokens of the workload: routing, experts and combine ({dt:.1f} s)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synth
    shape = workload(args.workload, args.tokens, args.experts)
    x_np = synth.make_x(shape)
    w_np = synth.make_weights(shape)
    steps, warm = args.steps, args.warmup
    budget = 150.0
    n = _pick_sample(shape, x_np, w_np, budget / max(1, steps + warm))
    for _ in range(min(warm, 1)):
        _oracle_sample(shape, x_np, w_np, n)
    ts = [_oracle_sample(shape, x_np, w_np, n) for _ in range(steps)]
    value = n * steps / sum(ts)
    line = {"metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": args.gpus, "steps": steps,
            "warmup": warm, "ms_per_step": round(1e3 * sum(ts) / steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 accumulation (oracle)",
            "data": "synthetic (seeded, counter-based generator)", "impl": "reference",
            "config": dict(describe(shape), parallelism="single GPU" if args.gpus <= 1 else f"replicas x{args.gpus}"),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": f"first {n} tokens of the workload per step"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse_args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
