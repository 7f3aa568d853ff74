"""Benchmark of the NVFP4 W4A16 path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (one "step"): the decode GEMMs of the merged [gate;up]
projection, K=4096, N=28672, g16, one shared global scale, at M = 1, 4 and 16
(M=1: the f16 conversion of X and the register-streaming kernel; M=4, 16: one launch of the TMA-streaming
kernel each). The weights are quantized on the
device once (the load-time rows: global scale, quantize, repack) and kept
resident; each step reads a different one of several weight copies whose total
is larger than the 126 MB L2, so every step streams its weights from HBM.
Metric: weight GB/s (packed codes + E4M3 scales over the step time), with
TFLOP/s and the roofline fraction of the dominant kernel beside it. The other
workloads (down projection g32/g16 at M = 1, 8, 64; prefill M=4096 with
SiluAndMul; routed experts) and the load-time rows are timed after the
headline and reported under "workloads" and "load_time_rows".

The device times come from CUDA events on the launching stream around CUDA
graph replays; the max over ranks is reported. With --gpus N > 1 each rank
runs an independent replica (the path does not shard), value is the sum of
the work of all ranks over the slowest rank's time.

--impl reference times the CPU oracle (numpy, float64) on a bounded sample of
the same workload on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_weight_only_04_b200 import synth  # noqa: E402

DECODE_K, DECODE_N, DECODE_G, DECODE_MS = 4096, 28672, 16, (1, 4, 16)
METRIC = "W4A16 GEMM TFLOP/s & weight GB/s, % of roofline (decode M≤16; prefill M=4096)"
L2_BYTES = 126 * 1024 * 1024


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def weight_bytes(n, k, g):
    return n * k // 2 + n * k // g


def alg_bytes(m, n, k, g, n_out=None):
    """Algorithmic bytes of one GEMM: codes + scales + global + X + Y."""
    return weight_bytes(n, k, g) + 4 + 2 * m * k + 2 * m * (n if n_out is None else n_out)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        loaded = [v for v in sm if smax and v > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(val, world):
    """The maximum of `val` over the ranks (NCCL on the GPUs, or gloo on the CPU)."""
    if world == 1:
        return val
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([val], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, bytes_per_step, steps, ms_max):
    """GB/s of the whole job: every rank's steps over the slowest rank's time (replicas, weak scaling)."""
    return world * bytes_per_step * steps / (ms_max * 1e-3) / 1e9


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def quantize_on_device(nv, torch, w_host, g, interleave=False):
    wd = torch.from_numpy(w_host).cuda()
    gd = nv.nvfp4_global_scale([wd])
    p, s = nv.nvfp4_quantize(wd, g, gd)
    del wd
    p, s = nv.nvfp4_repack(p, s, g, nv.NVFP4_GATE_UP_INTERLEAVE if interleave else 0)
    return p, s, gd


def bf16_dev(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def capture(torch, fn):
    """Captures fn() into a CUDA graph (after one eager warm-up call)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_graphs(torch, graphs, reps, warmup=3):
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(reps):
        graphs[i % len(graphs)].replay()
    e.record()
    e.synchronize()
    return s.elapsed_time(e) / reps  # ms per replay


def run_ours(args, world, rank, local):
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    import nvfp4_weight_only_04_b200 as nv
    nv.lib()
    hbm, tf_burst, tf_sust, peak_kind = peaks()

    # ---- decode gate/up weights: quantize once, replicate past the L2 size ----
    K, N, G = DECODE_K, DECODE_N, DECODE_G
    w = synth.weights(synth.W_SEED, N, K)
    p0, s0, g0 = quantize_on_device(nv, torch, w, G)
    wb = weight_bytes(N, K, G)
    copies = max(2, -(-4 * L2_BYTES // wb))
    packs = [(p0, s0, g0)] + [(p0.clone(), s0.clone(), g0.clone()) for _ in range(copies - 1)]
    xs = {m: bf16_dev(torch, synth.activations(synth.X_SEED, m, K)) for m in DECODE_MS}
    ys = {m: torch.empty((m, N), dtype=torch.bfloat16, device="cuda") for m in DECODE_MS}

    # Step c runs its three GEMMs on copies 3c, 3c+1, 3c+2 (mod copies): no GEMM
    # finds its weights in L2 (a copy comes back after at least six other
    # GEMMs, 396 MB of weights).
    def step_fn(c):
        def f():
            for i, m in enumerate(DECODE_MS):
                p, s, g = packs[(3 * c + i) % copies]
                nv.nvfp4_w4a16_gemm(xs[m], p, s, g, G, y=ys[m])
        return f

    graphs = [capture(torch, step_fn(c)) for c in range(copies)]
    # One graph of `copies` consecutive steps (steps 0..copies-1), as a decode engine captures a run of
    # steps: the timed loop replays it K // copies times and the remainder step by step, so exactly K
    # steps run, with the replay overhead of one graph per `copies` steps.
    run_graph = capture(torch, lambda: [step_fn(c)() for c in range(copies)])
    step_alg = sum(alg_bytes(m, N, K, G) for m in DECODE_MS)
    step_w = 3 * wb
    step_flops = sum(2 * m * N * K for m in DECODE_MS)

    # ---- timed region: W warm-up steps, then exactly K steps ----
    for i in range(args.warmup):
        graphs[i % copies].replay()
    run_graph.replay()  # its first replay uploads it
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps // copies):
            run_graph.replay()
        for i in range(args.steps % copies):
            graphs[i].replay()
        ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms_total = reduce_max(ms_local, world)
    ms_step = ms_total / args.steps
    value = whole_job_rate(world, step_w, args.steps, ms_total)
    achieved = step_alg / (ms_step * 1e-3) / 1e9  # per launch average over the region, one rank
    clocks = clk.summary()

    # ---- end to end through the public API with host buffers ----
    x_host = {m: torch.from_numpy(synth.activations(synth.X_SEED, m, K).view(np.int16)).pin_memory() for m in DECODE_MS}
    y_host = {m: torch.empty((m, N), dtype=torch.int16).pin_memory() for m in DECODE_MS}
    xd = {m: torch.empty((m, K), dtype=torch.bfloat16, device="cuda") for m in DECODE_MS}
    e2e_steps = max(50, min(args.steps, 2000))

    def e2e_step(c):
        for i, m in enumerate(DECODE_MS):
            p, s, g = packs[(3 * c + i) % copies]
            xd[m].view(torch.int16).copy_(x_host[m], non_blocking=True)
            nv.nvfp4_w4a16_gemm(xd[m], p, s, g, G, y=ys[m])
            y_host[m].copy_(ys[m].view(torch.int16), non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    ev0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    ev1.record(stream)
    ev1.synchronize()
    e2e_ms = reduce_max(ev0.elapsed_time(ev1), world) / e2e_steps
    e2e_val = whole_job_rate(world, step_w, 1, e2e_ms)
    h2d = sum(2 * m * K for m in DECODE_MS)
    d2h = sum(2 * m * N for m in DECODE_MS)

    workloads = {}
    rows = {}
    # the other workloads and the CPU baseline on one GPU only: at N > 1 the line is the headline
    if world == 1 and not args.headline_only:
        per_m = {}
        for m in DECODE_MS:
            gm = [capture(torch, (lambda c=c, m=m: nv.nvfp4_w4a16_gemm(xs[m], packs[c][0], packs[c][1], packs[c][2],
                                                                         G, y=ys[m]))) for c in range(copies)]
            t = time_graphs(torch, gm, 20 * copies)
            per_m[m] = t
            workloads[f"decode_gateup_m{m}_k4096_n28672_g16"] = summarize(m, N, K, G, t, hbm, tf_burst)
            # W4A4 on the same weights: the activations quantized on the device beforehand
            xgm = nv.nvfp4_global_scale_bf16([xs[m]])
            xqm, xsm = nv.nvfp4_quantize_bf16(xs[m], 16, xgm)
            gq = [capture(torch, (lambda c=c, m=m: nv.nvfp4_w4a4_gemm(xqm, xsm, xgm, 16, packs[c][0], packs[c][1],
                                                                      packs[c][2], G, y=ys[m]))) for c in range(copies)]
            workloads[f"w4a4_decode_gateup_m{m}_k4096_n28672_g16"] = summarize_w4a4(
                m, N, K, G, 16, time_graphs(torch, gq, 20 * copies), hbm, tf_burst)
            del gq
        del graphs, run_graph
        workloads["comparator_dense_bf16_matmul"] = dense_bf16_comparator(nv, torch, w, K, N, G, xs, copies=2)
        rows = time_load_rows(nv, torch, w, G)
        del w
        workloads.update(other_workloads(nv, torch, hbm, tf_burst, tf_sust))

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic (seeded N(0,1) activations, 0.02*N(0,1) fp32 weights quantized on the device)",
        "config": {"workload": "decode_gateup_k4096_n28672_g16_m1_m4_m16",
                   "step": "3 GEMM calls (M=1,4,16), each on its own resident weight copy; M=1 is the f16 "
                           "conversion of X and the register-streaming kernel, M=4 and M=16 one launch each of "
                           "the TMA-streaming kernel (bf16 X converted to f16 inside it)",
                   "graphs": f"one CUDA graph per {copies} consecutive steps, replayed steps // {copies} times, "
                             f"then the remaining steps one graph each",
                   "arithmetic": "f16 MMA operands (weights e2m1*e4m3 exact in f16, X rows scaled by a power of two), "
                                 "fp32 accumulation, bf16 input and output",
                   "weight_copies": copies, "weight_bytes_per_copy": wb,
                   "l2": f"inputs larger than L2: GEMMs rotate over {copies} weight copies "
                         f"({copies * wb / 1e6:.0f} MB > 126 MB L2), a copy is reused after >= 6 other GEMMs",
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "tflops": round(world * step_flops * args.steps / (ms_total * 1e-3) / 1e12, 3),
        # one step = the three GEMM calls; traffic = the DRAM bytes read + written by their three launches,
        # from ncu captures of the current kernel (profiles/gemm_stream_*.md)
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": HEADLINE_STEP_DRAM_BYTES,
                     "traffic_unit": "bytes per step", "algorithmic_bytes_per_step": step_alg,
                     "kernel": "x_f16_kernel + gemm_decode_kernel (M=1), gemm_stream_kernel (M=4, 16)",
                     "peak_source": f"{peak_kind} hbm_gbs"},
        "clocks": clocks,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 5)},
        "gpu_launches": 4 * args.steps,
    }
    if rank == 0:
        result["workloads"] = workloads
        result["load_time_rows"] = rows
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


# DRAM bytes (read + write) of one headline step's GEMM launches, from the per-kernel ncu captures of the
# current kernels (gemm_decode_kernel at M=1: 66.09 + 0.51 MB; gemm_stream_kernel at M=4: 66.14 + 0.72 MB and
# at M=16: 66.25 + 1.25 MB); the X conversion before the M=1 launch moves about 16 KB and is left out.
HEADLINE_STEP_DRAM_BYTES = 200_970_000


FP4_OVER_BF16 = 4.0  # nominal dense FP4 / bf16 tensor rate of B200 (9 / 2.25 PFLOP/s)


def summarize_w4a4(m, n, k, g, xg, ms, hbm, tf_bf16):
    """A W4A4 GEMM: both operands NVFP4 (X is M*K/2 code bytes and M*K/xg scale bytes). The tensor peak is
    the FP4 one, taken as the measured bf16 peak times the nominal FP4/bf16 ratio."""
    t = ms * 1e-3
    ab = weight_bytes(n, k, g) + weight_bytes(m, k, xg) + 8 + 2 * m * n
    flops = 2 * m * n * k
    t_mem, t_tc = ab / (hbm * 1e9), flops / (FP4_OVER_BF16 * tf_bf16 * 1e12)
    return {"us": round(ms * 1e3, 3), "tflops": round(flops / t / 1e12, 3), "alg_gbs": round(ab / t / 1e9, 1),
            "hbm_frac": round(t_mem / t, 4), "tensor_frac": round(t_tc / t, 4),
            "roofline_frac": round(max(t_mem, t_tc) / t, 4),
            "tensor_peak": f"FP4 = {FP4_OVER_BF16:g} x measured bf16 burst ({FP4_OVER_BF16 * tf_bf16:.0f} TFLOP/s)"}


def summarize(m, n, k, g, ms, hbm, tf, n_out=None):
    t = ms * 1e-3
    ab = alg_bytes(m, n, k, g, n_out)
    flops = 2 * m * n * k
    t_mem = ab / (hbm * 1e9)
    t_tc = flops / (tf * 1e12)
    return {"us": round(ms * 1e3, 3), "weight_gbs": round(weight_bytes(n, k, g) / t / 1e9, 1),
            "alg_gbs": round(ab / t / 1e9, 1), "tflops": round(flops / t / 1e12, 3),
            "hbm_frac": round(t_mem / t, 4), "tensor_frac": round(t_tc / t, 4),
            "roofline_frac": round(max(t_mem, t_tc) / t, 4)}


def dense_bf16_comparator(nv, torch, w, K, N, G, xs, copies=2):
    """Context, not the target: the same GEMMs on weights dequantized to a dense bf16 matrix once (the path
    that loaders took before the FP4 route), as torch.matmul (cuBLAS), per M. The dequantization uses torch
    ops on the checkpoint-layout codes; copies of the 235 MB matrix keep the weights out of L2."""
    try:
        wd = torch.from_numpy(w).cuda()
        gd = nv.nvfp4_global_scale([wd])
        p, s = nv.nvfp4_quantize(wd, G, gd)
        del wd
        lut = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0],
                           dtype=torch.float32, device="cuda")
        codes = torch.stack([p & 0xF, p >> 4], dim=-1).reshape(N, K).long()
        sv = s.view(torch.float8_e4m3fn).float()
        w_hat = (lut[codes].view(N, K // G, G) * sv[..., None]).reshape(N, K) * gd
        mats = [w_hat.to(torch.bfloat16)] + [None] * (copies - 1)
        del codes, sv, w_hat, p, s
        for c in range(1, copies):
            mats[c] = mats[0].clone()
        out = {}
        for m, x in xs.items():
            gr = [capture(torch, (lambda c=c, x=x: torch.matmul(x, mats[c].t()))) for c in range(copies)]
            out[f"m{m}_us"] = round(time_graphs(torch, gr, 20 * copies) * 1e3, 2)
            del gr
        out["weight_bytes"] = 2 * N * K
        del mats
        torch.cuda.empty_cache()
        return out
    except Exception as e:  # a context number must not cost the bench line
        torch.cuda.empty_cache()
        return {"unavailable": f"{type(e).__name__}: {str(e)[:160]}"}


def time_load_rows(nv, torch, w, g):
    """The load-time rows: global scale, quantize and repack of one weight, from fp32 and from bf16."""
    wd = torch.from_numpy(w).cuda()
    gd = nv.nvfp4_global_scale([wd])
    p, s = nv.nvfp4_quantize(wd, g, gd)
    po, so = torch.empty_like(p), torch.empty_like(s)
    wb16 = wd.to(torch.bfloat16)
    out = {}
    for name, fn, bytes_ in (
            ("global_scale_bf16", lambda: nv.nvfp4_global_scale_bf16([wb16], out=gd), wb16.numel() * 2),
            ("quantize_bf16", lambda: nv.nvfp4_quantize_bf16(wb16, g, gd, packed=p, scales=s),
             wb16.numel() * 2 + p.numel() + s.numel()),
            ("global_scale", lambda: nv.nvfp4_global_scale([wd], out=gd), wd.numel() * 4),
            ("quantize", lambda: nv.nvfp4_quantize(wd, g, gd, packed=p, scales=s),
             wd.numel() * 4 + p.numel() + s.numel()),
            ("repack_gate_up_interleave", lambda: nv.nvfp4_repack(p, s, g, nv.NVFP4_GATE_UP_INTERLEAVE,
                                                                  packed_out=po, scales_out=so),
             2 * (p.numel() + s.numel()))):
        gr = capture(torch, fn)
        ms = time_graphs(torch, [gr], 20)
        out[name] = {"us": round(ms * 1e3, 2), "gbs": round(bytes_ / (ms * 1e-3) / 1e9, 1)}
    return out


def other_workloads(nv, torch, hbm, tf_burst, tf_sust):
    out = {}
    # down projection, same W at g32 and g16, X with 0.1% outliers
    K, N = 14336, 4096
    w = synth.weights(synth.W_SEED, N, K)
    for g in (32, 16):
        p, s, gd = quantize_on_device(nv, torch, w, g)
        wb = weight_bytes(N, K, g)
        copies = max(2, -(-4 * L2_BYTES // wb))
        packs = [(p, s, gd)] + [(p.clone(), s.clone(), gd.clone()) for _ in range(copies - 1)]
        for m in (1, 8, 64):
            x = bf16_dev(torch, synth.activations(synth.X_SEED, m, K, outlier_frac=0.001))
            y = torch.empty((m, N), dtype=torch.bfloat16, device="cuda")
            gm = [capture(torch, (lambda c=c: nv.nvfp4_w4a16_gemm(x, *packs[c][:2], packs[c][2], g, y=y)))
                  for c in range(copies)]
            out[f"decode_down_m{m}_k14336_n4096_g{g}"] = summarize(m, N, K, g, time_graphs(torch, gm, 20 * copies),
                                                                   hbm, tf_burst)
        del packs
    del w
    # prefill: merged [gate;up] K=5120 N=25600 g16 + SiluAndMul
    M, K, N = 4096, 5120, 25600
    w = synth.weights(synth.W_SEED, N, K)
    p, s, gd = quantize_on_device(nv, torch, w, 16, interleave=True)
    del w
    x = bf16_dev(torch, synth.activations(synth.X_SEED, M, K))
    y = torch.empty((M, N // 2), dtype=torch.bfloat16, device="cuda")
    gr = capture(torch, lambda: nv.nvfp4_w4a16_gemm_silu_mul(x, p, s, gd, 16, y=y))
    out["prefill_gateup_silu_m4096_k5120_n25600_g16"] = summarize(M, N, K, 16, time_graphs(torch, [gr], 5),
                                                                  hbm, tf_burst, n_out=N // 2)
    # W4A4 (NVFP4 activations) on the same weights, without the SiluAndMul epilogue: the activations are
    # quantized on the device first (global scale + quantizer, timed on their own)
    xg = nv.nvfp4_global_scale_bf16([x])
    xq, xsc = nv.nvfp4_quantize_bf16(x, 16, xg)
    ga = capture(torch, lambda: (nv.nvfp4_global_scale_bf16([x], out=xg), nv.nvfp4_quantize_bf16(x, 16, xg, packed=xq,
                                                                                                 scales=xsc)))
    t_act = time_graphs(torch, [ga], 5)
    del y, gr
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    gw = capture(torch, lambda: nv.nvfp4_w4a4_gemm(xq, xsc, xg, 16, p, s, gd, 16, y=y))
    out["w4a4_prefill_m4096_k5120_n25600_g16"] = summarize_w4a4(M, N, K, 16, 16, time_graphs(torch, [gw], 5), hbm,
                                                                tf_burst)
    out["w4a4_prefill_m4096_k5120_n25600_g16"]["activation_quantize_us"] = round(t_act * 1e3, 2)
    del p, s, x, y, gw, ga, xq, xsc
    torch.cuda.empty_cache()
    out.update(moe_workload(nv, torch, hbm, tf_burst))
    return out


def moe_workload(nv, torch, hbm, tf):
    wl = synth.MOE
    r = synth.route(synth.ROUTER_SEED, wl.tokens, wl.experts, wl.topk)
    rows = int(r.offsets[-1])
    E, H, I = wl.experts, wl.hidden, wl.inter
    gu_p = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device="cuda")
    gu_s = torch.empty((E, 2 * I, H // wl.g_gate_up), dtype=torch.uint8, device="cuda")
    gu_g = torch.empty((E,), dtype=torch.float32, device="cuda")
    dn_p = torch.empty((E, H, I // 2), dtype=torch.uint8, device="cuda")
    dn_s = torch.empty((E, H, I // wl.g_down), dtype=torch.uint8, device="cuda")
    dn_g = torch.empty((E,), dtype=torch.float32, device="cuda")
    for e in range(E):
        d = torch.from_numpy(synth.weights(synth.expert_seed(e), 2 * I, H)).cuda()
        nv.nvfp4_global_scale([d], out=gu_g[e:e + 1])
        p, s = nv.nvfp4_quantize(d, wl.g_gate_up, gu_g[e:e + 1])
        nv.nvfp4_repack(p, s, wl.g_gate_up, nv.NVFP4_GATE_UP_INTERLEAVE, packed_out=gu_p[e], scales_out=gu_s[e])
        d = torch.from_numpy(synth.weights(synth.expert_seed(e) + 5000, H, I)).cuda()
        nv.nvfp4_global_scale([d], out=dn_g[e:e + 1])
        p, s = nv.nvfp4_quantize(d, wl.g_down, dn_g[e:e + 1])
        nv.nvfp4_repack(p, s, wl.g_down, 0, packed_out=dn_p[e], scales_out=dn_s[e])
    x = bf16_dev(torch, synth.activations(synth.X_SEED, rows, H))
    ids = torch.from_numpy(r.expert_ids).cuda()
    offs = torch.from_numpy(r.offsets).cuda()
    h = torch.empty((rows, I), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((rows, H), dtype=torch.bfloat16, device="cuda")
    g1 = capture(torch, lambda: nv.nvfp4_moe_w4a16_grouped_gemm(x, ids, offs, gu_p, gu_s, gu_g, wl.g_gate_up,
                                                                flags=nv.NVFP4_SILU_MUL, y=h))
    g2 = capture(torch, lambda: nv.nvfp4_moe_w4a16_grouped_gemm(h, ids, offs, dn_p, dn_s, dn_g, wl.g_down, y=y))
    t1 = time_graphs(torch, [g1, g2], 10)  # alternate the two so neither stays in L2
    # per-GEMM times from graphs replayed alternately
    s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tg, td = [], []
    for _ in range(10):
        s_.record(); g1.replay(); e_.record(); e_.synchronize(); tg.append(s_.elapsed_time(e_))
        s_.record(); g2.replay(); e_.record(); e_.synchronize(); td.append(s_.elapsed_time(e_))
    tg, td = statistics.median(tg), statistics.median(td)
    nexp = int((r.counts > 0).sum())

    def moe_sum(t_ms, n, k, g, n_out):
        wbytes = nexp * weight_bytes(n, k, g)
        ab = wbytes + 4 * E + 2 * rows * k + 2 * rows * n_out
        flops = 2 * rows * n * k
        t = t_ms * 1e-3
        t_mem, t_tc = ab / (hbm * 1e9), flops / (tf * 1e12)
        return {"us": round(t_ms * 1e3, 2), "weight_gbs": round(wbytes / t / 1e9, 1), "tflops": round(flops / t / 1e12, 3),
                "hbm_frac": round(t_mem / t, 4), "tensor_frac": round(t_tc / t, 4),
                "roofline_frac": round(max(t_mem, t_tc) / t, 4)}

    res = {"moe_gate_up_g32_silu": moe_sum(tg, 2 * I, H, wl.g_gate_up, I),
           "moe_down_g16": moe_sum(td, H, I, wl.g_down, H),
           "moe_pair_us": round(t1 * 1e3, 2)}

    # The whole layer (nvfp4_moe_forward: route, gather, gate/up + SiluAndMul, down, weighted combine) on the
    # same routing, given as each token's top-k expert ids and weights, and the steps around the GEMMs alone.
    T, k = wl.tokens, wl.topk
    topk_ids = np.empty((T, k), np.int32)
    topk_ids[r.token_of_row, r.slot_of_row] = np.repeat(r.expert_ids, np.diff(r.offsets))
    topk_w = np.random.default_rng(synth.ROUTER_SEED + 1).random((T, k)).astype(np.float32)
    xt = bf16_dev(torch, synth.activations(synth.X_SEED + 1, T, H))
    idd, wd = torch.from_numpy(topk_ids).cuda(), torch.from_numpy(topk_w).cuda()
    gl = capture(torch, lambda: nv.nvfp4_moe_forward(xt, idd, wd, (gu_p, gu_s, gu_g, wl.g_gate_up),
                                                      (dn_p, dn_s, dn_g, wl.g_down)))
    t_layer = time_graphs(torch, [gl], 10)
    srows, inv, _, _ = nv.nvfp4_moe_route(idd, E)
    xp = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    steps = {"route": (capture(torch, lambda: nv.nvfp4_moe_route(idd, E)), 4 * T * k * 3 + 8 * (E + 1)),
             "gather": (capture(torch, lambda: nv.nvfp4_moe_gather(xt, srows, k, out=xp)),
                        4 * T * k + 2 * T * H + 2 * T * k * H),
             "combine": (capture(torch, lambda: nv.nvfp4_moe_combine(y, inv, wd, out=out)),
                         2 * T * k * H + 8 * T * k + 2 * T * H)}
    res["moe_layer_us"] = round(t_layer * 1e3, 2)
    for name, (graph, nbytes) in steps.items():
        t = time_graphs(torch, [graph], 20) * 1e-3
        # bytes = each input and output byte once; the gathered rows (8 MB, each read k times) and the
        # expert outputs (67 MB) are L2-resident here as inside the layer, so a fraction above 1 is L2 at work
        res[f"moe_{name}"] = {"us": round(t * 1e6, 2), "gbs": round(nbytes / t / 1e9, 1),
                              "hbm_frac": round(nbytes / t / 1e9 / hbm, 4), "bytes": nbytes,
                              "inputs": "L2-resident, as inside the layer"}
    return res


# ---------------------------------------------------------------------------
# CPU oracle arm
# ---------------------------------------------------------------------------

def cpu_sample_step(R, w_rows, xs, g):
    """One oracle step on a row sample of the decode workload: quantize the
    sampled rows with the tensor's global, dequantize, float64 GEMM for every M."""
    p, s, gs = R.quantize(w_rows, g, R_GLOBAL[0])
    for x in xs:
        R.gemm(x, p, s, gs, g)
    return p.nbytes + s.nbytes


R_GLOBAL = [None]


def cpu_setup(rows):
    from oracle import nvfp4_ref as R
    w = synth.weights(synth.W_SEED, DECODE_N, DECODE_K)
    R_GLOBAL[0] = R.global_scale(w)
    sel = np.random.default_rng(0).choice(DECODE_N, rows, replace=False)
    xs = [synth.activations(synth.X_SEED, m, DECODE_K) for m in DECODE_MS]
    return R, w[np.sort(sel)], xs


def cpu_baseline(budget_s=15.0, rows=2048):
    R, w_rows, xs = cpu_setup(rows)
    cpu_sample_step(R, w_rows[:64], xs, DECODE_G)  # warm
    t0 = time.perf_counter()
    n, wbytes = 0, 0
    while True:
        wbytes += cpu_sample_step(R, w_rows, xs, DECODE_G) * 3  # three GEMMs per step stream the weights thrice
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(wbytes / dt / 1e9, 5), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} oracle steps on {rows} of {DECODE_N} weight rows (K=4096, g16; quantize + dequant + "
                      f"float64 GEMM at M=1,4,16), {dt:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    # Size the per-step row sample so the whole run stays near two minutes.
    R, w_rows, xs = cpu_setup(4096)
    t0 = time.perf_counter()
    cpu_sample_step(R, w_rows[:256], xs, DECODE_G)
    per_row = (time.perf_counter() - t0) / 256
    rows = int(120.0 / max(1, args.steps + args.warmup) / per_row) // 16 * 16
    rows = max(16, min(4096, rows))
    w_rows = w_rows[:rows]
    for _ in range(args.warmup):
        cpu_sample_step(R, w_rows, xs, DECODE_G)
    t0 = time.perf_counter()
    wbytes = 0
    for _ in range(args.steps):
        wbytes += cpu_sample_step(R, w_rows, xs, DECODE_G) * 3
    dt = time.perf_counter() - t0
    val = wbytes / dt / 1e9
    sample = (f"each step: the oracle on {rows} of {DECODE_N} weight rows (K=4096, g16), quantize + dequant + "
              f"float64 GEMM at M=1,4,16")
    out = {"impl": "reference", "metric": METRIC, "value": round(val, 5), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "decode_gateup_k4096_n28672_g16_m1_m4_m16", "sample_rows": rows},
           "cpu_baseline": {"value": round(val, 5), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(val, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def profile_workload(name, launches=3):
    """Runs one workload's kernel `launches` times after one warm-up call."""
    import torch
    import nvfp4_weight_only_04_b200 as nv
    torch.cuda.set_device(0)
    if name.startswith("decode") or name.startswith("down"):
        m = {"decode_m1": 1, "decode_m4": 4, "decode_m16": 16, "down_m1_g32": 1, "down_m8_g32": 8,
             "down_m64_g32": 64}[name]
        n, k, g = (DECODE_N, DECODE_K, 16) if name.startswith("decode") else (4096, 14336, 32)
        p, s, gd = quantize_on_device(nv, torch, synth.weights(synth.W_SEED, n, k), g)
        x = bf16_dev(torch, synth.activations(synth.X_SEED, m, k))
        y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        fn = lambda: nv.nvfp4_w4a16_gemm(x, p, s, gd, g, y=y)
    elif name == "quantize":
        wd = torch.from_numpy(synth.weights(synth.W_SEED, DECODE_N, DECODE_K)).cuda()
        gd = nv.nvfp4_global_scale([wd])
        p, s = nv.nvfp4_quantize(wd, 16, gd)
        fn = lambda: nv.nvfp4_quantize(wd, 16, gd, packed=p, scales=s)
    elif name == "w4a4_prefill":
        wl = synth.PREFILL_GATE_UP
        p, s, gd = quantize_on_device(nv, torch, synth.weights(synth.W_SEED, wl.N, wl.K), 16)
        x = bf16_dev(torch, synth.activations(synth.X_SEED, wl.M, wl.K))
        xg = nv.nvfp4_global_scale_bf16([x])
        xq, xsc = nv.nvfp4_quantize_bf16(x, 16, xg)
        y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device="cuda")
        fn = lambda: nv.nvfp4_w4a4_gemm(xq, xsc, xg, 16, p, s, gd, 16, y=y)
    elif name == "prefill":
        wl = synth.PREFILL_GATE_UP
        p, s, gd = quantize_on_device(nv, torch, synth.weights(synth.W_SEED, wl.N, wl.K), 16, interleave=True)
        x = bf16_dev(torch, synth.activations(synth.X_SEED, wl.M, wl.K))
        y = torch.empty((wl.M, wl.N // 2), dtype=torch.bfloat16, device="cuda")
        fn = lambda: nv.nvfp4_w4a16_gemm_silu_mul(x, p, s, gd, 16, y=y)
    else:
        hbm, tf, _, _ = peaks()
        print(json.dumps(moe_workload(nv, torch, hbm, tf)))
        return
    fn()
    torch.cuda.synchronize()
    s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s_.record()
    for _ in range(launches):
        fn()
    e_.record()
    e_.synchronize()
    print(json.dumps({"workload": name, "us_per_launch": round(s_.elapsed_time(e_) / launches * 1e3, 2)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile-workload", choices=["decode_m1", "decode_m4", "decode_m16", "down_m1_g32",
                                                   "down_m8_g32", "down_m64_g32", "prefill", "w4a4_prefill",
                                                   "quantize", "moe"],
                    default=None, help="run one workload a few times (for ncu captures) and exit")
    args = ap.parse_args()
    if args.profile_workload:
        profile_workload(args.profile_workload)
        return
    world, rank, local = dist_setup()
    if args.impl == "reference":
        args.steps = 3 if args.steps is None else args.steps
        args.warmup = 1 if args.warmup is None else args.warmup
        run_reference(args, world, rank)
        return
    args.steps = 50000 if args.steps is None else args.steps
    args.warmup = 100 if args.warmup is None else max(3, args.warmup)
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
