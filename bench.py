#!/usr/bin/env python
"""Benchmark of the W4A4 quantized linear layer on B200.

One step = one pass of the layer's hot path over one batch: online MXFP4 quantization of the
activation, then the tcgen05 block-scaled FP4 GEMM with the PRQuant tail K-extension (the two
launches replayed from a CUDA graph, as a serving loop would issue them), on the
PRQuant tail-residual workload (W [2560, 9728] -> K' = 9856, M = 2048 tokens, the prefill case).
`value` is whole-job TFLOP/s (2*M*N*K' per step over all ranks), timed with CUDA events on the
device with inputs resident; `e2e` is the same through the C ABI from pinned host buffers.
Extra cases (decode M=16, mid M=512, the single MXFP4 linear layer) are reported under "cases".

Multi-GPU: the path shards into independent replicas (no collective); each rank runs the same
workload on its own GPU and `value` sums the ranks' work over the slowest rank's time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlinear|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 linear TFLOP/s (prefill) & weight-stream GB/s (decode) vs B200 roofline"
NOMINAL_FP4_OVER_BF16 = 4.0      # 9 PFLOP/s dense FP4 / 2.25 PFLOP/s dense bf16


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------------------ workloads
def prquant_workload(M: int, seed: int = 3):
    """PRQuant tail-residual layer: W [2560, 9728] bf16 Student-t(3), k = 128 tail channels;
    X [M, 9728] N(0,1) with 0.5% outlier channels x50, permuted like the weight."""
    import synth
    import bit_quantized_moe_tcgen05_b200 as ql
    N, C, k = 2560, 9728, 128
    wb = synth.to_bf16_bits(synth.student_t(seed, (N, C), 3.0))
    perm, codes, scales = ql.prepare_prquant(wb, k)          # offline, library host code
    xb, _ = synth.activations_bf16(seed, M, C, 0.005, 50.0)
    xb = np.ascontiguousarray(xb[:, perm])
    return dict(name=f"prquant_tail_n{N}_c{C}_k{k}_m{M}", N=N, C=C, k=k, M=M, codes=codes,
                scales=scales, x=xb)


def mxfp4_workload(M: int = 16, seed: int = 1):
    """Single MXFP4 linear layer: X [16, 2048] N(0,1) with 1% outlier channels x20, W [2048, 2048]
    uniform E2M1 codes with E8M0 exponents uniform in [120, 130]."""
    import synth
    N = K = 2048
    codes = synth.uniform_nibble_bytes(seed, N, K)
    scales = synth.uniform_bytes(seed + 1, (N, K // 32), 120, 130)
    xb, _ = synth.activations_bf16(seed, M, K, 0.01, 20.0)
    return dict(name=f"mxfp4_linear_n{N}_k{K}_m{M}", N=N, C=K, k=0, M=M, codes=codes,
                scales=scales, x=xb)


def work_of(w) -> dict:
    M, N, C, k = w["M"], w["N"], w["C"], w["k"]
    Kp = C + k
    flops = 2.0 * M * N * Kp
    weight_bytes = N * Kp // 2 + N * Kp // 32
    bytes_ = weight_bytes + M * C * 2 + M * N * 2          # W codes+scales, X bf16 in, Y bf16 out
    gemm_bytes = weight_bytes + M * C // 2 + M * C // 32 + M * N * 2
    return dict(flops=flops, bytes=bytes_, gemm_bytes=gemm_bytes, weight_bytes=weight_bytes)


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, device_index: int):
        self.p = None
        self.path = None
        self.dev = device_index

    def __enter__(self):
        os.makedirs(os.path.join(ROOT, "gpurun_out"), exist_ok=True)
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_{os.getpid()}.csv")
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except Exception:
                self.p.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.p is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
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
                    if v.lower() == "active":
                        reasons.add(nm)
        med = float(np.median(sm)) if sm else None
        return {"sm_mhz": med, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ GPU arm
def _time_graph(graph, steps: int, flush, stream) -> float:
    """Mean device time (ms) of `steps` replays of a captured graph, L2 flushed before each."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in evs:
        flush()
        a.record(stream)
        graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def run_case(w, steps: int, warmup: int, device, flush, e2e: bool = False):
    """Times `steps` forwards (quantize + GEMM) replayed from CUDA graphs, so the numbers are
    device time without host launch gaps.  Also times each kernel alone the same way, and (e2e)
    the public forward call from pinned host memory with the copies inside the timed region."""
    import torch
    import bit_quantized_moe_tcgen05_b200 as ql
    lin = ql.QLinear(w["codes"], w["scales"], k_tail=w["k"])
    M, N = w["M"], w["N"]
    x = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).to(device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    ws = torch.empty(lin.workspace_bytes(M), dtype=torch.uint8, device=device)
    for _ in range(warmup):                       # eager warm-up (also sets kernel attributes)
        lin.quantize_input(x, ws)
        lin.gemm(M, y, ws)
    ql.check()
    g_step, g_q, g_g = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        lin.quantize_input(x, ws)
        lin.gemm(M, y, ws)
    with torch.cuda.graph(g_q):
        lin.quantize_input(x, ws)
    with torch.cuda.graph(g_g):
        lin.gemm(M, y, ws)
    stream = torch.cuda.current_stream(device)
    for g in (g_step, g_q, g_g):
        for _ in range(warmup):
            g.replay()
    ql.check()
    step_ms = _time_graph(g_step, steps, flush, stream)
    q_ms = _time_graph(g_q, steps, flush, stream)
    g_ms = _time_graph(g_g, steps, flush, stream)
    ql.check()
    out = dict(step_ms=step_ms, quant_ms=q_ms, gemm_ms=g_ms, launches=2 * steps)
    if e2e:
        xh = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
        yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        xd = torch.empty_like(x)
        for _ in range(warmup):
            xd.copy_(xh, non_blocking=True)
            lin.forward(xd, out=y, ws=ws)
            yh.copy_(y, non_blocking=True)
        torch.cuda.synchronize(device)
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush()
            e0[i].record(stream)
            xd.copy_(xh, non_blocking=True)
            lin.forward(xd, out=y, ws=ws)
            yh.copy_(y, non_blocking=True)
            e1[i].record(stream)
        torch.cuda.synchronize(device)
        ql.check()
        out["e2e_ms"] = float(np.mean([e0[i].elapsed_time(e1[i]) for i in range(steps)]))
        out["h2d"] = M * w["C"] * 2
        out["d2h"] = M * N * 2
        out["launches"] += 2 * steps
    del g_step, g_q, g_g
    lin.close()
    return out


def cpu_baseline(w, budget_s: float = 15.0) -> dict:
    """The oracle as it stands (numpy, fp64) on a bounded sample of the same workload: the first
    m_s tokens through quantize + augmented GEMM against the full weight."""
    from oracle import formats as F, mx, gemm as G
    import synth
    N, C, k = w["N"], w["C"], w["k"]
    codes = F.unpack_nibbles(w["codes"])
    m_s = 1
    xd_all = synth.bf16_bits_to_f64(w["x"])
    best = None
    while True:
        t0 = time.perf_counter()
        xd = xd_all[:m_s]
        xc, xs = mx.quantize_e8m0_b32(xd)
        if k:
            xc = np.concatenate([xc, xc[:, C - k:]], axis=1)
            xs = np.concatenate([xs, xs[:, (C - k) // 32:]], axis=1)
        y = G.gemm_ref(mx.dequant_e8m0_b32(xc, xs), mx.dequant_e8m0_b32(codes, w["scales"]))
        dt = time.perf_counter() - t0
        best = (m_s, dt)
        if dt > budget_s / 3 or m_s >= w["M"]:
            break
        m_s = min(w["M"], m_s * 4)
    m_s, dt = best
    flops = 2.0 * m_s * N * (C + k)
    cores = len(os.sched_getaffinity(0))
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{m_s} of {w['M']} tokens of {w['name']} (quantize + fp64 GEMM incl. weight "
                      f"dequant), {dt:.2f} s; numpy BLAS may use every core"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="qlinear", choices=["qlinear", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cases", default="all", choices=["all", "headline"])
    ap.add_argument("--workload", default="prquant_m2048",
                    choices=["prquant_m2048", "prquant_m512", "prquant_m16", "mxfp4_m16"],
                    help="headline workload (default: the PRQuant prefill case)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    head = {"prquant_m2048": lambda: prquant_workload(2048),
            "prquant_m512": lambda: prquant_workload(512),
            "prquant_m16": lambda: prquant_workload(16),
            "mxfp4_m16": lambda: mxfp4_workload(16)}[args.workload]()
    wk = work_of(head)

    if args.impl == "reference":
        if rank != 0:
            return
        cb = cpu_baseline(head)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "TFLOP/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": wk["flops"] / (cb["value"] * 1e12) * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": head["name"], "M": head["M"],
                                                "N": head["N"], "K_aug": head["C"] + head["k"],
                                                "parallelism": "replicas"},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    peaks = measured_peaks()
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)

    def flush():
        flush_buf.fill_(1)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(device)

    # warm up + headline timing (device) with clock sampling
    barrier()
    with ClockSampler(local) as clk:
        res = run_case(head, args.steps, args.warmup, device, flush, e2e=True)
    barrier()
    step_ms = res["step_ms"]
    e2e_ms = res["e2e_ms"]
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([step_ms, e2e_ms], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        step_ms, e2e_ms = float(t[0]), float(t[1])
    value = world * wk["flops"] / (step_ms * 1e-3) / 1e12
    e2e_val = world * wk["flops"] / (e2e_ms * 1e-3) / 1e12

    fp4_peak = peaks["bf16"] * NOMINAL_FP4_OVER_BF16
    gemm_tflops = wk["flops"] / (res["gemm_ms"] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": gemm_tflops / fp4_peak, "traffic": None,
                "kernel": "fp4_gemm_kernel (tcgen05.mma kind::mxf4 block32)",
                "peak_source": f"{peaks['src']} bf16 burst {peaks['bf16']} x {NOMINAL_FP4_OVER_BF16}"
                               " (nominal FP4/bf16 dense ratio)"}

    cases = {}
    if args.cases == "all":
        for wl in (prquant_workload(16), prquant_workload(512), mxfp4_workload(16)):
            r = run_case(wl, args.steps, args.warmup, device, flush)
            wkk = work_of(wl)
            cases[wl["name"]] = {
                "step_us": r["step_ms"] * 1e3, "gemm_us": r["gemm_ms"] * 1e3,
                "quant_us": r["quant_ms"] * 1e3,
                "tflops": wkk["flops"] / (r["step_ms"] * 1e-3) / 1e12,
                "weight_stream_gbs": wkk["weight_bytes"] / (r["gemm_ms"] * 1e-3) / 1e9,
                "gemm_hbm_frac": wkk["gemm_bytes"] / (r["gemm_ms"] * 1e-3) / 1e9 / peaks["hbm"],
                "gemm_tensor_frac": wkk["flops"] / (r["gemm_ms"] * 1e-3) / 1e12 / fp4_peak,
            }
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4-e2m1/e8m0 (fp32 accumulate, bf16 out)",
        "data": "synthetic",
        "config": {"workload": head["name"], "M": head["M"], "N": head["N"], "K": head["C"],
                   "k_tail": head["k"], "K_aug": head["C"] + head["k"],
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "flushed between steps (256 MiB write)"},
        "roofline": roofline,
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
        "clocks": clk.summary(),
        "kernel_us": {"quant_mx_e8m0_b32": res["quant_ms"] * 1e3, "fp4_gemm": res["gemm_ms"] * 1e3},
        "cases": cases,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(head)
    print(json.dumps(line))


if __name__ == "__main__":
    main()
