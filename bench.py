#!/usr/bin/env python
"""Benchmark of the W4A4 quantized linear layer on B200.

Headline workload (the MXCode VQ configuration): W [2560, 9728] stored as 8-bit indices into
per-64x64-QBlock FP4 codebooks with E4M3-B16 scales and an FP32 tensor scale; activations bf16
quantized online to E4M3-B16.  One step = the layer's whole hot path (E4M3-B16 activation
quantization, in-GEMM codebook decode, block16 tcgen05 MMA, epilogue) at each of the decode
batch sizes M = 1, 8 and 64.  Metric: weight-stream GB/s = weight bytes streamed (3 passes per
step) / step time, whole job.  Launches are replayed from CUDA graphs; each step uses the next of
R weight copies whose total exceeds the 126 MB L2, so every pass streams from HBM.

Extra cases (one GPU only): the PRQuant tail-residual layer at M = 2048 (prefill, TFLOP/s), 512
and 16; the single MXFP4 layer at M = 16; the INT4 dense + block-sparse residual layer at
M = 4096, 256, 16 and 1; and the routed MoE FFN (128 experts, top-8, 2048 tokens).  Exactly
`--steps` steps are timed for the headline.

Multi-GPU: the layer shards into independent replicas (no collective); each rank runs the same
workload on its own GPU and `value` sums the ranks' work over the slowest rank's time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlinear|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 linear TFLOP/s (prefill) & weight-stream GB/s (decode) vs B200 roofline"
NOMINAL_FP4_OVER_BF16 = 4.0      # 9 PFLOP/s dense FP4 / 2.25 PFLOP/s dense bf16
L2_BYTES = 126 * 1024 * 1024


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the timed GEMM kernel,
# from ncu captures under profiles/: the headline's GEMM launches averaged over M = 1, 8, 64 (the
# current kernels). An entry is None while its kernel has changed since its capture: the PRQuant
# M = 2048 GEMM's unsplit epilogue was changed after its capture (24.59 MB per launch then).
NCU_TRAFFIC_PER_LAUNCH = {"vq": (11.0144e6 + 11.0659e6 + 11.3400e6) / 3, "prquant_m2048": None}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------------------------------ workloads
def _pack_nibbles(c: np.ndarray) -> np.ndarray:
    return ((c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)).astype(np.uint8)


def _vq_weights(seed: int):
    """W [2560, 9728] Student-t(4) as bf16 bits and its seeded k-means FP4 codebooks per 64x64
    QBlock (256 entries of d = 4), data synthesis only."""
    import synth
    N, K = 2560, 9728
    wb = synth.to_bf16_bits(synth.student_t(seed, (N, K), 4.0))
    cb = synth.vq_codebooks(seed, synth.bf16_bits_to_f64(wb))
    return wb, cb


def make_vq(Ms=(1, 8, 64), seed: int = 2, prep_with: str = "library") -> dict:
    """MXCode-style VQ layer: W [2560, 9728] Student-t(4) -> PreScale E4M3-B16 scales + FP32
    tensor scale, seeded k-means FP4 codebooks per 64x64 QBlock (256 entries of d = 4), 8-bit
    indices; X [M, 9728] N(0,1) for each M.  prep_with = "library" prepares the weight with the
    library's host code (GPU arm), "oracle" with the CPU oracle (reference arm and CPU baseline:
    that arm never loads the library)."""
    import synth
    N, K = 2560, 9728
    wb, cb = _vq_weights(seed)
    cbp = _pack_nibbles(cb)
    if prep_with == "oracle":
        from oracle import vq as ovq
        p = ovq.prepare(synth.bf16_bits_to_f64(wb), cb)
        ts, sb, idx = p["ts"], p["sb"], p["idx"]
        make = None
    else:
        import bit_quantized_moe_tcgen05_b200 as ql
        ts, sb, idx = ql.prepare_vq_prescale(wb, cbp)
        make = lambda: ql.QLinear(None, sb, wfmt=ql.QL_W_VQ_PRESCALE_E4M3_B16,
                                  w_tensor_scale=float(ts), indices=idx, codebooks=cbp)
    xs = {M: synth.activations_bf16(seed, M, K, 0.0, 1.0)[0] for M in Ms}
    wbytes = idx.nbytes + cbp.nbytes + sb.nbytes
    return dict(name=f"mxcode_vq_n{N}_k{K}_m{'-'.join(map(str, Ms))}", kind="vq", N=N, K=K, C=K,
                Ms=list(Ms), xs=xs, weight_bytes=wbytes, make=make, wb=wb, cb=cb,
                oracle_prep=dict(ts=ts, sb=sb, idx=idx) if prep_with == "oracle" else None)


_PRQ_CACHE = {}


def _prquant_weight(seed: int):
    if seed not in _PRQ_CACHE:
        import synth
        import bit_quantized_moe_tcgen05_b200 as ql
        wb = synth.to_bf16_bits(synth.student_t(seed, (2560, 9728), 3.0))
        _PRQ_CACHE[seed] = ql.prepare_prquant(wb, 128)
    return _PRQ_CACHE[seed]


def make_prquant(M: int, seed: int = 3) -> dict:
    """PRQuant tail-residual layer: W [2560, 9728] bf16 Student-t(3), k = 128 tail channels
    (library host preparation); X [M, 9728] N(0,1) with 0.5% outlier channels x50, permuted."""
    import synth
    import bit_quantized_moe_tcgen05_b200 as ql
    N, C, k = 2560, 9728, 128
    perm, codes, scales = _prquant_weight(seed)
    xb, _ = synth.activations_bf16(seed, M, C, 0.005, 50.0)
    xb = np.ascontiguousarray(xb[:, perm])
    return dict(name=f"prquant_tail_n{N}_c{C}_k{k}_m{M}", kind="mx", N=N, K=C + k, C=C, Ms=[M],
                xs={M: xb}, weight_bytes=codes.nbytes + scales.nbytes,
                make=lambda: ql.QLinear(codes, scales, k_tail=k))


def make_mxfp4(M: int = 16, seed: int = 1) -> dict:
    """Single MXFP4 linear layer: X [16, 2048] N(0,1) with 1% outlier channels x20, W [2048, 2048]
    uniform E2M1 codes with E8M0 exponents uniform in [120, 130]."""
    import synth
    import bit_quantized_moe_tcgen05_b200 as ql
    N = K = 2048
    codes = synth.uniform_nibble_bytes(seed, N, K)
    scales = synth.uniform_bytes(seed + 1, (N, K // 32), 120, 130)
    xb, _ = synth.activations_bf16(seed, M, K, 0.01, 20.0)
    return dict(name=f"mxfp4_linear_n{N}_k{K}_m{M}", kind="mx", N=N, K=K, C=K, Ms=[M], xs={M: xb},
                weight_bytes=codes.nbytes + scales.nbytes,
                make=lambda: ql.QLinear(codes, scales))


def make_int4(M: int, seed: int = 5) -> dict:
    """MosaicQuant-style layer: W [8192, 8192] Student-t(4) -> INT4 per 128-group + 655 residual
    blocks of 16 x 128 chosen over the 4096-token calibration X (library host preparation);
    X [M, 8192] = the first M calibration rows (N(0,1), 1% outlier channels x30)."""
    import synth
    import bit_quantized_moe_tcgen05_b200 as ql
    N = K = 8192
    wb = synth.to_bf16_bits(synth.student_t(seed, (N, K), 4.0))
    xcal, _ = synth.activations_bf16(seed, 4096, K, 0.01, 30.0)
    p = ql.prepare_int4_bsr(wb, xcal, 0.02)
    wbytes = p["codes"].nbytes + p["scales"].nbytes + p["rowptr"].nbytes + p["col"].nbytes + \
        p["rcodes"].nbytes + p["rscales"].nbytes
    bsr = dict(rowptr=p["rowptr"], col=p["col"], rcodes=p["rcodes"], rscales=p["rscales"])
    nnz = len(p["col"])
    return dict(name=f"int4_bsr_n{N}_k{K}_nnzb{nnz}_m{M}", kind="int4", N=N, K=K, C=K, Ms=[M],
                xs={M: np.ascontiguousarray(xcal[:M])}, weight_bytes=wbytes,
                extra_flops_per_token=2.0 * nnz * 16 * 128,
                make=lambda: ql.QLinear(p["codes"], p["scales"], wfmt=ql.QL_W_INT4_G128_BSR, bsr=bsr))


def flops_of(w, M) -> float:
    return 2.0 * M * w["N"] * w["K"] + M * w.get("extra_flops_per_token", 0.0)


def forward_bytes_of(w, M) -> float:
    """Algorithmic bytes of one one-launch forward (activation quantization fused into the GEMM):
    weight payload + bf16 x read + bf16 y written."""
    return w["weight_bytes"] + 2.0 * M * w["C"] + 2.0 * M * w["N"]


def gemm_bytes_of(w, M) -> float:
    """Algorithmic bytes of one GEMM launch: weight payload + quantized activation + bf16 y."""
    if w["kind"] == "int4":
        return w["weight_bytes"] + M * w["C"] + M * w["C"] / 32 + 2.0 * M * w["N"]
    sf = 16 if w["kind"] == "vq" else 32
    return w["weight_bytes"] + M * w["C"] / 2 + M * w["C"] / sf + 2.0 * M * w["N"]


def make_moe(seed: int = 4) -> dict:
    """MoE grouped FFN: 128 experts, top-8, hidden 2048, intermediate 768, per-row 16-centroid
    bf16 codebooks with 4-bit indices (seeded 1-D k-means on Student-t(4)), 2048 tokens N(0,1),
    Zipf(1.1) router logits."""
    import synth
    E, H, I, T, k = 128, 2048, 768, 2048, 8
    gi, gc, di, dc = [], [], [], []
    for e in range(E):
        c, i = synth.cluster_rows(seed * 1000 + e, 2 * I, H)
        gc.append(c); gi.append(i)
        c, i = synth.cluster_rows(seed * 1000 + 500 + e, H, I)
        dc.append(c); di.append(i)
    xb, _ = synth.activations_bf16(seed, T, H, 0.0, 1.0)
    logits = synth.zipf_router_logits(seed, T, E)
    flops = 2.0 * T * k * (2 * I * H + H * I)
    wbytes = E * (2 * I * H + H * I) // 2 + E * (2 * I + H) * 32
    return dict(name=f"moe_e{E}_top{k}_h{H}_i{I}_t{T}", E=E, H=H, I=I, T=T, k=k, x=xb,
                logits=logits, gi=np.concatenate(gi), gc=np.concatenate(gc),
                di=np.concatenate(di), dc=np.concatenate(dc), flops=flops, weight_bytes=wbytes)


def run_moe(w, steps: int, warmup: int, device) -> dict:
    """Device time of the whole routed FFN forward (routing, x quantization, gate/up GEMM with
    SwiGLU + requantization, down GEMM, combine), replayed from a CUDA graph."""
    import torch
    import bit_quantized_moe_tcgen05_b200 as ql
    layer = ql.MoE(w["gi"], w["gc"], w["di"], w["dc"], w["E"], w["k"])
    x = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).to(device)
    lg = torch.from_numpy(w["logits"]).to(device)
    y = torch.empty((w["T"], w["H"]), dtype=torch.bfloat16, device=device)
    ws = layer.workspace(w["T"], device)
    for _ in range(warmup):
        layer(x, lg, out=y, ws=ws)
    ql.check()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(x, lg, out=y, ws=ws)
    for _ in range(warmup):
        g.replay()
    ms = _elapsed(g.replay, steps, torch.cuda.current_stream(device)) / steps
    ql.check()
    del g
    layer.close()
    return dict(step_ms=ms, steps=steps)


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, device_index: int):
        self.p = None
        self.dev = device_index

    def __enter__(self):
        self.path = os.path.join(tempfile.gettempdir(), f"qlinear_clocks_{os.getpid()}.csv")
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
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ ranks
def max_over_ranks(vals, device):
    """Element-wise maximum of a list of floats over all ranks of the default process group (the
    slowest rank's device times); the list itself when there is no group or a single rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_throughput(units_per_step_per_rank: float, world: int, step_ms: float) -> float:
    """Whole-job throughput: every rank processes its own units each step (replicas), and the
    step takes as long as the slowest rank."""
    return world * units_per_step_per_rank / (step_ms * 1e-3)


# ------------------------------------------------------------------------------ GPU arm
def _elapsed(fn, reps: int, stream) -> float:
    """Device time (ms) of `reps` calls of fn, bracketed by synchronisation and CUDA events."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def count_kernel_launches(fn) -> int | None:
    """Kernel launches that fn issues: fn is captured into a CUDA graph and its kernel nodes
    counted (None where the graph cannot be inspected)."""
    import torch
    try:
        from cuda.bindings import runtime as cudart
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            fn()
        err, _, n = cudart.cudaGraphGetNodes(g.raw_cuda_graph(), 0)
        if err != cudart.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = cudart.cudaGraphGetNodes(g.raw_cuda_graph(), n)
        kernels = 0
        for nd in nodes:
            e2, t = cudart.cudaGraphNodeGetType(nd)
            if e2 == cudart.cudaError_t.cudaSuccess and t == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kernels += 1
        del g
        return kernels
    except Exception:
        return None


def run_case(w, steps: int, warmup: int, device, e2e: bool = False, flush_bytes: int = 0):
    """Device time per step (ms) of w's forwards (every M of w["Ms"] per step), replayed from a
    CUDA graph over R rotating weight copies with R * weight bytes > L2 (or with an explicit L2
    flush before each replay), plus per-kernel times measured the same way, plus (e2e) the public
    forward call from pinned host memory with the copies inside the timed region."""
    import torch
    import bit_quantized_moe_tcgen05_b200 as ql
    steps = max(1, steps)
    R = 1 if flush_bytes else min(64, L2_BYTES // w["weight_bytes"] + 2)
    layers = [w["make"]() for _ in range(R)]
    Ms = w["Ms"]
    xs = {M: torch.from_numpy(w["xs"][M].view(np.int16)).view(torch.bfloat16).to(device) for M in Ms}
    ys = {M: torch.empty((M, w["N"]), dtype=torch.bfloat16, device=device) for M in Ms}
    wss = {M: torch.empty(layers[0].workspace_bytes(M), dtype=torch.uint8, device=device) for M in Ms}
    flush_buf = torch.empty(flush_bytes, dtype=torch.uint8, device=device) if flush_bytes else None
    # rotation mode: one write larger than L2 before each timed region, so that a short run
    # (fewer steps than weight copies) starts from cold weights as well
    evict_buf = None if flush_bytes else torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)

    def fwd(layer, M):   # the public call: one launch for decode sizes (quantizer fused in)
        layer.forward(xs[M], out=ys[M], ws=wss[M])

    for _ in range(warmup):
        for layer in layers:
            for M in Ms:
                fwd(layer, M)
    ql.check()
    stream = torch.cuda.current_stream(device)
    g_all, g_q, g_g = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all):
        for layer in layers:
            for M in Ms:
                fwd(layer, M)
    with torch.cuda.graph(g_q):
        for layer in layers:
            for M in Ms:
                layer.quantize_input(xs[M], wss[M])
    with torch.cuda.graph(g_g):
        for layer in layers:
            for M in Ms:
                layer.gemm(M, ys[M], wss[M])
    # Exactly `steps` steps are timed: `full` replays of the R-layer graphs, then one replay of a
    # graph over the first `part` layers.
    full, part = divmod(steps, R)
    p_all = p_q = p_g = None
    if part:
        p_all, p_q, p_g = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(p_all):
            for layer in layers[:part]:
                for M in Ms:
                    fwd(layer, M)
        with torch.cuda.graph(p_q):
            for layer in layers[:part]:
                for M in Ms:
                    layer.quantize_input(xs[M], wss[M])
        with torch.cuda.graph(p_g):
            for layer in layers[:part]:
                for M in Ms:
                    layer.gemm(M, ys[M], wss[M])
    for g in (g_all, g_q, g_g, p_all, p_q, p_g):
        if g is not None:
            for _ in range(warmup):
                g.replay()
    ql.check()
    kernels_per_step = count_kernel_launches(lambda: [fwd(layer, M) for M in Ms for layer in layers[:1]])

    def timed(graph, pgraph):
        if flush_buf is None:
            def run():
                for _ in range(full):
                    graph.replay()
                if pgraph is not None:
                    pgraph.replay()
            evict_buf.fill_(1)
            return _elapsed(run, 1, stream) / steps
        tot = 0.0                                     # R == 1: one flushed replay per step
        for _ in range(steps):
            flush_buf.fill_(1)
            tot += _elapsed(graph.replay, 1, stream)
        return tot / steps

    out = dict(R=R, step_ms=timed(g_all, p_all), quant_ms=timed(g_q, p_q),
               gemm_ms=timed(g_g, p_g), steps=steps, kernels_per_step=kernels_per_step)
    ql.check()
    if e2e:
        xh = {M: torch.from_numpy(w["xs"][M].view(np.int16)).view(torch.bfloat16).pin_memory()
              for M in Ms}
        yh = {M: torch.empty((M, w["N"]), dtype=torch.bfloat16).pin_memory() for M in Ms}
        xd = {M: torch.empty_like(xs[M]) for M in Ms}
        count = [0]

        def e2e_step():
            layer = layers[count[0] % R]
            count[0] += 1
            for M in Ms:
                xd[M].copy_(xh[M], non_blocking=True)
                layer.forward(xd[M], out=ys[M], ws=wss[M])
                yh[M].copy_(ys[M], non_blocking=True)

        for _ in range(warmup):
            e2e_step()
        out["e2e_ms"] = _elapsed(e2e_step, steps, stream) / steps
        out["h2d"] = sum(M * w["C"] * 2 for M in Ms)
        out["d2h"] = sum(M * w["N"] * 2 for M in Ms)
        ql.check()
    del g_all, g_q, g_g, p_all, p_q, p_g
    for layer in layers:
        layer.close()
    return out


# ------------------------------------------------------------------------------ CPU baseline
def cpu_baseline_vq(w, budget_s: float = 20.0) -> dict:
    """The oracle as it stands (numpy element-wise codecs, plain C fp64 sums) on a bounded sample
    of the headline workload: whole forwards (E4M3-B16 activation quantization, codebook decode,
    dequantized fp64 GEMM) at the workload's batch sizes, as many as fit the time budget.  The
    weight is prepared by the oracle too (oracle.vq.prepare), never by the library."""
    from oracle import vq
    import synth
    cb = w["cb"]
    if w.get("oracle_prep") is None:
        w["oracle_prep"] = vq.prepare(synth.bf16_bits_to_f64(w["wb"]), cb)
    prep = w["oracle_prep"]
    done, t0 = [], time.perf_counter()
    for M in w["Ms"] * 4:
        vq.forward(synth.bf16_bits_to_f64(w["xs"][M]), prep, cb)
        done.append(M)
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": len(done) * w["weight_bytes"] / dt / 1e9, "unit": "GB/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{len(done)} forwards (M = {done}) of {w['name']}, {dt:.1f} s; "
                      "fp64 C sums on every core (OpenMP)"}


# ------------------------------------------------------------------------------ tensor peaks
TENSOR_KINDS = {"fp4_mxf4_block32": 0, "fp4_mxf4nvf4_block16": 1, "int8": 2, "bf16": 3}


def measure_tensor_peaks(device, burst_ms: float = 4.0, sustain_s: float = 1.5) -> dict:
    """TFLOP/s of back-to-back tcgen05 MMAs (M = 128, N = 256) on operands resident in shared
    memory, one CTA per SM (ql_tensor_peak): the most a GEMM of that instruction kind can reach
    on this GPU.  burst = best single launch of ~burst_ms after a warm-up; sustained = launches
    back to back for ~sustain_s (the clocks settle under the power cap).  The bf16 figure is the
    same method on the pipe whose cuBLAS throughput MEASURED_PEAKS.json holds (a check)."""
    import ctypes
    import torch
    import bit_quantized_moe_tcgen05_b200 as ql
    stream = torch.cuda.current_stream(device)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    out = {}
    for name, kind in TENSOR_KINDS.items():
        fl = ctypes.c_double()

        def launch(iters):
            st = ql.lib.ql_tensor_peak(kind, 256, iters, sms, ctypes.byref(fl), stream.cuda_stream)
            if st != 0:
                raise ql.QLError(st, "ql_tensor_peak")
            return fl.value

        launch(64)
        ql.check()
        ms = _elapsed(lambda: launch(256), 1, stream)
        it = max(256, int(256 * burst_ms / max(ms, 1e-3)))
        best = 0.0
        for _ in range(5):
            ms = _elapsed(lambda: launch(it), 1, stream)
            best = max(best, fl.value / (ms * 1e-3) / 1e12)
        reps = max(2, int(sustain_s * 1e3 / max(ms, 1e-3)))
        ms = _elapsed(lambda: launch(it), reps, stream)
        ql.check()
        out[name] = {"burst": best, "sustained": reps * fl.value / (ms * 1e-3) / 1e12}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=32)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="qlinear", choices=["qlinear", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cases", default="all", choices=["all", "none"])
    ap.add_argument("--workload", default="vq", choices=["vq", "prquant_m2048", "prquant_m512",
                                                         "prquant_m16", "mxfp4_m16", "int4_m4096",
                                                         "int4_m256", "int4_m16", "int4_m1", "moe"])
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # The oracle on the host cores, on the headline workload prepared by the oracle itself;
        # this arm never loads the CUDA library.  Under torchrun only rank 0 runs it.
        if rank != 0:
            return
        if args.workload != "vq":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the "
                              "oracle on the headline VQ workload only"}))
            return
        head = make_vq(prep_with="oracle")
        cb = cpu_baseline_vq(head)
        units = len(head["Ms"]) * head["weight_bytes"] / 1e9
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": cb["value"], "unit": cb["unit"],
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": units / cb["value"] * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": head["name"], "N": head["N"], "K": head["K"], "M": head["Ms"],
                       "parallelism": "single",
                       "l2": "rotating weight copies totalling > 126 MB L2 (no flush)"},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": cb["unit"], "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)

    if args.workload == "moe":
        w = make_moe()
        r = run_moe(w, args.steps, args.warmup, device)
        peaks = measured_peaks()
        tf = w["flops"] / (r["step_ms"] * 1e-3) / 1e12
        print(json.dumps({"metric": METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": 1,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["step_ms"],
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "bf16 MMA on exact MXFP4 / codebook values, fp32 accumulate",
                          "data": "synthetic", "config": {"workload": w["name"]},
                          "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16"],
                                       "unit": "TFLOP/s", "frac": tf / peaks["bf16"],
                                       "traffic": None, "kernel": "whole routed FFN forward"}}))
        return
    builders = {"vq": make_vq, "prquant_m2048": lambda: make_prquant(2048),
                "prquant_m512": lambda: make_prquant(512), "prquant_m16": lambda: make_prquant(16),
                "mxfp4_m16": lambda: make_mxfp4(16), "int4_m4096": lambda: make_int4(4096),
                "int4_m256": lambda: make_int4(256), "int4_m16": lambda: make_int4(16),
                "int4_m1": lambda: make_int4(1)}
    head = builders[args.workload]()
    decode = head["kind"] == "vq" or max(head["Ms"]) <= 64
    unit = "GB/s" if decode else "TFLOP/s"

    def per_step_units(w):
        if decode:
            return len(w["Ms"]) * w["weight_bytes"] / 1e9
        return sum(flops_of(w, M) for M in w["Ms"]) / 1e12

    config = {"workload": head["name"], "N": head["N"], "K": head["K"], "M": head["Ms"],
              "parallelism": "replicas" if world > 1 else "single",
              "l2": ("rotating weight copies totalling > 126 MB L2 (no flush)" if decode
                     else "flushed before each step (256 MiB write)")}
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(device)

    peaks = measured_peaks()
    barrier()
    with ClockSampler(local) as clk:
        res = run_case(head, args.steps, args.warmup, device, e2e=True,
                       flush_bytes=0 if decode else 256 << 20)
    barrier()
    step_ms, e2e_ms = max_over_ranks([res["step_ms"], res["e2e_ms"]], device)
    units = per_step_units(head)
    value = job_throughput(units, world, step_ms)
    e2e_val = job_throughput(units, world, e2e_ms)

    tp = measure_tensor_peaks(device)
    fp4_peak = tp["fp4_mxf4_block32"]["burst"]
    int8_peak = tp["int8"]["burst"]
    nl = len(head["Ms"])
    # the dominant kernel: the GEMM launch of each forward (it streams the weight), timed alone
    # by the graph of GEMM calls on a quantized workspace: at M = 1 the decode kernel, above it
    # (E4M3-B16 activations) the general split-K GEMM, as the forward's plan chooses
    if decode:
        alg = sum(gemm_bytes_of(head, M) for M in head["Ms"]) / nl
        ach = alg / (res["gemm_ms"] / nl * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                    "frac": ach / peaks["hbm"], "traffic": NCU_TRAFFIC_PER_LAUNCH.get(args.workload),
                    "kernel": ("GEMM launch per forward, averaged over M = " +
                               ", ".join(map(str, head["Ms"])) +
                               ": fp4_decode_kernel at M = 1, fp4_gemm_kernel (split-K) above; "
                               "VQ decode in shared memory, block16 MMA"),
                    "algorithmic_bytes_per_launch": alg,
                    "peak_source": f"{peaks['src']} HBM copy bandwidth (MEASURED_PEAKS.json)"}
    else:
        alg = sum(flops_of(head, M) for M in head["Ms"]) / nl
        ach = alg / (res["gemm_ms"] / nl * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": ach, "peak": fp4_peak, "unit": "TFLOP/s",
                    "frac": ach / fp4_peak, "traffic": NCU_TRAFFIC_PER_LAUNCH.get(args.workload),
                    "kernel": "fp4_gemm_kernel (mxf4)",
                    "algorithmic_flops_per_launch": alg,
                    "peak_source": "measured: tcgen05 kind::mxf4 block32 MMA loop, burst"}

    def case_line(wl, r, M):
        int4 = wl["kind"] == "int4"
        pk = int8_peak if int4 else fp4_peak
        d = {"step_us": r["step_ms"] * 1e3, "gemm_us": r["gemm_ms"] * 1e3,
             "quant_us": r["quant_ms"] * 1e3,
             "tflops": flops_of(wl, M) / (r["step_ms"] * 1e-3) / 1e12,
             "gemm_tflops": flops_of(wl, M) / (r["gemm_ms"] * 1e-3) / 1e12,
             "tensor_peak_tflops": pk,
             "tensor_peak": ("measured int8 (tcgen05 kind::i8 MMA loop, burst)" if int4
                             else "measured fp4 (tcgen05 kind::mxf4 MMA loop, burst)"),
             "weight_stream_gbs": wl["weight_bytes"] / (r["step_ms"] * 1e-3) / 1e9,
             "l2": "flushed (256 MiB write)" if r["R"] == 1 else f"{r['R']} rotating weight copies"}
        d["gemm_tensor_frac"] = d["gemm_tflops"] / pk
        if M <= 64 and not int4:   # one-launch forward: its bytes against HBM
            d["hbm_frac"] = forward_bytes_of(wl, M) / (r["step_ms"] * 1e-3) / 1e9 / peaks["hbm"]
        else:
            d["gemm_hbm_frac"] = gemm_bytes_of(wl, M) / (r["gemm_ms"] * 1e-3) / 1e9 / peaks["hbm"]
        return d

    cases, prefill = {}, None
    if args.cases == "all" and world == 1:
        int4_4096 = make_int4(4096)
        int4_cases = [dict(int4_4096, name=int4_4096["name"].replace("_m4096", f"_m{M}"), Ms=[M],
                           xs={M: np.ascontiguousarray(int4_4096["xs"][4096][:M])})
                      for M in (256, 16, 1)]
        for wl, flush in ((make_prquant(2048), 256 << 20), (make_prquant(512), 0),
                          (make_prquant(16), 0), (make_mxfp4(16), 0), (int4_4096, 256 << 20),
                          *[(c, 0) for c in int4_cases]):
            r = run_case(wl, 8, args.warmup, device, flush_bytes=flush)
            cases[wl["name"]] = case_line(wl, r, wl["Ms"][0])
            if wl["name"].endswith("_m2048") and wl["name"].startswith("prquant"):
                c = cases[wl["name"]]
                prefill = {"workload": wl["name"], "value": c["gemm_tflops"], "unit": "TFLOP/s",
                           "step_tflops": c["tflops"],
                           "roofline": {"bound": "tensor", "achieved": c["gemm_tflops"],
                                        "peak": fp4_peak, "unit": "TFLOP/s",
                                        "frac": c["gemm_tflops"] / fp4_peak,
                                        "traffic": NCU_TRAFFIC_PER_LAUNCH.get("prquant_m2048"),
                                        "kernel": "fp4_gemm_kernel (mxf4 block32, PRQuant tail)",
                                        "peak_source": "measured"}}
        mw = make_moe()
        r = run_moe(mw, 10, args.warmup, device)
        tf = mw["flops"] / (r["step_ms"] * 1e-3) / 1e12
        cases[mw["name"]] = {"step_us": r["step_ms"] * 1e3, "tflops": tf,
                             "bf16_tensor_frac": tf / peaks["bf16"],
                             "fp4_tensor_frac": tf / fp4_peak,
                             "l2": "weights 317 MB > L2"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    kps = res.get("kernels_per_step")   # counted in a captured graph of one step's forwards
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": res["steps"],
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("fp4-e2m1 E4M3-B16 (+fp32 tensor scales), fp32 accumulate, bf16 out"
                  if head["kind"] == "vq" else "fp4-e2m1 E8M0-B32, fp32 accumulate, bf16 out"),
        "data": "synthetic", "config": config, "roofline": roofline,
        "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": kps * res["steps"] if kps is not None else None,
        "clocks": clk.summary(),
        "kernel_us_per_step": {"forward": res["step_ms"] * 1e3,
                               "split_api_quantize": res["quant_ms"] * 1e3,
                               "split_api_gemm": res["gemm_ms"] * 1e3},
        "tensor_peaks_tflops": tp,
    }
    line["cases"] = cases
    if not args.no_cpu_baseline and head["kind"] == "vq" and world == 1:
        line["cpu_baseline"] = cpu_baseline_vq(head)
    if prefill is not None:   # last, so that the end of the line (what log tails keep) holds it
        line["prefill"] = prefill
    print(json.dumps(line))


if __name__ == "__main__":
    main()
