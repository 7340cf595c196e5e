"""Benchmark of the W4A16 decode path on B200 (one JSON line on rank 0).

Workload (one "step"): one decode token through three Llama-2-7B-class projection shapes,
W4A16 g=128 (INT4 codes, binary16 S and Z per 128 weights), X bf16 1 x K:
    4096 x 4096, 11008 x 4096, 4096 x 11008     (W: N x K, ~N(0, 0.02))
i.e. three wq_w4a16_gemm calls at M = 1. The metric is HBM throughput of the GEMV in GB/s
of algorithmic bytes (N*K/2 packed + 4*N*K/128 for S and Z + 2K for x + 2N for y).
Weights cycle through rotating copies totalling more than 3x the L2 cache, so every
launch streams its weights from HBM. Timing: CUDA graphs of the steps, CUDA events on the
capturing stream, barrier + synchronize on both sides, max over ranks.

Also reported (outside the timed step): per-shape times of the step, M = 4, 8, 16 and 32
on the same shapes, W8A16 decode at M = 1 on them, the quantizer over the 70B-class weights
(28672 x 8192, 8192 x 28672) and the 70B decode layer at M = 1, 8 and 32 on them, the
prefill GEMM (2048 x 4096 x 11008) in W4A16 and in W8A16, the oracle on the host cores
(cpu_baseline) and the end-to-end rate through host buffers (e2e: one H2D copy of the
step's X rows, the three calls, one D2H copy of its Y rows, a synchronize).
roofline.traffic comes from profiles/gemv_traffic.json while the decode kernels' sources
match the hash recorded there.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import wq_inputs  # noqa: E402

METRIC = "W4A16 GEMV HBM GB/s (% of peak) at M=1; prefill TFLOP/s (% BF16 peak)"
UNIT = "GB/s"
SHAPES = wq_inputs.SHAPES_7B
WORKLOAD = ("7B-class decode GEMV, M=1, W4A16 g128 asymmetric INT4 (fp16 S, Z), "
            "shapes 4096x4096, 11008x4096, 4096x11008, X bf16 ~N(0,1), W ~N(0,0.02)")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def gemv_bytes(M, N, K, group=128):
    """Algorithmic bytes of one W4A16 matmul: packed codes, S and Z, X and Y."""
    return N * K // 2 + 4 * N * (K // group) + 2 * M * K + 2 * M * N


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------------ distributed

def dist_setup(n_gpus):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU oracle baseline

class OracleGemv:
    """The oracle's decode GEMV (fp64 numpy: unpack, dequantize, multiply) on a sample of
    rows of each shape. Inputs are quantized by the oracle once, outside any timing."""

    def __init__(self, shapes, rows_per_shape):
        import oracle

        self.oracle = oracle
        self.work = []
        for (N, K) in shapes:
            n = min(rows_per_shape, N)
            Wb = wq_inputs.weight_bf16(n, K, 0.02)
            codes, S, Z = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), 128)
            X = wq_inputs.bf16_bits_to_f64(wq_inputs.act_bf16(1, K))
            self.work.append((oracle.pack_int4(codes), S, Z, X, n, K))
        self.bytes = sum(gemv_bytes(1, n, K) for (_, _, _, _, n, K) in self.work)

    def run(self):
        """One pass over the sample; returns seconds."""
        o = self.oracle
        t0 = time.perf_counter()
        for packed, S, Z, X, n, K in self.work:
            Y = o.w4a16_matmul(X, o.unpack_int4(packed), S, Z, 128, "exact")
            assert Y.shape == (1, n)
        return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(target_s=10.0, rows=1024):
    """Oracle GB/s on a bounded sample: `rows` rows of each shape, passes until ~target_s."""
    og = OracleGemv(SHAPES, rows)
    og.run()
    tt, passes = 0.0, 0
    while tt < target_s:
        tt += og.run()
        passes += 1
    return {"value": round(og.bytes * passes / tt / 1e9, 4), "unit": UNIT,
            "cores": blas_threads(), "host_cores": os.cpu_count(), "kind": "oracle",
            "threading": "unpack and dequantize run single-threaded in numpy; only the fp64 "
                         "matmul uses the BLAS threads counted in 'cores'",
            "sample": f"{rows} rows of each of the 3 shapes at M=1 (unpack + dequant + fp64 "
                      f"matmul), {passes} passes in {tt:.1f} s"}


def c3_oracle_parity(Wb, gpu):
    """The GPU quantizer's codes, S' and Z on the C3 outlier weights against the oracle: every
    row at per tensor, 256 sampled rows (the first and last among them) at g = 128 and per
    channel. Returns {granularity: bool}."""
    import oracle

    W = wq_inputs.bf16_bits_to_f64(Wb)
    N = W.shape[0]
    rows = np.sort(np.random.default_rng(3).choice(N, 256, replace=False))
    rows[0], rows[-1] = 0, N - 1
    out = {}
    for name, (group, packed, S, Z) in gpu.items():
        if group == 0:
            codes, So, Zo = oracle.quantize_rtn_asym(W, 0)
            ok = np.array_equal(packed, oracle.pack_int4(codes))
        else:
            codes, So, Zo = oracle.quantize_rtn_asym(W[rows], group)
            ok = np.array_equal(packed[rows], oracle.pack_int4(codes))
            S, Z = S[rows], Z[rows]
        f16 = lambda v: np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)
        ok = ok and np.array_equal(S.ravel(), f16(So).ravel()) and \
            np.array_equal(Z.ravel(), f16(Zo).ravel())
        out[name] = bool(ok)
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows = 256
    og = OracleGemv(SHAPES, rows)
    for _ in range(args.warmup):
        og.run()
    total = sum(og.run() for _ in range(args.steps))
    value = og.bytes * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD + f" (CPU oracle, {rows} sampled rows per shape per step)"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": blas_threads(),
                         "host_cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{rows} rows of each of the 3 shapes per step"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------- GPU bench

def graph_time_us(fn, reps, warm=3):
    """Per-call microseconds of `fn` captured `reps` times in one CUDA graph."""
    import torch

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(warm):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = math.inf
    for _ in range(3):
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1e3 / reps)
    del g
    return best


_CUDART = None


def upload_graph(g, stream):
    """cudaGraphUpload of a captured graph on `stream`: moves the graph's one-time setup
    (its first-launch upload to the device) out of the timed region. Returns False when the
    runtime call is unavailable."""
    global _CUDART
    import ctypes

    try:
        if _CUDART is None:
            _CUDART = ctypes.CDLL("libcudart.so.12")
        rc = _CUDART.cudaGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                                     ctypes.c_void_p(stream.cuda_stream))
        return rc == 0
    except (OSError, AttributeError, RuntimeError):
        return False


def run_gpu(args):
    import torch

    import w4a16_dequant_matmul_b200 as wq

    rank, world = dist_setup(args.gpus)
    wq.build_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    # ---- weights: quantize once per shape on the GPU, then rotating copies > 3x L2
    base = []
    for (N, K) in SHAPES:
        W = wq_inputs.weight_bf16(N, K, 0.02)
        Wt = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).to(dev)
        packed, S, Z = wq.wq_quantize_rtn_g128(Wt)
        base.append((packed, S, Z))
        del Wt
    set_bytes = sum(p.numel() + 2 * s.numel() + 2 * z.numel() for p, s, z in base)
    nsets = max(4, math.ceil(3 * l2 / set_bytes))
    sets = [[(p.clone(), s.clone(), z.clone()) for (p, s, z) in base] for _ in range(nsets)]
    X = [torch.from_numpy(wq_inputs.act_bf16(1, K).view(np.int16)).view(torch.bfloat16).to(dev)
         for (_, K) in SHAPES]
    Y = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for (N, _) in SHAPES]
    step_bytes = sum(gemv_bytes(1, N, K) for (N, K) in SHAPES)
    assert wq.wq_get_status() == 0

    def step(i):
        for j, (p, s, z) in enumerate(sets[i % nsets]):
            wq.wq_w4a16_gemm(X[j], p, s, z, 128, Y=Y[j])

    # The timed steps run from CUDA graphs captured for exactly that count: one graph of all
    # of them up to kMaxGraphSteps, else graphs of B steps (a multiple of the weight sets)
    # and one of the remainder, so the timed region does not depend on how the step count
    # divides into graphs (each graph boundary breaks the launch overlap between kernels).
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(nsets):
            step(i)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(nsteps):
                step(i)
        return g

    kMaxGraphSteps = 1024
    if args.steps <= kMaxGraphSteps:
        plan = [(capture(args.steps), 1)]
    else:
        B = nsets * math.ceil(512 / nsets)
        plan = [(capture(B), args.steps // B)]
        if args.steps % B:
            plan.append((capture(args.steps % B), 1))
    g_warm = capture(max(args.warmup, 3))
    # The first launch of a freshly captured graph also uploads it to the device (measured
    # about 6 us per step extra on a 20-step graph); upload every graph before timing.
    uploaded = all(upload_graph(g, torch.cuda.current_stream()) for g, _ in plan)
    uploaded = upload_graph(g_warm, torch.cuda.current_stream()) and uploaded

    def run_timed():
        for g, reps in plan:
            for _ in range(reps):
                g.replay()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        barrier(world)
        torch.cuda.synchronize()
        # The W warm-up steps are queued right before the timed ones (no synchronize between):
        # while they run, the host submits the timed graphs, so the timed region opens on a
        # busy stream instead of waiting for the first submission. It holds exactly K steps.
        g_warm.replay()
        ev0.record()
        run_timed()
        ev1.record()
        torch.cuda.synchronize()
        barrier(world)
        dt_local = ev0.elapsed_time(ev1) * 1e-3
        soak = 0
        if dt_local < 1.5 and not args.no_soak:  # keep the step graphs running for the sampler
            reps = int(1.5 / max(dt_local, 1e-6)) + 1
            for _ in range(reps):
                run_timed()
            soak = reps * args.steps
            torch.cuda.synchronize()
    dt = ev0.elapsed_time(ev1) * 1e-3
    dt = max_over_ranks(dt, world)
    value = step_bytes * args.steps * world / dt / 1e9
    achieved = step_bytes * args.steps / dt / 1e9   # per GPU: the dominant kernel's rate
    assert wq.wq_get_status() == 0

    # ---- per-shape kernel rates (graph of 4*nsets launches each)
    per_shape = {}
    for j, (N, K) in enumerate(SHAPES):
        k = [0]

        def one(j=j, k=k):
            p, s, z = sets[k[0] % nsets][j]
            k[0] += 1
            wq.wq_w4a16_gemm(X[j], p, s, z, 128, Y=Y[j])
        us = graph_time_us(one, 4 * nsets)
        per_shape[f"{N}x{K}"] = {"us": round(us, 3), "GB/s": round(gemv_bytes(1, N, K) / us / 1e3, 1)}

    # ---- secondary: M = 4, 8, 16, 32 on the same shapes
    secondary = {}
    for M in (4, 8, 16, 32):
        tot_b, tot_us = 0, 0.0
        for j, (N, K) in enumerate(SHAPES):
            Xm = torch.from_numpy(wq_inputs.act_bf16(M, K).view(np.int16)).view(torch.bfloat16).to(dev)
            Ym = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            k = [0]

            def one(j=j, k=k, Xm=Xm, Ym=Ym):
                p, s, z = sets[k[0] % nsets][j]
                k[0] += 1
                wq.wq_w4a16_gemm(Xm, p, s, z, 128, Y=Ym)
            try:
                us = graph_time_us(one, 2 * nsets)
            except wq.WQError as e:
                secondary[f"gemv_M{M}"] = f"unavailable: {e}"
                break
            tot_b += gemv_bytes(M, N, K)
            tot_us += us
        else:
            secondary[f"gemv_M{M}_GB/s"] = round(tot_b / tot_us / 1e3, 1)

    # ---- secondary: W8A16 decode (INT8 per-channel weights) at M = 1 on the same shapes,
    # rotating weight sets larger than L2
    try:
        base8 = []
        for (N, K) in SHAPES:
            Wt = torch.from_numpy(wq_inputs.weight_bf16(N, K, 0.02).view(np.int16)).view(torch.bfloat16).to(dev)
            q8, s8, _ = wq.wq_quantize_rtn_g128(Wt, 8, K, False)
            base8.append((q8, s8))
            del Wt
        set8 = sum(q.numel() + 2 * s.numel() for q, s in base8)
        n8 = max(2, math.ceil(3 * l2 / set8))
        sets8 = [[(q.clone(), s.clone()) for q, s in base8] for _ in range(n8)]
        tot_b, tot_us = 0, 0.0
        for j, (N, K) in enumerate(SHAPES):
            k = [0]

            def one8(j=j, k=k):
                q, s = sets8[k[0] % n8][j]
                k[0] += 1
                wq.wq_w8a16_gemm(X[j], q, s, Y=Y[j])
            tot_us += graph_time_us(one8, 4 * n8)
            tot_b += N * K + 2 * N + 2 * K + 2 * N  # codes, scales, x, y
        secondary["w8a16_decode_M1_GB/s"] = round(tot_b / tot_us / 1e3, 1)
        del sets8, base8
    except wq.WQError as e:
        secondary["w8a16_decode_M1_GB/s"] = f"unavailable: {e}"

    # ---- secondary: quantizer over the 70B-class weights, then the 70B decode layer
    # (M = 1, 8, 32) on the two quantized matrices, alternating (250 MB > L2)
    qres, q70 = {}, []
    for (N, K) in wq_inputs.SHAPES_70B:
        Wt = (torch.randn(N, K, device=dev) * 0.015).to(torch.bfloat16)
        p = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((N, K // 128), dtype=torch.float16, device=dev)
        z = torch.empty_like(s)
        us = graph_time_us(lambda: wq.wq_quantize_rtn_g128(Wt, packed=p, S=s, Z=z), 5)
        qb = N * K * 2 + N * K // 2 + 4 * N * (K // 128)
        qres[f"{N}x{K}"] = {"us": round(us, 1), "GB/s": round(qb / us / 1e3, 1)}
        q70.append((N, K, p, s, z))
        del Wt
    secondary["quantizer_70b"] = qres
    d70 = {}
    for M in (1, 8, 32):
        Xs = [torch.from_numpy(wq_inputs.act_bf16(M, K).view(np.int16)).view(torch.bfloat16).to(dev)
              for (_, K, _, _, _) in q70]
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for (N, _, _, _, _) in q70]

        def both(Xs=Xs, Ys=Ys):
            for j, (N, K, p, s, z) in enumerate(q70):
                wq.wq_w4a16_gemm(Xs[j], p, s, z, 128, Y=Ys[j])
        us = graph_time_us(both, 4)
        b70 = sum(gemv_bytes(M, N, K) for (N, K, _, _, _) in q70)
        d70[f"M{M}"] = {"us_per_pair": round(us, 1), "GB/s": round(b70 / us / 1e3, 1),
                        "frac": round(b70 / us / 1e3 / peaks["hbm_gbs"], 4)}
    secondary["decode_70b"] = dict(d70, shapes="28672x8192 + 8192x28672 per step")
    del q70
    assert wq.wq_get_status() == 0

    # ---- secondary: outlier stress (C3): W 4096 x 4096 ~N(0, 0.02) with 0.1% of the input
    # columns x U(20, 100), X 8 x 4096 with the same channels scaled; relative Frobenius errors
    # of the weights and of Y = X W^T after GPU quantization at g = 128, per output channel
    # (g = K) and per tensor. The codes are compared with the oracle in the CPU leg.
    c3, c3_codes = {}, {}
    Wb3, Xb3, cols3 = wq_inputs.outlier_config(N=4096, K=4096, M=8)
    W3 = torch.from_numpy(Wb3.view(np.int16)).view(torch.bfloat16).to(dev)
    X3 = torch.from_numpy(Xb3.view(np.int16)).view(torch.bfloat16).to(dev)
    W3d, X3d = W3.double(), X3.double()
    Y3ref = X3d @ W3d.T
    for name, group in (("g128", 128), ("per_channel", 4096), ("per_tensor", 0)):
        if group:
            pk3, s3, z3 = wq.wq_quantize_rtn_g128(W3, 4, group, True)
        else:
            pk3, s3, z3 = wq.wq_quantize_rtn_per_tensor(W3)
        What3 = wq.wq_dequant(pk3, s3, z3, group, torch.float32).double()
        Y3 = wq.wq_w4a16_gemm(X3, pk3, s3, z3, group).double()
        c3[name] = {
            "weight_rel_err": round(float((W3d - What3).norm() / W3d.norm()), 6),
            "output_rel_err": round(float((Y3ref - Y3).norm() / Y3ref.norm()), 6)}
        c3_codes[name] = (group, pk3.cpu().numpy(), s3.cpu().numpy().view(np.uint16),
                          z3.cpu().numpy().view(np.uint16))
    assert wq.wq_get_status() == 0
    c3["weight_err_order_g128_lt_channel_lt_tensor"] = bool(
        c3["g128"]["weight_rel_err"] < c3["per_channel"]["weight_rel_err"]
        < c3["per_tensor"]["weight_rel_err"])
    c3["outlier_columns"] = [int(c) for c in cols3]
    secondary["c3_outlier"] = c3
    del W3, X3, W3d, X3d, Y3ref

    # ---- secondary: prefill GEMM (tensor cores)
    prefill = None
    try:
        P = wq_inputs.PREFILL
        Wt = (torch.randn(P["N"], P["K"], device=dev) * 0.02).to(torch.bfloat16)
        pk, s, z = wq.wq_quantize_rtn_g128(Wt)
        Xp = torch.randn(P["M"], P["K"], device=dev).to(torch.bfloat16)
        Yp = torch.empty((P["M"], P["N"]), dtype=torch.bfloat16, device=dev)
        us = graph_time_us(lambda: wq.wq_w4a16_gemm(Xp, pk, s, z, 128, Y=Yp), 10)
        tflops = 2.0 * P["M"] * P["N"] * P["K"] / us / 1e6
        prefill = {"us": round(us, 1), "TFLOP/s": round(tflops, 1),
                   "peak": peaks["bf16_tflops"], "frac": round(tflops / peaks["bf16_tflops"], 4),
                   "shape": "M=2048 N=11008 K=4096"}
        q8, s8, _ = wq.wq_quantize_rtn_g128(Wt, 8, P["K"], False)
        us8 = graph_time_us(lambda: wq.wq_w8a16_gemm(Xp, q8, s8, Y=Yp), 10)
        tf8 = 2.0 * P["M"] * P["N"] * P["K"] / us8 / 1e6
        prefill["w8a16"] = {"us": round(us8, 1), "TFLOP/s": round(tf8, 1),
                            "frac": round(tf8 / peaks["bf16_tflops"], 4)}
        del Wt, pk, s, z, Xp, Yp, q8, s8
    except Exception as e:  # the tensor-core path may be missing
        prefill = f"unavailable: {e}"
    secondary["prefill"] = prefill

    # ---- secondary: offline quantization variants on one 7B-class layer (11008 x 4096):
    # scale folding (SmoothQuant factors from 64 calibration tokens, the folded quantizer, X/s)
    # and GPTQ (512 calibration tokens; 1024 x 1024 and the full layer's 4096 x 4096 slice)
    offline = {}
    try:
        Wt = (torch.randn(11008, 4096, device=dev) * 0.02).to(torch.bfloat16)
        Xc = torch.randn(64, 4096, device=dev).to(torch.bfloat16)
        sf = wq.wq_smooth_scales(wq.wq_channel_stat(Xc, wq.WQ_STAT_ABSMAX),
                                 wq.wq_channel_stat(Wt, wq.WQ_STAT_ABSMAX), 0.5)
        pk, s, z = wq.wq_quantize_rtn_scaled(Wt, sf)
        us = graph_time_us(lambda: wq.wq_quantize_rtn_scaled(Wt, sf, packed=pk, S=s, Z=z), 5)
        fold_b = Wt.numel() * 2 + 4 * 4096 + pk.numel() + 4 * s.numel()
        offline["quantize_rtn_scaled_11008x4096"] = {"us": round(us, 1),
                                                     "GB/s": round(fold_b / us / 1e3, 1)}
        g_times = {}
        for (n, k) in ((1024, 1024), (4096, 4096)):
            Wg = Wt[:n, :k].contiguous()
            Xg = torch.randn(512, k, device=dev).to(torch.bfloat16)
            ws = torch.empty(wq.wq_gptq_workspace_bytes(n, k), dtype=torch.uint8, device=dev)
            wq.wq_quantize_gptq(Wg, Xg, workspace=ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            wq.wq_quantize_gptq(Wg, Xg, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            g_times[f"{n}x{k}_T512_ms"] = round(e0.elapsed_time(e1), 2)
            del Wg, Xg, ws
        offline["gptq"] = g_times
        assert wq.wq_get_status() == 0
        del Wt, Xc, sf, pk, s, z
    except Exception as e:
        offline = f"unavailable: {e}"
    secondary["offline_quantizers"] = offline

    # ---- e2e: through the public API with host buffers per step: the step's three X rows
    # arrive in one pinned buffer (one H2D copy) and its three Y rows leave in one (one D2H)
    kx = [x.shape[1] for x in X]
    ny = [y.shape[1] for y in Y]
    Xh_all = torch.cat([x.cpu() for x in X], dim=1).pin_memory()
    Xd_all = torch.empty_like(Xh_all, device=dev)
    Yd_all = torch.empty((1, sum(ny)), dtype=torch.bfloat16, device=dev)
    Yh_all = torch.empty((1, sum(ny)), dtype=torch.bfloat16).pin_memory()
    Xd = list(torch.split(Xd_all, kx, dim=1))
    Yd = list(torch.split(Yd_all, ny, dim=1))
    h2d = Xh_all.numel() * 2
    d2h = Yh_all.numel() * 2
    cur = torch.cuda.current_stream()

    def e2e_step(i):
        Xd_all.copy_(Xh_all, non_blocking=True)
        for j, (p, s, z) in enumerate(sets[i % nsets]):
            wq.wq_w4a16_gemm(Xd[j], p, s, z, 128, Y=Yd[j])
        Yh_all.copy_(Yd_all, non_blocking=True)
        cur.synchronize()

    for i in range(3):
        e2e_step(i)
    barrier(world)
    t0 = time.perf_counter()
    for i in range(args.steps):
        e2e_step(i)
    t_e2e = max_over_ranks(time.perf_counter() - t0, world)
    e2e = {"value": round(step_bytes * args.steps * world / t_e2e / 1e9, 2), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "note": "host wall clock; per step: one H2D copy of the three X rows from pinned "
                   "memory, 3 wq_w4a16_gemm calls via the Python binding, one D2H copy of "
                   "the three Y rows, stream sync; weights resident (quantized once)"}

    if rank == 0:
        # DRAM traffic per step from the committed ncu capture, only while the decode kernels'
        # sources are the ones it was taken with (else null)
        traffic = None
        tf = os.path.join(ROOT, "profiles", "gemv_traffic.json")
        if os.path.exists(tf):
            with open(tf) as f:
                rec = json.load(f)
            if rec.get("sources_sha256") == decode_sources_sha256():
                traffic = rec.get("bytes_per_step")
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": 1, "group": 128,
                       "l2": f"inputs larger than L2: {nsets} rotating weight sets, "
                             f"{nsets * set_bytes / 1e6:.0f} MB vs L2 {l2 / 1e6:.0f} MB",
                       "bytes_per_step": step_bytes, "parallelism": f"replicas x{world}",
                       "graphs": "steps replayed from CUDA graphs uploaded before the timed "
                                 "region" if uploaded else "steps replayed from CUDA graphs "
                                 "(upload unavailable: the first replay includes it)"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                         "peak_source": peak_src,
                         "kernel": "gemv_imma_bulk (4096x4096, 11008x4096) + gemv_tma "
                                   "integer path (4096x11008), M=1"},
            "per_shape": per_shape,
            "secondary": secondary,
            "clocks": dict(clk.summary(), **({"soak_steps_after_timed_region": soak}
                                             if soak else {})),
            "e2e": e2e,
            "gpu_launches": len(SHAPES) * args.steps,
            "cpu_baseline": cpu_baseline() if not args.no_cpu_baseline else None,
        }
        if not args.no_cpu_baseline:
            secondary["c3_outlier"]["bitexact_vs_oracle"] = c3_oracle_parity(Wb3, c3_codes)
        print(json.dumps(line), flush=True)
    del plan, g_warm
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


CASES = ("quantize_70b", "gemv_m1_7b", "gemv_m4_7b", "gemv_m16_7b", "gemv_m1_70b", "gemv_m8_70b",
         "prefill", "prefill_w8")


DECODE_SOURCES = ("gemv.cu", "gemv_imma.cu", "gemv_tma.cu", "imma_digits.cuh", "mma_frag.cuh",
                  "ptx.cuh", "common.cuh")


def decode_sources_sha256():
    """Hash of the sources the M = 1 decode kernels compile from (csrc/ of the package)."""
    import hashlib

    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "w4a16_dequant_matmul_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def run_case(name, reps):
    """Launch one kernel family `reps` times on one named workload, untimed, for a profiler
    to capture (e.g. ncu -k <kernel> -s <skip> -c <count> python bench.py --case NAME)."""
    import torch

    import w4a16_dequant_matmul_b200 as wq

    wq.build_library()
    dev = torch.device("cuda", torch.cuda.current_device())

    def bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    if name == "quantize_70b":
        N, K = wq_inputs.SHAPES_70B[0]
        Wt = (torch.randn(N, K, device=dev) * 0.015).to(torch.bfloat16)
        p = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((N, K // 128), dtype=torch.float16, device=dev)
        z = torch.empty_like(s)
        for _ in range(reps):
            wq.wq_quantize_rtn_g128(Wt, packed=p, S=s, Z=z)
    elif name.startswith("gemv_m"):
        M = int(name[len("gemv_m"):].split("_")[0])
        work = []
        for (N, K) in (wq_inputs.SHAPES_70B if name.endswith("_70b") else SHAPES):
            packed, S, Z = wq.wq_quantize_rtn_g128(bf16(wq_inputs.weight_bf16(N, K, 0.02)))
            work.append((bf16(wq_inputs.act_bf16(M, K)), packed, S, Z))
        for _ in range(reps):
            for (X, packed, S, Z) in work:
                wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    else:
        P = wq_inputs.PREFILL
        Wt = (torch.randn(P["N"], P["K"], device=dev) * 0.02).to(torch.bfloat16)
        Xp = torch.randn(P["M"], P["K"], device=dev).to(torch.bfloat16)
        if name == "prefill":
            pk, s, z = wq.wq_quantize_rtn_g128(Wt)
            for _ in range(reps):
                wq.wq_w4a16_gemm(Xp, pk, s, z, 128)
        else:
            q, s, _ = wq.wq_quantize_rtn_g128(Wt, 8, P["K"], False)
            for _ in range(reps):
                wq.wq_w8a16_gemm(Xp, q, s)
    torch.cuda.synchronize()
    st = wq.wq_get_status()
    print(f"case {name}: {reps} reps, status {st}")
    return 0 if st == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="libwq", choices=["libwq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-soak", action="store_true",
                    help="no clock soak after a short timed region (for profiler runs)")
    ap.add_argument("--case", choices=CASES,
                    help="only launch this workload's kernel --case-reps times (profiling)")
    ap.add_argument("--case-reps", type=int, default=3)
    args = ap.parse_args()
    if args.case:
        return run_case(args.case, args.case_reps)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
