"""Throughput of the ConvRot256 INT8 linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step is one forward of the whole path on one batch: the fused
ConvRot256 rotate + per-row INT8 quantiser over X [M, K] (bf16), then the
tcgen05 INT8 GEMM with the fused scale/bias/BF16 epilogue into Y [M, N].
The weights are prepared once before timing (offline weight rotation and
quantisation, as the method stores them). Default workload: the QKV-style
projection M32700/K5376/N16128 (the shape the sglang PR "Tune Kitchen INT8
row splitting for SM120" times in its Benchmark & Profiling table).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream (one pair per kernel), with a 256 MiB write between
steps to flush the 126 MB L2; barrier + synchronize around the region; the
max over ranks. Ranks (torchrun, one per GPU) each run their own batch of M
rows against their own copy of the weights: rows are independent, so there
is no collective on the data path ("replicas", weak scaling).

Rank 0 prints ONE JSON line. `--impl reference` times the CPU oracle (plain
C, OpenMP over rows) on a bounded sample of rows of the same workload.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "INT8 linear TOPS (2MNK/s): ConvRot256 rotate+quantize + INT8 GEMM + epilogue"
UNIT = "TOPS"
PAGE_MS = {"qkv_m32700_k5376_n16128": 10.5752, "ragged_m8193_k5376_n16128": 2.7743}
L2_FLUSH_BYTES = 256 << 20
NOMINAL_INT8_OVER_BF16 = 2.0  # dense tensor peaks: 4.5 POPS int8 / 2.25 PFLOP/s bf16
NOMINAL_FP4_OVER_BF16 = 4.0  # 9 PFLOP/s dense fp4 / 2.25 PFLOP/s bf16


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------- ranks


def shard_rows(M: int, rank: int, world: int):
    """Contiguous, balanced rows [lo, hi) of an M-row batch owned by `rank`
    when the rows are split over `world` ranks (strong scaling). Rows of the
    linear are independent, so no collective is needed on the data path."""
    base, rem = divmod(M, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (timings are
    reported as the slowest rank's). A no-op without a process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.lines: list[tuple[float, str]] = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return

        def pump():
            for line in self.proc.stdout:
                self.lines.append((time.time(), line.strip()))

        self.thread = threading.Thread(target=pump, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 10:
            time.sleep(0.05)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [l for (t, l) in self.lines if t0 <= t <= t1 + 0.05]
        if not rows:
            rows = [l for (_, l) in self.lines[-3:]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in rows:
            f = [x.strip() for x in l.split(",")]
            try:
                sm.append(float(f[2]))
                smax.append(float(f[3]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle


NORM_EPS = 1e-6


def norm_inputs(cfg, M):
    """Residual [M, K] and RMSNorm weight [K] of the --path norm workload
    (bf16, seeded from the config's seed)."""
    import torch

    g = torch.Generator().manual_seed(cfg.seed + 1000)
    R = torch.randn(M, cfg.K, generator=g).to(torch.bfloat16)
    w = (1.0 + 0.25 * torch.randn(cfg.K, generator=g)).to(torch.bfloat16)
    return R, w


def oracle_sample(cfg, X_bits, Qw, s_w, bias_bits, seconds: float, act: str = "none",
                  norm=None):
    """Time the oracle on a bounded sample of rows (quantise + linear rows;
    with ``norm`` = (residual bits, weight bits) the input RMSNorm first).
    Returns (TOPS, rows, seconds, threads)."""
    import oracle

    def run(rows):
        t = time.perf_counter()
        Xs = X_bits[:rows]
        if norm is not None:
            Xs, _ = oracle.rmsnorm_rows(Xs, norm[0][:rows], norm[1], NORM_EPS)
        Qx, s_x = oracle.quantize_rows_bf16(Xs, act=act)
        oracle.linear_rows(Qx, s_x, Qw, s_w, bias_bits, np.arange(rows))
        return time.perf_counter() - t

    probe = 8
    target = 1.25 * seconds
    run(probe)  # first touch of the weights, thread start-up
    dt = run(probe)
    rows = int(max(probe, min(cfg.M, probe * target / max(dt, 1e-6))))
    dt = run(rows)
    if dt < seconds and rows < cfg.M:
        # a probe of 8 rows leaves most host threads idle: size again from this run
        rows = int(max(probe, min(cfg.M, rows * target / max(dt, 1e-6))))
        dt = run(rows)
    tops = 2.0 * rows * cfg.N * cfg.K / dt / 1e12
    return tops, rows, dt, oracle.num_threads()


def oracle_inputs(cfg):
    import oracle

    X, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = oracle.rotate_quant_weight(W.numpy())
    return workloads.bf16_bits(X), Qw, s_w, workloads.bf16_bits(bias)


def run_reference(args, cfg, rank, world):
    """The oracle, as it stands, on the host cores: each step quantises a
    bounded sample of the batch's rows and computes all N outputs of those
    rows (the path chosen by --path)."""
    if rank != 0:
        return 0
    import oracle

    X, W, bias = workloads.make_inputs(cfg)
    X_bits, bias_bits = workloads.bf16_bits(X), workloads.bf16_bits(bias)
    if args.path == "nvfp4":
        Qw, Sw, s_tw = oracle.rotate_quant_weight_nvfp4(W.numpy())

        def run(rows):
            Qa, Sa, s_ta = oracle.quantize_rotate_nvfp4(X_bits[:rows])
            oracle.nvfp4_linear_rows(Qa, Sa, s_ta, Qw, Sw, s_tw, bias_bits)
        what, dtype = "ConvRot NVFP4 quantisation of those rows + their outputs", "fp4-e2m1"
    elif args.path == "w4a4":
        Qw4, s_w = oracle.rotate_quant_weight_int4(W.numpy())

        def run(rows):
            oracle.convrot_w4a4_linear(X_bits[:rows], Qw4, s_w, bias_bits)
        what, dtype = "convrot_w4a4_linear of those rows", "int8"
    elif args.path == "norm":
        Qw, s_w = oracle.rotate_quant_weight(W.numpy())
        R, w = norm_inputs(cfg, cfg.M)
        R_bits, w_bits = workloads.bf16_bits(R), workloads.bf16_bits(w)

        def run(rows):
            Xn, _ = oracle.rmsnorm_rows(X_bits[:rows], R_bits[:rows], w_bits, NORM_EPS)
            Qx, s_x = oracle.quantize_rows_bf16(Xn)
            oracle.linear_rows(Qx, s_x, Qw, s_w, bias_bits, np.arange(rows))
        what, dtype = ("input RMSNorm with residual, quantize_and_rotate_rowwise and the outputs "
                       "of those rows"), "int8"
    else:
        Qw, s_w = oracle.rotate_quant_weight(W.numpy())

        def run(rows):
            Qx, s_x = oracle.quantize_rows_bf16(X_bits[:rows], act=args.act)
            oracle.linear_rows(Qx, s_x, Qw, s_w, bias_bits, np.arange(rows))
        what, dtype = "quantize_and_rotate_rowwise of those rows + their outputs", "int8"
    total_budget = 150.0
    per_step = total_budget / max(1, args.steps + args.warmup)
    run(4)  # first touch of the weights, thread start-up
    t_probe = time.perf_counter()
    run(16)
    t_row = (time.perf_counter() - t_probe) / 16
    rows = int(max(1, min(cfg.M, per_step / max(t_row, 1e-9))))
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        run(rows)
        dt = time.perf_counter() - t
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    tops = 2.0 * rows * cfg.N * cfg.K / (ms / 1e3) / 1e12
    sample = (f"{rows} of {cfg.M} rows per step ({what}, all {cfg.N} outputs each), oracle in "
              f"plain C on host cores")
    line = {"metric": METRIC, "value": tops, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype, "data": "synthetic", "impl": "reference",
            "config": config_dict(cfg, world, "weak", args.act, args.path),
            "cpu_baseline": {"value": tops, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": tops, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def config_dict(cfg, world, scaling="weak", act="none", path="int8"):
    par = (f"replicas x{world}: every rank runs the whole batch" if scaling == "weak"
           else f"rows split over {world} ranks")
    return {"workload": cfg.name, "M": cfg.M, "K": cfg.K, "N": cfg.N, "seed": cfg.seed,
            "x_dist": cfg.x_dist, "outlier_channels": cfg.n_outlier,
            "parallelism": par + " (rows are independent: no collective on the data path)",
            "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write); X is also larger than L2",
            "weights": "rotated + quantised once before timing (offline)",
            "input_act": act, "path": path,
            **({"input_norm": f"RMSNorm with a residual and a weight, eps {NORM_EPS} (residual "
                              f"~ N(0, 1), weight ~ 1 + N(0, 0.25^2), seed + 1000)"}
               if path == "norm" else {})}


# ---------------------------------------------------------------- GPU arm


def run_ours(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import int8_quantized_linear_convrot256_b200 as ck

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    P = peaks()

    X, W, bias = workloads.make_inputs(cfg)
    if args.scaling == "strong":
        lo, hi = shard_rows(cfg.M, rank, world)
        X = X[lo:hi].contiguous()
    Xd = X.to(dev)
    bd = bias.to(dev)
    Wcpu = W
    M, N, K = X.shape[0], cfg.N, cfg.K
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ck.clear_device_error()
    rows = (lo, hi) if args.scaling == "strong" else None
    pth = make_path(ck, args.path, args.act, cfg, Xd, W, bd, Y, dev, rows)
    quantize, gemm = pth["quantize"], pth["gemm"]
    Qw, s_w = pth["Qw"], pth["s_w"]
    ws = torch.empty((ck.workspace_bytes(M, K),), dtype=torch.uint8, device=dev)

    def step():
        quantize()
        gemm()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        quantize()
        ev[i][1].record(stream)
        gemm()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall1 = time.time()
    status = ck.device_error()
    if status != ck.CK_OK:
        clocks.stop()
        raise RuntimeError(f"device error during the timed region: {ck.status_string(status)}")

    # ---- the quantiser by itself (context for its in-step time: here no GEMM
    # runs right before it, so the SM clock has not just been held at the
    # power cap; a second of idle lets the board settle first, and it runs
    # before the MMA-only probe below, which loads the board the same way)
    time.sleep(1.0)
    q_alone = []
    for _ in range(SUBPATH_STEPS):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        quantize()
        e1.record(stream)
        torch.cuda.synchronize()
        q_alone.append(e0.elapsed_time(e1))
    ms_q_alone = sorted(q_alone)[len(q_alone) // 2]

    probe_tops = None
    probe_clocks = None
    if args.path in ("int8", "norm") and not args.no_probe:
        t_p0 = time.time()
        probe_tops = max_over_ranks([i8_probe_tops(ck, stream)], dev)[0]
        probe_clocks = clocks.summary(t_p0, time.time())
    clocks.stop()

    q_ms = [e[0].elapsed_time(e[1]) for e in ev]
    g_ms = [e[1].elapsed_time(e[2]) for e in ev]
    s_ms = [e[0].elapsed_time(e[2]) for e in ev]
    ms_step = sum(s_ms) / len(s_ms)
    ms_q = sum(q_ms) / len(q_ms)
    ms_g = sum(g_ms) / len(g_ms)
    srt = sorted(s_ms)
    spread = [srt[len(srt) // 2], srt[0], srt[-1]]  # median, min, max of the steps
    ms_step, ms_q, ms_g, *spread = max_over_ranks([ms_step, ms_q, ms_g, *spread], dev)


    # ---- end to end through the public composite call, host buffers
    if args.no_e2e or args.path in ("w4a4", "nvfp4", "norm"):
        ms_e2e = float("nan")
    else:
        ms_e2e = run_e2e(args, X, Xd, Qw, s_w, bd, Y, ws, stream, world, dev)
    del pth, quantize, gemm, ws

    # ---- the other paths of the same workload, briefly (one GPU, default path)
    subpaths = None
    if world == 1 and args.path == "int8" and args.act == "none" and not args.no_subpaths:
        del Qw, s_w
        subpaths = {}
        for sp in ("norm", "w4a4", "nvfp4"):
            sub = make_path(ck, sp, "none", cfg, Xd, W, bd, Y, dev, None)
            for _ in range(3):
                flush.zero_()
                sub["quantize"]()
                sub["gemm"]()
            sq, sg, ss_ = time_steps(sub["quantize"], sub["gemm"], flush, SUBPATH_STEPS, stream)
            del sub
            torch.cuda.synchronize()
            subpaths[sp] = path_record(sp, cfg, M, P, sq, sg, ss_)
        if ck.device_error() != ck.CK_OK:
            raise RuntimeError("device error while timing the other paths")
    return report(args, cfg, rank, world, P, X, Wcpu, bias, ms_step, ms_q, ms_g, ms_e2e,
                  clocks, t_wall0, t_wall1, spread, probe_tops, probe_clocks, subpaths,
                  ms_q_alone)


SUBPATH_STEPS = 10


def make_path(ck, path, act, cfg, Xd, W, bd, Y, dev, rows):
    """Device inputs and the two launches (quantiser, GEMM) of one path's step
    on the workload: weights prepared offline first (rotated and quantised;
    for w4a4 also unpacked once); `rows` = (lo, hi) keeps that row shard."""
    import torch

    M, N, K = Xd.shape[0], cfg.N, cfg.K
    d = {}
    if path == "w4a4":
        # packed INT4 weights, unpacked to int8 codes once (offline, like the
        # rotation and quantisation of the weights)
        Qw4, s_w = ck.rotate_quant_weight_int4(W.to(dev))
        Qw = ck.unpack_int4(Qw4)
        del Qw4
    elif path == "nvfp4":
        Qw, Sw, s_w = ck.rotate_quant_weight_nvfp4(W.to(dev))
    else:
        Qw, s_w = ck.rotate_quant_weight(W.to(dev))
    if path == "nvfp4":
        Qx = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        Sx = torch.empty((ck.nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device=dev)
        s_x = torch.empty((1,), dtype=torch.float32, device=dev)
    else:
        Qx = torch.empty((M, K), dtype=torch.int8, device=dev)
        s_x = torch.empty((M,), dtype=torch.float32, device=dev)
    if path == "norm":
        R, w_norm = norm_inputs(cfg, cfg.M)
        if rows is not None:
            R = R[rows[0]:rows[1]].contiguous()
        Rd, gd = R.to(dev), w_norm.to(dev)
        Ro = torch.empty_like(Rd)  # the residual output (a separate buffer: steps stay equal)

    def quantize():
        if path == "w4a4":
            # convrot_w4a4_linear on the unpacked weights: INT4 codes of X
            ck.quantize_rotate_rowwise_int4(Xd, Qx, s_x)
        elif path == "nvfp4":
            ck.quantize_rotate_nvfp4(Xd, Qx, Sx, s_x)
        elif path == "norm":
            # int8_linear's input RMSNorm and residual inside the quantiser
            ck.quantize_rotate_rowwise_norm(Xd, Rd, gd, NORM_EPS, residual_out=Ro, Qx=Qx, s_x=s_x)
        elif act == "none":
            ck.quantize_rotate_rowwise(Xd, Qx, s_x)
        else:
            ck.quantize_rotate_rowwise_act(Xd, act, Qx, s_x)

    def gemm():
        if path == "nvfp4":
            ck.nvfp4_gemm(Qx, Sx, s_x, Qw, Sw, s_w, bd, out=Y)
        else:
            ck.int8_gemm_rowscale(Qx, s_x, Qw, s_w, bd, out=Y)

    d.update(quantize=quantize, gemm=gemm, Qw=Qw, s_w=s_w)
    return d


def time_steps(quantize, gemm, flush, steps, stream):
    """Per-step CUDA-event times (quantiser, GEMM, step) in ms, L2 flushed
    between steps."""
    import torch

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        quantize()
        ev[i][1].record(stream)
        gemm()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    return ([e[0].elapsed_time(e[1]) for e in ev], [e[1].elapsed_time(e[2]) for e in ev],
            [e[0].elapsed_time(e[2]) for e in ev])


def path_bytes_and_peak(path, M, K, P):
    """Algorithmic bytes of a path's quantiser launch, and its GEMM's peak."""
    if path == "nvfp4":
        # bf16 X read once (the absmax pass's re-read is not algorithmic),
        # packed FP4 codes and one E4M3 scale per 16 values written
        return 2.0 * M * K + 0.5 * M * K + M * K / 16.0 + 4.0, P["bf16_tflops"] * NOMINAL_FP4_OVER_BF16
    if path == "norm":
        # X and the residual read, the residual output, codes and row scales
        # written (the normalised rows never reach memory)
        return 7.0 * M * K + 4.0 * M, P["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    return 3.0 * M * K + 4.0 * M, P["bf16_tflops"] * NOMINAL_INT8_OVER_BF16


def path_record(path, cfg, M, P, q_ms, g_ms, s_ms):
    n = len(s_ms)
    ms_q, ms_g, ms_s = sum(q_ms) / n, sum(g_ms) / n, sum(s_ms) / n
    ops = 2.0 * M * cfg.N * cfg.K
    q_bytes, gpeak = path_bytes_and_peak(path, M, cfg.K, P)
    return {"steps": n, "ms_per_step": ms_s, "tops": ops / (ms_s / 1e3) / 1e12,
            "gemm": {"ms_per_launch": ms_g, "tops": ops / (ms_g / 1e3) / 1e12,
                     "frac": ops / (ms_g / 1e3) / 1e12 / gpeak, "peak": gpeak},
            "quantizer": {"ms_per_launch": ms_q, "bytes_per_launch": q_bytes,
                          "gbs": q_bytes / (ms_q / 1e3) / 1e9,
                          "frac": q_bytes / (ms_q / 1e3) / 1e9 / P["hbm_gbs"]},
            "launches_per_step": 2}


PROBE_MMAS = 50_000


def i8_probe_tops(ck, stream):
    """The device's INT8 tensor-core ceiling (ck_test_i8_mma_peak: back-to-back
    pair MMAs of the GEMM's shape, no memory traffic), best of five ~4 ms
    launches after one warm-up, timed with events on the launching stream
    (short bursts: MMA-only load reaches the power cap within milliseconds)."""
    import torch

    ck.test_i8_mma_peak(PROBE_MMAS // 10, stream=stream)
    best = 0.0
    for _ in range(5):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ops = ck.test_i8_mma_peak(PROBE_MMAS, stream=stream)
        e1.record(stream)
        e1.synchronize()
        best = max(best, ops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    return best


E2E_CHUNK_ROWS = 2048


def run_e2e(args, X, Xd, Qw, s_w, bd, Y, ws, stream, world, dev):
    """The same linear through the host-buffer entry point: X from pinned host
    memory, Y back into pinned host memory, chunks of rows pipelined so the
    copies in, the kernels and the copies out overlap (ck_int8_linear_host)."""
    import torch
    import torch.distributed as dist

    import int8_quantized_linear_convrot256_b200 as ck

    M, N = Y.shape
    K = X.shape[1]
    X_host = X.pin_memory()
    Y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    chunk = min(E2E_CHUNK_ROWS, M)
    hws = torch.empty(ck.host_workspace_bytes(chunk, N, K), dtype=torch.uint8, device=Qw.device)
    e2e_steps = max(1, min(args.steps, 10))
    for _ in range(2):
        ck.int8_linear_host(X_host, Qw, s_w, bd, out=Y_host, chunk_rows=chunk, workspace=hws,
                            stream=stream, input_act=args.act)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        ck.int8_linear_host(X_host, Qw, s_w, bd, out=Y_host, chunk_rows=chunk, workspace=hws,
                            stream=stream, input_act=args.act)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / e2e_steps
    return max_over_ranks([ms_e2e], dev)[0]


def report(args, cfg, rank, world, P, X, Wcpu, bias, ms_step, ms_q, ms_g, ms_e2e, clocks,
           t_wall0, t_wall1, spread=None, probe_tops=None, probe_clocks=None, subpaths=None,
           ms_q_alone=None):
    # per-rank work: the full batch (weak, replicas) or this rank's row shard
    # (strong); the job's total is world x per-rank (weak) or the whole batch
    M, N, K = X.shape[0], cfg.N, cfg.K
    ops = 2.0 * M * N * K
    job_ops = world * ops if args.scaling == "weak" else 2.0 * cfg.M * N * K
    value = job_ops / (ms_step / 1e3) / 1e12
    e2e_value = job_ops / (ms_e2e / 1e3) / 1e12
    gemm_tops = ops / (ms_g / 1e3) / 1e12
    q_bytes, int8_peak = path_bytes_and_peak(args.path, M, K, P)
    q_gbs = q_bytes / (ms_q / 1e3) / 1e9
    ratio = NOMINAL_FP4_OVER_BF16 if args.path == "nvfp4" else NOMINAL_INT8_OVER_BF16
    sustained_peak = P["bf16_tflops_sustained"] * ratio
    # DRAM bytes of one launch of the dominant kernel, from an ncu capture of
    # this workload (profiles/<kernel>__<workload>.dram.json), if there is one
    traffic = None
    kname = ("gemm_nvfp4_pair_kernel" if args.path == "nvfp4" else "gemm_i8_pair_kernel") \
        if M > 128 else ("gemm_nvfp4_kernel" if args.path == "nvfp4" else "gemm_i8_kernel")
    prof = os.path.join(ROOT, "profiles", f"{kname}__{cfg.name}.dram.json")
    if os.path.exists(prof) and args.scaling == "weak":
        try:
            traffic = float(json.load(open(prof))["dram_bytes_per_launch"])
        except Exception:
            traffic = None

    line = None
    if rank == 0:
        cpu = None
        # (the w4a4 and nvfp4 paths have their oracle in the reference arm only)
        if world == 1 and not args.no_cpu_baseline and args.path in ("int8", "norm"):
            X_bits = workloads.bf16_bits(X)
            import oracle

            Qw_o, s_w_o = oracle.rotate_quant_weight(Wcpu.numpy())
            norm = None
            if args.path == "norm":
                R_o, w_o = norm_inputs(cfg, cfg.M)  # the same seeded values as on the device
                norm = (workloads.bf16_bits(R_o), workloads.bf16_bits(w_o))
            tops, rows, dt, cores = oracle_sample(cfg, X_bits, Qw_o, s_w_o,
                                                  workloads.bf16_bits(bias), args.cpu_seconds,
                                                  args.act, norm)
            what = "input RMSNorm, " if norm is not None else ""
            cpu = {"value": tops, "unit": UNIT, "cores": cores, "kind": "oracle",
                   "sample": f"{rows} of {cfg.M} rows ({what}rotate+quantise and all {cfg.N} "
                             f"outputs of those rows) in {dt:.1f} s, plain C oracle, OpenMP over "
                             f"rows"}
        page_ms = PAGE_MS.get(cfg.name)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step,
            "ms_per_step_median_min_max": spread,
            "higher_is_better": True,
            "scaling": args.scaling,
            "vs_baseline": value / (2.0 * cfg.M * N * K / (page_ms / 1e3) / 1e12) if page_ms else None,
            "dtype": "fp4-e2m1" if args.path == "nvfp4" else "int8", "data": "synthetic",
            "impl": "ours",
            "config": config_dict(cfg, world, args.scaling, args.act, args.path),
            "roofline": {"kernel": (("gemm_nvfp4_pair_kernel (2-SM " if M > 128 else
                                     "gemm_nvfp4_kernel (") + "tcgen05 kind::mxf4nvf4, E4M3 block "
                                    "scales, fused epilogue)" if args.path == "nvfp4" else
                                    "gemm_i8_pair_kernel (2-SM tcgen05 kind::i8, fused epilogue, "
                                    "TMA store)" if M > 128 else
                                    "gemm_i8_kernel (tcgen05 kind::i8, fused epilogue)"),
                         "bound": "tensor", "achieved": gemm_tops, "peak": int8_peak,
                         "unit": "TFLOP/s", "frac": gemm_tops / int8_peak, "traffic": traffic,
                         "peak_source": f"{P['source']} bf16 burst {P['bf16_tflops']} TFLOP/s x "
                                        + (f"nominal fp4/bf16 ratio {NOMINAL_FP4_OVER_BF16}"
                                           if args.path == "nvfp4" else
                                           f"nominal int8/bf16 ratio {NOMINAL_INT8_OVER_BF16}"),
                         ("frac_of_spec_9000" if args.path == "nvfp4" else "frac_of_spec_4500"):
                             gemm_tops / (9000.0 if args.path == "nvfp4" else 4500.0),
                         "frac_of_measured_sustained": gemm_tops / sustained_peak,
                         **({"i8_probe_tops": probe_tops, "frac_of_i8_probe": gemm_tops / probe_tops,
                             "i8_probe_clocks": probe_clocks}
                            if probe_tops else {}),
                         "ms_per_launch": ms_g},
            "quantizer": {"kernel": ("nvfp4_warp_kernel<1> + <2> (ConvRot256 + NVFP4, two "
                                     "passes over X, staging private to each warp)" if args.path == "nvfp4" else
                                     "quant_norm_bulk_kernel (input RMSNorm with residual "
                                     "fused into ConvRot256 + per-row INT8)"
                                     if args.path == "norm" else
                                     ("quant_rows_bulk_kernel" if K <= 28672 else
                                      "quant_rows_two_pass_kernel") + " (ConvRot256 + per-row INT8)"),
                          "bound": "hbm", "achieved": q_gbs, "peak": P["hbm_gbs"], "unit": "GB/s",
                          "frac": q_gbs / P["hbm_gbs"], "frac_of_spec_8000": q_gbs / 8000.0,
                          "bytes_per_launch": q_bytes, "ms_per_launch": ms_q,
                          **({"alone": {"ms_per_launch": ms_q_alone,
                                        "frac": q_bytes / (ms_q_alone / 1e3) / 1e9 / P["hbm_gbs"],
                                        "note": f"median of {SUBPATH_STEPS} launches timed by "
                                                "themselves after the timed region and a second "
                                                "of idle, L2 flushed before each; not the "
                                                "metric"}}
                             if ms_q_alone else {})},
            "cpu_baseline": cpu,
            "e2e": None if (args.no_e2e or args.path in ("w4a4", "nvfp4", "norm")) else {"value": e2e_value, "unit": UNIT, "ms_per_step": ms_e2e,
                    "h2d_bytes_per_step": int(X.numel() * 2), "d2h_bytes_per_step": int(M * N * 2),
                    "call": f"ck_int8_linear_host: X from and Y to pinned host memory, chunks of "
                            f"{min(E2E_CHUNK_ROWS, M)} rows with copies overlapped with the kernels"},
            "gpu_launches": {"nvfp4": 4}.get(args.path, 2) * args.steps,
            "clocks": clocks.summary(t_wall0, t_wall1),
        }
        if subpaths:
            line["other_paths"] = {
                "note": f"the same workload's other paths, {SUBPATH_STEPS} steps each after 3 "
                        "warm-up steps, timed with CUDA events after the main measurement: norm = "
                        "int8_linear with its input RMSNorm and a residual fused into the "
                        "quantiser; w4a4 = convrot_w4a4_linear (INT4 codes, weights unpacked "
                        "once offline); nvfp4 = ConvRot NVFP4 (two-pass FP4 quantiser, "
                        "block-scaled FP4 GEMM, GEMM peak = 4 x bf16)",
                **subpaths}
    return line


def launch_ranks(args, argv) -> int:
    """Runs this script once per GPU under torch.distributed.run (one process
    per rank, rendezvous on 127.0.0.1) and returns the launcher's status."""
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_dry(args, cfg, rank, world):
    """The rank plumbing without a GPU (gloo): every rank times a small host
    loop for each step, the times are reduced as the max over ranks, and rank
    0 prints a JSON line with the same keys as a real run."""
    import torch.distributed as dist

    times = []
    for i in range(args.warmup + args.steps):
        if world > 1:
            dist.barrier()
        t = time.perf_counter()
        float(np.sum(np.arange(10000, dtype=np.float64)))
        if i >= args.warmup:
            times.append(1e3 * (time.perf_counter() - t))
    ms = max_over_ranks([sum(times) / len(times)])[0]
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": None, "unit": UNIT, "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                          "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None,
                          "dtype": "int8", "data": "synthetic", "impl": args.impl,
                          "dry_run": "gloo ranks on the host, no GPU work",
                          "config": config_dict(cfg, world, args.scaling, args.act, args.path)}),
              flush=True)
    return 0


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs of this node; above 1 the script starts one rank per GPU itself "
                         "(torch.distributed.run) unless it already runs as a rank")
    ap.add_argument("--dry-run", action="store_true",
                    help="exercise the rank launch and the max-over-ranks timing on the host "
                         "(gloo), with no GPU work")
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=workloads.HEADLINE.name, choices=sorted(workloads.BY_NAME))
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: every rank runs the whole batch (replicas); strong: the "
                         "batch's rows are split over the ranks")
    ap.add_argument("--path", default="int8", choices=["int8", "w4a4", "nvfp4", "norm"],
                    help="int8: int8_linear; w4a4: convrot_w4a4_linear (INT4 codes, packed "
                         "INT4 weights unpacked once, offline); nvfp4: ConvRot NVFP4 (two-pass "
                         "FP4 quantiser + block-scaled FP4 GEMM); norm: int8_linear with its "
                         "input RMSNorm and a residual (normalised inside the quantiser)")
    ap.add_argument("--act", default="none", choices=["none", "relu", "silu", "gelu_tanh"],
                    help="input activation folded into the quantiser (int8_linear(input_act=...))")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-subpaths", action="store_true",
                    help="skip the brief timing of the norm, w4a4 and nvfp4 paths that the "
                         "default (int8) run adds to its line")
    ap.add_argument("--no-probe", action="store_true",
                    help="skip the INT8 tensor-core peak probe run after the timed region")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end measurement (profiling runs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args, argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but {world} ranks were started")
    cfg = workloads.BY_NAME[args.workload]

    if args.dry_run:
        import datetime

        import torch.distributed as dist

        if world > 1:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        try:
            return run_dry(args, cfg, rank, world)
        finally:
            if world > 1:
                dist.destroy_process_group()

    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)

    import torch
    import torch.distributed as dist

    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, cfg, rank, world, local_rank)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
