#!/usr/bin/env python3
"""Benchmark of the microscaling FP4 hot path on B200.

One step = one pass of the quantization path over the heavy-tailed
1024 x 131072 bf16 tensor (Student-t(3) with 1% outliers x20):
MXFP4 quantize, NVFP4 quantize (tensor scale computed, i.e. the amax pass
plus the quantize pass), MXFP4 dequantize and NVFP4 dequantize (bf16 out).
`value` = algorithmic bytes of the step / device time of the step (GB/s).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (weak scaling): one process per GPU under torchrun, every rank
runs the same step on its own tensor; value = all ranks' bytes / max time.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

ROWS, COLS = 1024, 131072

# DRAM bytes (read + write) per launch of the roofline kernel at 1024 x 131072:
# dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of the MXFP4
# quantize kernel on 512 rows of this workload, scaled by rows.  Set to None
# whenever that kernel changes, until it is captured again.
QUANT_MX_TRAFFIC_BYTES = 2 * (134_259_712 + 17_949_952)
# Nominal B200 figures the fractions are also given against ("frac_spec"):
# ~8 TB/s HBM3e and ~9 PFLOP/s dense FP4 (the gpt-oss MXFP4 article's B200
# paragraph).  "frac" is always against the measured peaks.
SPEC_HBM_GBS = 8000.0
SPEC_FP4_TFLOPS = 9000.0
WORKLOAD = "quantize sweep 1024x131072 bf16 Student-t(3)+1% outliers x20: MXFP4 + NVFP4 quantize and dequantize"
METRIC = "FP4 quantize GB/s (% HBM peak)"


def step_bytes(rows=ROWS, cols=COLS):
    """Algorithmic HBM bytes of one step (each tensor read or written once per
    kernel pass; the NVFP4 amax pass reads x once more)."""
    n = rows * cols
    mx_q = n * (2 + 0.5 + 1 / 32)          # read x, write nibbles + E8M0 scales
    nv_q = n * (2 + 2 + 0.5 + 1 / 16)      # amax read, read x, write nibbles + E4M3 scales
    mx_d = n * (0.5 + 1 / 32 + 2)          # read nibbles + scales, write bf16
    nv_d = n * (0.5 + 1 / 16 + 2)
    return {"mx_quantize": mx_q, "nv_quantize": nv_q, "mx_dequantize": mx_d, "nv_dequantize": nv_d}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def fp4_tensor_peak():
    """Dense FP4 tensor peak: the measured bf16 GEMM burst figure x 4, the
    nominal fp4 / bf16 ratio (9 / 2.25 PFLOP/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return 4.0 * float(json.load(open(p))["bf16_tflops"]), "measured bf16 burst x 4"
    return 4.0 * 1590.0, "fallback bf16 x 4"


def time_graph(torch, fn, warmup: int, reps: int):
    """Average device time of `fn` (ms) over `reps` launches captured in one
    CUDA graph, after `warmup` captured launches."""
    fn()
    torch.cuda.synchronize()
    gw = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw):
        for _ in range(warmup):
            fn()
    gt = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gt):
        for _ in range(reps):
            fn()
    gw.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    gt.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def bench_rotate(torch, fp4, inputs, dev, reps: int, fmts=None):
    """Fused rotate + quantize of 8192x4096 bf16 activations (Laplace(0,1), 1%
    outlier channels x50), k in {0,16,32,64,128}, MXFP4, NVFP4 and MXFP4 on
    16-element blocks.  Eight input copies (537 MB) are rotated so every call
    reads x from HBM (one fits in L2).  Bytes per element: read 2 + nibbles
    0.5 + scales 1/32 (MX) or 1/16 (NV, MX16); the NVFP4 amax pass re-reads x
    from L2 and is not counted."""
    hbm, kind = peaks()
    x = inputs.rotate_acts()
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    copies = [xd.clone() for _ in range(8)]
    n = xd.numel()
    res = {"peak_gbs": hbm, "peak_kind": kind, "workload": "rotate+quantize 8192x4096 bf16", "cases": {}}
    for fmt, name, bpe in ((fp4.FP4_MXFP4, "mxfp4", 2 + 0.5 + 1 / 32), (fp4.FP4_NVFP4, "nvfp4", 2 + 0.5 + 1 / 16),
                           (fp4.FP4_MXFP4_16, "mxfp4_16", 2 + 0.5 + 1 / 16)):
        if fmts is not None and name not in fmts:
            continue
        outs = fp4.quantize(xd, fmt)
        for k in (0, 16, 32, 64, 128):
            it = [0]

            def call():
                fp4.quantize(copies[it[0] % 8], fmt, hadamard_k=k, out=outs)
                it[0] += 1

            ms = time_graph(torch, call, 3, reps * 8)
            gbs = n * bpe / (ms * 1e-3) / 1e9
            res["cases"][f"{name}_k{k}"] = {"us": ms * 1e3, "gbs": gbs, "frac": gbs / hbm,
                                            "frac_spec": gbs / SPEC_HBM_GBS}
        # the MSE block-scale search (same bytes, more arithmetic per block)
        for k in (0, 128):
            it = [0]

            def call_mse():
                fp4.quantize(copies[it[0] % 8], fmt, hadamard_k=k, out=outs, scale_search=fp4.FP4_SCALE_MSE)
                it[0] += 1

            ms = time_graph(torch, call_mse, 3, reps * 8)
            gbs = n * bpe / (ms * 1e-3) / 1e9
            res["cases"][f"{name}_mse_k{k}"] = {"us": ms * 1e3, "gbs": gbs, "frac": gbs / hbm,
                                                "frac_spec": gbs / SPEC_HBM_GBS}
        # the sparse residual lane (TransFP4 Eq.(3)): 4 more bytes per 32 elements
        for k in (0, 32):
            it = [0]

            def call_res():
                fp4.quantize_residual(copies[it[0] % 8], fmt, hadamard_k=k)
                it[0] += 1

            ms = time_graph(torch, call_res, 3, reps * 8)
            gbs = n * (bpe + 4 / 32) / (ms * 1e-3) / 1e9
            res["cases"][f"{name}_residual_k{k}"] = {"us": ms * 1e3, "gbs": gbs, "frac": gbs / hbm,
                                                     "frac_spec": gbs / SPEC_HBM_GBS}
    del copies, xd
    torch.cuda.empty_cache()
    return res


def bench_l2_encode(torch, fp4, inputs, dev, reps: int):
    """The encode pass of NVFP4 with a computed tensor scale, on its own
    footing: MXFP4 and NVFP4 (a static s_g, so no tensor-maximum pass)
    quantize of one 8192x4096 bf16 tensor (the rotate workload, k = 0) that
    stays in L2 (67 MB).  Three untimed calls of each come first, in that
    order (after one call of each that allocates the outputs): the launches a
    profiler captures.  Then each is timed in a graph of calls on the same
    tensor."""
    hbm, kind = peaks()
    x = inputs.rotate_acts()
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    g = torch.tensor([0.0123], dtype=torch.float32, device=dev)
    om = fp4.quantize(xd, fp4.FP4_MXFP4)
    on = fp4.quantize(xd, fp4.FP4_NVFP4, gscale=g)
    torch.cuda.synchronize()
    for _ in range(3):
        fp4.quantize(xd, fp4.FP4_MXFP4, out=om)
    for _ in range(3):
        fp4.quantize(xd, fp4.FP4_NVFP4, gscale=g, out=on)
    torch.cuda.synchronize()
    res = {"peak_gbs": hbm, "peak_kind": kind, "workload": "quantize 8192x4096 bf16, x in L2", "cases": {}}
    for name, fn in (("mxfp4", lambda: fp4.quantize(xd, fp4.FP4_MXFP4, out=om)),
                     ("nvfp4_static", lambda: fp4.quantize(xd, fp4.FP4_NVFP4, gscale=g, out=on))):
        ms = time_graph(torch, fn, 3, reps * 8)
        res["cases"][name] = {"us": ms * 1e3}
    return res


def bench_decode(torch, fp4, inputs, dev, reps: int, fmts=None, m_list=(1, 4, 16),
                 shapes=((14336, 4096), (4096, 14336))):
    """Decode shapes: M in {1,4,16} bf16 activations quantized online inside
    the timed call (fp4_linear), W 14336x4096 and 4096x14336 pre-quantized,
    BF16 out.  W copies are rotated so the weight stream comes from HBM.  The
    weights are marked static (prepared once, read-only), so each call's
    decode kernel streams its W while the previous call finishes.  Each
    format's weights are also timed with the sparse residual lane
    (fp4_linear_residual, no rotation), the "_residual_" rows."""
    hbm, kind = peaks()
    res = {"peak_gbs": hbm, "peak_kind": kind, "copies": 0, "cases": {}}
    for (N, K) in shapes:
        _, w = inputs.decode_linear(1, N, K)
        wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
        del w
        # the third case is the workload's literal reading: NVFP4 activations
        # against MXFP4 weights, bound once to the NVFP4 scale form
        for fmt, name, wfmt in ((fp4.FP4_NVFP4, "nvfp4", fp4.FP4_NVFP4), (fp4.FP4_MXFP4, "mxfp4", fp4.FP4_MXFP4),
                                (fp4.FP4_NVFP4, "nvfp4act_mxfp4w", fp4.FP4_MXFP4),
                                (fp4.FP4_MXFP4_16, "mxfp4_16", fp4.FP4_MXFP4_16)):
            if fmts is not None and name not in fmts:
                continue
            W0 = fp4.quantize(wd, wfmt)
            if wfmt != fmt:
                W0 = fp4.mx_to_nv(W0)
            wbytes = W0[0].numel() + W0[1].numel()
            copies = max(2, int(2 * 126e6 // wbytes) + 1)
            Ws = [tuple(t.clone() for t in W0) for _ in range(copies)]
            res["copies"] = copies
            for M in m_list:
                a, _ = inputs.decode_linear(M, 8, K)
                x = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
                C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                ws = torch.empty((fp4.linear_workspace_size(M, N, K, fmt),), dtype=torch.uint8, device=dev)
                it = [0]

                def call():
                    W = Ws[it[0] % copies]
                    it[0] += 1
                    fp4.linear(x, W, fmt, out=C, workspace=ws, weights_static=True)

                ms = time_graph(torch, call, 3, reps * copies)
                b = wbytes + M * K * 2 + M * N * 2
                gbs = b / (ms * 1e-3) / 1e9
                res["cases"][f"{name}_M{M}_N{N}_K{K}"] = {"us": ms * 1e3, "gbs": gbs, "frac": gbs / hbm,
                                                          "frac_spec": gbs / SPEC_HBM_GBS}
                if wfmt != fmt:
                    continue

                # the same call with the sparse residual lane (TransFP4 Eq.(3))
                def call_res():
                    W = Ws[it[0] % copies]
                    it[0] += 1
                    fp4.linear_residual(x, W, fmt, out=C, weights_static=True)

                ms = time_graph(torch, call_res, 3, reps * copies)
                gbs = b / (ms * 1e-3) / 1e9
                res["cases"][f"{name}_residual_M{M}_N{N}_K{K}"] = {"us": ms * 1e3, "gbs": gbs, "frac": gbs / hbm,
                                                                   "frac_spec": gbs / SPEC_HBM_GBS}
            del Ws, W0
        del wd
    torch.cuda.empty_cache()
    return res


def bench_prefill(torch, fp4, inputs, dev, reps: int, M: int = 8192, fmts=None):
    """W4A4 prefill GEMM, 70B-MLP shape: A 8192x8192, W 28672x8192, BF16 out."""
    N, K = 28672, 8192
    a, w = inputs.prefill_linear(m=M)
    ad = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
    del a, w
    peak, kind = fp4_tensor_peak()
    out = {"workload": f"prefill W4A4 linear M={M} N={N} K={K}, BF16 out", "peak_tflops": peak, "peak_kind": kind}
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    for fmt, name in ((fp4.FP4_NVFP4, "nvfp4"), (fp4.FP4_MXFP4, "mxfp4"), (fp4.FP4_MXFP4_16, "mxfp4_16")):
        if fmts is not None and name not in fmts:
            continue
        A = fp4.quantize(ad, fmt)
        W = fp4.quantize(wd, fmt)
        ms = time_graph(torch, lambda: fp4.gemm(A, W, M, N, K, fmt, out=C), 3, reps)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[name] = {"ms": ms, "tflops": tf, "frac": tf / peak, "frac_spec": tf / SPEC_FP4_TFLOPS}
        q_ms = time_graph(torch, lambda: fp4.quantize(ad, fmt, out=A), 3, reps)
        out[name]["act_quantize_ms"] = q_ms
        out[name]["tflops_incl_act_quantize"] = 2.0 * M * N * K / ((ms + q_ms) * 1e-3) / 1e12
        # C quantized for the next layer in the GEMM epilogue (NVFP4 with a
        # given tensor scale; MXFP4 for MXFP4_16 operands), against BF16 C
        # followed by a quantize pass.
        ofmt = fp4.FP4_MXFP4 if fmt == fp4.FP4_MXFP4_16 else fmt
        gC = torch.full((1,), 0.05, dtype=torch.float32, device=dev)
        Cq = fp4.gemm_quantized(A, W, M, N, K, fmt, ofmt, gscale=gC if ofmt == fp4.FP4_NVFP4 else None)
        fq_ms = time_graph(torch, lambda: fp4.gemm_quantized(A, W, M, N, K, fmt, ofmt, out=Cq), 3, reps)
        gs = gC if ofmt == fp4.FP4_NVFP4 else None
        Cb = fp4.quantize(C, ofmt, gscale=gs)
        cq_ms = time_graph(torch, lambda: fp4.quantize(C, ofmt, gscale=gs, out=Cb), 3, reps)
        out[name]["quantized_out"] = {"ms": fq_ms, "tflops": 2.0 * M * N * K / (fq_ms * 1e-3) / 1e12,
                                      "frac": 2.0 * M * N * K / (fq_ms * 1e-3) / 1e12 / peak,
                                      "frac_spec": 2.0 * M * N * K / (fq_ms * 1e-3) / 1e12 / SPEC_FP4_TFLOPS,
                                      "unfused_bf16_then_quantize_ms": ms + cq_ms}
        del A, W, Cq, Cb
    del ad, wd, C
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- clocks -----
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.out = out
        return False

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in csv.reader(io.StringIO(self.out)):
            if len(row) < 9:
                continue
            try:
                mhz.append(float(row[1]))
                mx = float(row[2])
            except ValueError:
                continue
            for n, v in zip(names, row[5:9]):
                if v.strip() == "Active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "samples": len(mhz), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- dist -------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, ws: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if ws == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- oracle leg --
def oracle_step(x):
    """Times the CPU oracle (as it stands, OpenMP over rows) on one step."""
    import oracle
    rows = x.shape[0]
    t0 = time.perf_counter()
    qm, sm, _ = oracle.quantize(x, oracle.MXFP4)
    qn, sn, gn = oracle.quantize(x, oracle.NVFP4)
    oracle.dequantize(qm, sm, 1.0, oracle.MXFP4)
    oracle.dequantize(qn, sn, gn, oracle.NVFP4)
    dt = time.perf_counter() - t0
    b = sum(step_bytes(rows, COLS).values())
    return b / dt / 1e9, dt, oracle.num_threads()


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from fp4_microscaling_quantization_b200 import inputs
    oracle.build()
    rows = 256
    x = inputs.quant_sweep(rows=rows, seed=2)
    times = []
    for i in range(args.warmup + args.steps):
        gbs, dt, cores = oracle_step(x)
        if i >= args.warmup:
            times.append(dt)
    dt = statistics.mean(times)
    b = sum(step_bytes(rows, COLS).values())
    v = b / dt / 1e9
    sample = f"{rows} of {ROWS} rows of the same workload per step (oracle, OpenMP over rows)"
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD + f" (oracle sample: {rows} rows)"},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our leg ----
def run_ours(args):
    import torch

    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)

    import fp4_microscaling_quantization_b200 as fp4
    from fp4_microscaling_quantization_b200 import _lib, inputs

    if args.only:
        # profiling helper: one leg alone, no JSON contract
        if args.only == "prefill":
            r = bench_prefill(torch, fp4, inputs, dev, reps=args.steps, M=args.prefill_m, fmts=args.fmts)
        elif args.only == "rotate":
            r = bench_rotate(torch, fp4, inputs, dev, reps=args.steps, fmts=args.fmts)
        elif args.only == "l2-encode":
            r = bench_l2_encode(torch, fp4, inputs, dev, reps=args.steps)
        else:
            kw = {}
            if args.decode_m:
                kw["m_list"] = tuple(args.decode_m)
            if args.decode_nk:
                kw["shapes"] = tuple(tuple(int(v) for v in nk.split("x")) for nk in args.decode_nk)
            r = bench_decode(torch, fp4, inputs, dev, reps=args.steps, fmts=args.fmts, **kw)
        print(json.dumps({"only": args.only, "result": r}), flush=True)
        return 0

    x_np = inputs.quant_sweep(rows=args.rows, seed=2 + rank)
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    x = x_host.to(dev)
    rows, cols = x.shape
    stream = torch.cuda.current_stream(dev)

    qm, sm, gm = fp4.quantize(x, fp4.FP4_MXFP4)
    qn, sn, gn = fp4.quantize(x, fp4.FP4_NVFP4)
    dm = fp4.dequantize(qm, sm, gm, fp4.FP4_MXFP4, out_dtype=fp4.FP4_OUT_BF16)
    dn = fp4.dequantize(qn, sn, gn, fp4.FP4_NVFP4, out_dtype=fp4.FP4_OUT_BF16)
    torch.cuda.synchronize()

    names = ["mx_quantize", "nv_quantize", "mx_dequantize", "nv_dequantize"]

    def step(evs=None, marks=(0, 1, 2, 3, 4)):
        def mark(i):
            if evs is not None and i in marks:
                evs[i].record()
        mark(0)
        fp4.quantize(x, fp4.FP4_MXFP4, out=(qm, sm, gm))
        mark(1)
        fp4.quantize(x, fp4.FP4_NVFP4, out=(qn, sn, gn))
        mark(2)
        fp4.dequantize(qm, sm, gm, fp4.FP4_MXFP4, out_dtype=fp4.FP4_OUT_BF16, out=dm)
        mark(3)
        fp4.dequantize(qn, sn, gn, fp4.FP4_NVFP4, out_dtype=fp4.FP4_OUT_BF16, out=dn)
        mark(4)

    # The W warm-up steps and the K timed steps are each captured once into a
    # CUDA graph (no host work between kernels).  In the timed graph only the
    # MXFP4 quantize call (the roofline kernel, one launch per call) is
    # bracketed by event-record nodes: an event node between two kernels
    # also stops the next one from starting early, so the other call
    # boundaries are left free.  A second graph of the same steps with events
    # between all calls gives the per-call breakdown.
    step()
    torch.cuda.synchronize()
    launches0 = _lib.lib().fp4_kernel_launches()
    g_warm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_warm):
        for _ in range(args.warmup):
            step()
    roof_evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(args.steps)]
    launches1 = _lib.lib().fp4_kernel_launches()
    g_timed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_timed):
        for i in range(args.steps):
            step(roof_evs[i], marks=(0, 1))
    launches = _lib.lib().fp4_kernel_launches() - launches1
    evsets = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(args.steps)]
    g_break = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_break):
        for i in range(args.steps):
            step(evsets[i])
    torch.cuda.synchronize()

    g_warm.replay()
    torch.cuda.synchronize()
    per = {n: 0.0 for n in names}
    with ClockSampler(dev.index) as clk:
        barrier(ws)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        g_timed.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
    total_ms = t0.elapsed_time(t1)
    g_break.replay()
    torch.cuda.synchronize()
    for ev in evsets:
        for j, n in enumerate(names):
            per[n] += ev[j].elapsed_time(ev[j + 1])
    per = {n: v / args.steps for n, v in per.items()}
    total_ms = max_over_ranks(total_ms, ws, dev)
    ms_per_step = total_ms / args.steps

    sb = step_bytes(rows, cols)
    value = sum(sb.values()) * ws / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = peaks()

    # dominant single-launch kernel: MXFP4 quantize is one kernel launch per
    # call, timed inside the timed region
    dom = "mx_quantize"
    dom_ms = sum(ev[0].elapsed_time(ev[1]) for ev in roof_evs) / args.steps
    achieved = sb[dom] / (dom_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "quantize_kernel<MXFP4,k=0>", "achieved": achieved, "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                "frac_spec": achieved / SPEC_HBM_GBS, "peak_spec": SPEC_HBM_GBS,
                "traffic": QUANT_MX_TRAFFIC_BYTES if rows == ROWS else None,
                "launch_ms": dom_ms,
                "per_call_ms": per,
                "per_call_gbs": {n: sb[n] / (per[n] * 1e-3) / 1e9 for n in names}}

    # ---- end to end through the public API with host buffers ----------------
    e2e = None
    if not args.no_e2e:
        outs_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (qm, sm, qn, sn, gn)]
        h2d = x_host.numel() * 2
        d2h = sum(t.numel() * t.element_size() for t in outs_host)
        e_steps = max(2, min(args.steps, 5))
        qm_h, sm_h, qn_h, sn_h, gn_h = outs_host
        CH = 128  # rows per chunk: one 128-row block of the scale tile layout
        chunked = rows % CH == 0 and rows >= 2 * CH
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        nkb4_mx = (cols // 32 + 3) // 4
        sblk = nkb4_mx * 512  # MXFP4 scale bytes of one 128-row block

        def e2e_step():
            """H2D of x, the step, D2H of q/s/g.  With whole 128-row blocks the
            rows go in chunks: each chunk's copy in, MXFP4 quantize and
            dequantize, and copy out run on three streams and overlap with
            the neighbouring chunks; NVFP4, whose tensor scale needs every
            row, runs once all chunks are in."""
            if not chunked:
                x.copy_(x_host, non_blocking=True)
                step()
                for h, d in zip(outs_host, (qm, sm, qn, sn, gn)):
                    h.copy_(d, non_blocking=True)
                return
            start = torch.cuda.Event()
            start.record(stream)
            h2d_s.wait_event(start)
            d2h_s.wait_event(start)
            for c in range(rows // CH):
                r0, r1 = c * CH, (c + 1) * CH
                landed = torch.cuda.Event()
                with torch.cuda.stream(h2d_s):
                    x[r0:r1].copy_(x_host[r0:r1], non_blocking=True)
                    landed.record(h2d_s)
                stream.wait_event(landed)
                q_c, s_c = qm[r0:r1], sm[c * sblk:(c + 1) * sblk]
                fp4.quantize(x[r0:r1], fp4.FP4_MXFP4, out=(q_c, s_c, gm))
                fp4.dequantize(q_c, s_c, gm, fp4.FP4_MXFP4, out_dtype=fp4.FP4_OUT_BF16, out=dm[r0:r1])
                done = torch.cuda.Event()
                done.record(stream)
                d2h_s.wait_event(done)
                with torch.cuda.stream(d2h_s):
                    qm_h[r0:r1].copy_(q_c, non_blocking=True)
                    sm_h[c * sblk:(c + 1) * sblk].copy_(s_c, non_blocking=True)
            fp4.quantize(x, fp4.FP4_NVFP4, out=(qn, sn, gn))
            fp4.dequantize(qn, sn, gn, fp4.FP4_NVFP4, out_dtype=fp4.FP4_OUT_BF16, out=dn)
            nv_done = torch.cuda.Event()
            nv_done.record(stream)
            d2h_s.wait_event(nv_done)
            with torch.cuda.stream(d2h_s):
                for h, d in ((qn_h, qn), (sn_h, sn), (gn_h, gn)):
                    h.copy_(d, non_blocking=True)
                out_done = torch.cuda.Event()
                out_done.record(d2h_s)
            stream.wait_event(out_done)

        e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a0.elapsed_time(a1), ws, dev) / e_steps
        # the chunked copies back hold the whole-tensor results
        ref_q, ref_s, _ = fp4.quantize(x, fp4.FP4_MXFP4)
        torch.cuda.synchronize()
        if not (torch.equal(ref_q.cpu(), qm_h) and torch.equal(ref_s.cpu(), sm_h)
                and torch.equal(qn.cpu(), qn_h) and torch.equal(sn.cpu(), sn_h)):
            raise RuntimeError("end-to-end outputs differ from the device results")
        del ref_q, ref_s
        e2e = {"value": sum(sb.values()) * ws / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "pipeline": (f"{rows // CH} chunks of {CH} rows: copy in, MXFP4 quantize + dequantize and copy out "
                            "overlap on three streams; NVFP4 after the last chunk") if chunked else "serial"}

    # ---- NMSE of the step's outputs (host, untimed) ------------------------------
    idx = slice(0, 8)
    xs = inputs.bf16_bits_to_f32(x_np[idx]).astype(np.float64)

    def nmse(t):
        y = t[idx].float().cpu().numpy().astype(np.float64)
        return float(((xs - y) ** 2).sum() / (xs ** 2).sum())

    nmse_vals = {"mxfp4": nmse(dm), "nvfp4": nmse(dn), "rows_sampled": 8}

    gemm = None
    if not args.no_gemm:
        gemm = {"prefill": bench_prefill(torch, fp4, inputs, dev, reps=10),
                "decode": bench_decode(torch, fp4, inputs, dev, reps=10)}
    rotate = None if args.no_gemm else bench_rotate(torch, fp4, inputs, dev, reps=10)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        gbs, dt, cores = oracle_step(x_np)
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"one full step ({rows} x {cols}) on the host, {dt:.1f} s"}

    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD if rows == ROWS else WORKLOAD.replace(str(ROWS), str(rows)), "rows": rows, "cols": cols, "parallelism": f"replicas{ws}",
                   "l2": "inputs larger than L2 (268 MB bf16 tensor), no flush",
                   "step_bytes": sum(sb.values())},
        "frac_of_hbm_peak": value / ws / peak,
        "frac_of_hbm_spec": value / ws / SPEC_HBM_GBS,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "gemm": gemm,
        "rotate_quantize": rotate,
        "nmse": nmse_vals,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--rows", type=int, default=ROWS, help="rows of the tensor (profiling runs use fewer)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-gemm", action="store_true")
    ap.add_argument("--only", choices=["prefill", "decode", "rotate", "l2-encode"], default=None,
                    help="profiling helper: run one leg alone")
    ap.add_argument("--prefill-m", type=int, default=8192)
    ap.add_argument("--fmts", nargs="*", default=None)
    ap.add_argument("--decode-m", type=int, nargs="*", default=None, help="--only decode: activation rows")
    ap.add_argument("--decode-nk", nargs="*", default=None, help="--only decode: weight shapes NxK, e.g. 14336x4096")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
