"""Benchmark of the quantised-weight GEMM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hq|reference] [--workload NAME]

Metric: quantised GEMM TFLOPS (and weight GB/s, % of roofline) versus M.
Default workload ``w4a16_asym_sweep``: dense W4A16 with UINT4 weights, UINT4
zero points and bf16 scales per 128-K group, (N, K) in {(8192, 8192),
(28672, 8192), (8192, 28672)}, M swept over 1, 4, 16, 64, 256, 1024, 4096,
8192; A bf16 N(0, 1).  One step runs every (shape, M) GEMM once; the L2 is
flushed (a 512 MiB memset, untimed) before each GEMM and each GEMM is timed
with CUDA events on its stream.  ``value`` = total flops of a step / summed
GEMM time.  Other workloads (``--workload``): ``w4a16_dense_m16``,
``moe_w4a16_mxfp4``, ``moe_w4a8_mxfp8``, ``w4a4_nvfp4``, ``w8a8_fp8``.

Multi-GPU (torchrun): replicas only, every rank runs the same workload on
its own GPU; the timed region is bracketed by a barrier and a synchronise,
the time is the max over ranks and ``value`` counts every rank's flops.
``--impl reference`` times the CPU oracle (the only reference there is) on
a bounded sample of the same workload, on rank 0 only.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ---------------------------------------------------------------------------
# clocks sampler (nvidia-smi during the timed region)
# ---------------------------------------------------------------------------
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
class Op:
    """One library call of a step, with its algorithmic cost."""

    def __init__(self, name, run, flops, w_bytes, io_bytes, kernels, h2d=None, d2h=None, e2e=None):
        self.name = name
        self.run = run            # device-resident call
        self.flops = flops
        self.w_bytes = w_bytes    # packed weight + scale + zero bytes the call must read
        self.io_bytes = io_bytes  # activation + output bytes
        self.kernels = kernels    # library kernel launches per call
        self.h2d = h2d or 0
        self.d2h = d2h or 0
        self.e2e = e2e            # same call from pinned host buffers

    @property
    def bytes(self):
        return self.w_bytes + self.io_bytes


def _hq():
    import quantized_gemm_02_b200 as hq
    hq.lib()
    return hq


def desc_of(hq, w_dtype, group, scale_dtype, zero, glob, a_dtype):
    d = hq.QuantDesc()
    d.w_dtype, d.w_group, d.w_scale_dtype, d.w_has_zero, d.w_has_global, d.a_dtype = (
        w_dtype, group, scale_dtype, zero, glob, a_dtype)
    return d


def dense_op(hq, d, name, M, N, K, packed, w_bytes, gen, a_fmt="bf16", a_bits=None):
    """A dense hq_gemm over resident inputs (bf16 activations)."""
    dev = "cuda"
    A = synth.bf16_normal((M, K), gen, device=dev)
    C = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    wsb = hq.hq_gemm_workspace_bytes(d, M, N, K)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device=dev)
    A_h = A.cpu().pin_memory()
    C_h = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    A_e = torch.empty_like(A)

    def run():
        hq.hq_gemm(d, M, N, K, packed, A, None, None, C, ws, wsb)

    def e2e():
        A_e.copy_(A_h, non_blocking=True)
        hq.hq_gemm(d, M, N, K, packed, A_e, None, None, C, ws, wsb)
        C_h.copy_(C, non_blocking=True)

    return Op(name, run, 2.0 * M * N * K, w_bytes, M * K * 2 + M * N * 2, 1, M * K * 2, M * N * 2, e2e)


def packed_bytes_int4(N, K, group, zero):
    G = K // group
    return N * K // 2 + N * G * 2 + (N * G // 2 if zero else 0)


def workload_w4a16_asym_sweep(hq, gen_seed=0):
    shapes = [(8192, 8192), (28672, 8192), (8192, 28672)]
    Ms = [1, 4, 16, 64, 256, 1024, 4096, 8192]
    d = desc_of(hq, hq.HQ_UINT4, 128, hq.HQ_BF16, 1, 0, hq.HQ_BF16)
    gen = synth.generator(gen_seed, "cuda")
    ops = []
    keep = []
    for (N, K) in shapes:
        w = synth.int4_weights(1, N, K, 128, True, gen, device="cuda")
        packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device="cuda")
        hq.hq_pack_weights(d, 1, N, K, w["codes"], w["scales"], w["zeros"], None, packed)
        keep.append(packed)
        wb = packed_bytes_int4(N, K, 128, True)
        for M in Ms:
            ops.append(dense_op(hq, d, f"N{N}_K{K}_M{M}", M, N, K, packed, wb, gen))
    cfg = {"workload": "dense W4A16 UINT4 asym g128 bf16-scale, (N,K) in {(8192,8192),(28672,8192),(8192,28672)}, "
                       "M in {1,4,16,64,256,1024,4096,8192}",
           "shapes": shapes, "M": Ms, "l2": "flushed before every GEMM (512 MiB memset, untimed)"}
    return ops, cfg, keep


def workload_w4a16_dense_m16(hq, gen_seed=0):
    N = K = 4096
    M = 16
    d = desc_of(hq, hq.HQ_INT4, 128, hq.HQ_BF16, 0, 0, hq.HQ_BF16)
    gen = synth.generator(gen_seed, "cuda")
    w = synth.int4_weights(1, N, K, 128, False, gen, device="cuda")
    packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device="cuda")
    hq.hq_pack_weights(d, 1, N, K, w["codes"], w["scales"], None, None, packed)
    ops = [dense_op(hq, d, "N4096_K4096_M16", M, N, K, packed, packed_bytes_int4(N, K, 128, False), gen)]
    cfg = {"workload": "dense W4A16 INT4 sym g128, M=16, N=K=4096", "l2": "flushed before every GEMM"}
    return ops, cfg, [packed]


WORKLOADS = {
    "w4a16_asym_sweep": workload_w4a16_asym_sweep,
    "w4a16_dense_m16": workload_w4a16_dense_m16,
}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------
def cpu_baseline(workload: str, budget_s: float = 15.0):
    """Times the oracle as it stands on a bounded sample of the workload:
    decode one (N, K) weight matrix and multiply M rows in fp64."""
    import oracle as O
    gen = synth.generator(0)
    if workload == "w4a16_dense_m16":
        N, K, M, group, asym, wd = 4096, 4096, 16, 128, False, "int4"
    else:
        N, K, M, group, asym, wd = 8192, 8192, 16, 128, True, "uint4"
    w = synth.int4_weights(1, N, K, group, asym, gen)
    x = synth.bf16_normal((M, K), gen)
    desc = O.Desc(wd, group, "bf16", w_zero=asym)
    codes = synth.to_np_bits(w["codes"][0])
    scales = synth.to_np_bits(w["scales"][0])
    zeros = None if w["zeros"] is None else synth.to_np_bits(w["zeros"][0])
    xb = synth.to_np_bits(x)
    flops = 0.0
    t0 = time.perf_counter()
    n = 0
    while True:
        A, _ = O.decode_act("bf16", M, K, xb)
        W, col = O.decode_weights(desc, N, K, codes, scales, zeros)
        O.gemm(A, W, None, col)
        flops += 2.0 * M * N * K
        n += 1
        if time.perf_counter() - t0 > budget_s or n >= 50:
            break
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "sample": f"{n} x (decode {wd} g{group} W[{N},{K}] + fp64 GEMM M={M}), {dt:.1f} s; numpy BLAS threads",
            "seconds": dt}


# ---------------------------------------------------------------------------
def init_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args, ws, rank):
    if rank != 0:
        return 0
    steps = []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(args.workload, budget_s=max(2.0, 20.0 / (args.warmup + args.steps)))
        if i >= args.warmup:
            steps.append(cb)
    v = statistics.median([s["value"] for s in steps])
    line = {"impl": "reference", "metric": "quantized GEMM TFLOPS (CPU fp64 oracle)", "value": v, "unit": "TFLOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.median([s["seconds"] for s in steps]) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample": cb["sample"]},
            "cpu_baseline": {"value": v, "unit": "TFLOPS", "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"]},
            "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hq", choices=["hq", "reference"])
    ap.add_argument("--workload", default="w4a16_asym_sweep", choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    ws, rank, local = init_dist()
    if args.impl == "reference":
        return run_reference(args, ws, rank)

    hq = _hq()
    peaks = load_peaks()
    ops, cfg, keep = WORKLOADS[args.workload](hq)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    n_ops = len(ops)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops]

    def one_step(timed: bool, e2e: bool = False):
        times = []
        for i, op in enumerate(ops):
            flush.zero_()
            a, b = ev[i]
            a.record(stream)
            (op.e2e if e2e else op.run)()
            b.record(stream)
        torch.cuda.synchronize()
        for a, b in ev:
            times.append(a.elapsed_time(b))
        return times

    for _ in range(args.warmup):
        one_step(False)
    torch.cuda.synchronize()
    barrier(ws)
    clocks = Clocks(local)
    clocks.start()
    per_step = []
    per_op = np.zeros(n_ops)
    for _ in range(args.steps):
        t = one_step(True)
        per_step.append(sum(t))
        per_op += np.array(t)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    per_op /= args.steps
    ms_step = max_over_ranks(statistics.mean(per_step), ws)
    flops_step = sum(op.flops for op in ops)
    value = flops_step * ws / (ms_step / 1e3) / 1e12

    # end to end: host inputs copied in and outputs copied back inside the timed region
    for _ in range(1):
        one_step(False, e2e=True)
    e2e_steps = [sum(one_step(True, e2e=True)) for _ in range(args.steps)]
    e2e_ms = max_over_ranks(statistics.mean(e2e_steps), ws)

    # roofline of the dominant call (most time per step)
    i_dom = int(np.argmax(per_op))
    dom = ops[i_dom]
    t_dom = per_op[i_dom] / 1e3
    hbm_t = dom.bytes / (peaks["hbm_gbs"] * 1e9)
    flop_t = dom.flops / (peaks["bf16_tflops"] * 1e12)
    if flop_t >= hbm_t:
        roof = {"bound": "tensor", "achieved": dom.flops / t_dom / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": dom.bytes / t_dom / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = None
    roof["kernel"] = "hq stream_gemm (" + dom.name + ")"
    roof["peak_source"] = peaks["source"] + (" burst" if roof["bound"] == "tensor" else "")

    sweep = []
    for op, t in zip(ops, per_op):
        s = t / 1e3
        hb = op.bytes / s / 1e9
        sweep.append({"op": op.name, "us": round(t * 1e3, 2), "tflops": round(op.flops / s / 1e12, 2),
                      "weight_gbs": round(op.w_bytes / s / 1e9, 1), "hbm_frac": round(hb / peaks["hbm_gbs"], 3),
                      "tensor_frac": round(op.flops / s / 1e12 / peaks["bf16_tflops"], 3)})
    line = {
        "metric": "quantized GEMM TFLOPS and weight GB/s vs M (dense+MoE), % of roofline, 1xB200",
        "value": value, "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": cfg,
        "e2e": {"value": flops_step * ws / (e2e_ms / 1e3) / 1e12, "unit": "TFLOPS",
                "h2d_bytes_per_step": sum(op.h2d for op in ops), "d2h_bytes_per_step": sum(op.d2h for op in ops)},
        "gpu_launches": sum(op.kernels for op in ops) * args.steps,
        "roofline": roof, "clocks": clk, "sweep": sweep,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
