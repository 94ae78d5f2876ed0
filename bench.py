"""Benchmark of the quantised-weight GEMM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hq|reference] [--workload NAME]
                    [--shape M,N,K [--shape-fmt uint4|nvfp4|fp8]] [--eager] [--no-cpu-baseline]

Metric: quantised GEMM TFLOPS (and weight GB/s, % of roofline) versus M,
dense and MoE.  The default workload ``all`` runs every configuration once
per step:

  1. dense W4A16 INT4 symmetric g128, M = 16, N = K = 4096;
  2. dense W4A16 UINT4 + zero points g128, (N, K) in {(8192, 8192),
     (28672, 8192), (8192, 28672)}, M in {1, 4, 16, 64, 256, 1024, 4096, 8192};
  3. MoE W4A16 MXFP4, E = 256, top-8 softmax routing, H = 7168, I = 2048,
     T in {1, 16, 128, 1024, 4096}, grouped and indexed modes;
  4. MoE W4A8 (MXFP4 weights x MXFP8 activations quantised on the fly),
     Zipf(1.2) routing, T in {1, 64, 512, 4096}, both modes, fused weighted sum;
  5. dense W4A4 NVFP4 x NVFP4 and W8A8 FP8 at N = K = 7168, M in {1, 32, 256,
     2048, 8192} (activation quantisation inside the call), and the NVFP4 MoE
     at T = 4096 in both modes.

An MoE layer is timed as its library calls: the routing prepare, the
gate-up GEMM and the down GEMM with the weighted top-k sum.  The L2 is
flushed before every call (untimed: a 512 MiB memset, then one read of that
buffer, so that the timed call finds no line of its inputs in L2 and no dirty
line whose write-back it would pay for) and each call is timed
with CUDA events on its stream; each call is captured once in a CUDA graph
and replayed (``--eager`` times the plain calls).  ``value`` = total flops of
a step / summed call time; ``sweep`` lists every call with its roofline
fractions and ``per_config`` sums them per configuration.  The roofline
object describes the call of the five configurations that takes the most
time (the default workload's extra rows only appear in ``sweep``): HBM-bound
calls against
the measured copy bandwidth, tensor-bound ones against the measured bf16
peak times the nominal ratio of the call's MMA kind (FP8 and MXFP8 x FP4
weights 2, FP4 x FP4 4); ``traffic`` is the committed ncu DRAM figure when
the kernel sources still match it.  ``--workload`` picks one configuration
(``w4a16_dense_m16``, ``w4a16_asym_sweep``, ``moe_w4a16_mxfp4``,
``moe_w4a8_mxfp8``, ``w4a4_nvfp4``, ``w8a8_fp8``, ``moe_nvfp4``) or the
masked-layout MoE (``moe_masked_nvfp4``).

Multi-GPU (torchrun): replicas only, every rank runs the same workload on
its own GPU; the timed region is bracketed by a barrier and a synchronise,
the time is the max over ranks and ``value`` counts every rank's flops.
``--impl reference`` times the CPU oracle (the only reference there is) on
bounded samples of the same workload, on rank 0 only.
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

METRIC = "quantized GEMM TFLOPS and weight GB/s vs M (dense+MoE), % of roofline, 1xB200"

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
    """Samples the SM clock and the clock-event reasons of this rank's GPU
    during the timed region: NVML every 10 ms (read-only queries), else
    nvidia-smi every 50 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.nvml = None
        self.lines = []
        self.samples = []  # (sm_mhz, max_mhz, reason bits)
        self.stop_flag = threading.Event()

    def _nvml_handle(self, pynvml):
        try:
            props = torch.cuda.get_device_properties(self.index)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._nvml_handle(pynvml)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml

            def loop():
                while not self.stop_flag.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        rb = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), float(mx), int(rb)))
                    except Exception:
                        pass
                    time.sleep(0.01)

            self.th = threading.Thread(target=loop, daemon=True)
            self.th.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.stop_flag.set()
            self.th.join(timeout=2)
            if not self.samples:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
            reasons = set()
            for _, _, rb in self.samples:
                for n, bit in self.REASON_BITS.items():
                    if rb & bit:
                        reasons.add(n)
            return {"sm_mhz": statistics.median(x[0] for x in self.samples),
                    "sm_max_mhz": max(x[1] for x in self.samples), "reasons": sorted(reasons),
                    "samples": len(self.samples), "source": "nvml, 10 ms"}
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
                "samples": len(sm), "source": "nvidia-smi, 50 ms"}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
class Op:
    """One library call of a step, with its algorithmic cost."""

    def __init__(self, name, run, flops, w_bytes, io_bytes, kernels, h2d=None, d2h=None, e2e=None, kernel=None,
                 peak_ratio=1.0, config=0):
        self.name = name
        self.config = config      # which benchmark configuration (1..5) the call belongs to
        self.kernel = kernel      # the library kernel that dominates the call
        # dense tensor peak of the call's MMA kind relative to bf16 (nominal ratios: FP8 and
        # MXFP8-with-FP4-weights 2, FP4 x FP4 4), applied to the measured bf16 peak
        self.peak_ratio = peak_ratio
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


def dense_op(hq, d, name, M, N, K, packed, w_bytes, gen, config):
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

    return Op(name, run, 2.0 * M * N * K, w_bytes, M * K * 2 + M * N * 2, 1, M * K * 2, M * N * 2, e2e,
              kernel=gemm_kernel_name(M), config=config)


L2_NOTE = ("flushed before every call (512 MiB memset, then one read of that buffer so that no dirty line is "
           "left in L2; untimed)")

NOMINAL_HBM_GBS = 8000.0  # the nominal B200 figure the targets are quoted against


def sweep_entry(op, t_ms, peaks):
    """One sweep point: time, TFLOPS, weight GB/s and the fractions of the
    rooflines: HBM (measured copy bandwidth, and the nominal 8 TB/s), tensor
    (measured bf16 peak x the MMA kind's nominal ratio), and the combined
    roofline fraction max(bytes / BW, flops / peak) / t with the measured
    figures."""
    s = t_ms / 1e3
    hb = op.bytes / s / 1e9
    t_bw = op.bytes / (peaks["hbm_gbs"] * 1e9)
    t_fl = op.flops / (peaks["bf16_tflops"] * op.peak_ratio * 1e12)
    return {"op": op.name, "config": op.config, "us": round(t_ms * 1e3, 2),
            "tflops": round(op.flops / s / 1e12, 2),
            "weight_gbs": round(op.w_bytes / s / 1e9, 1), "hbm_frac": round(hb / peaks["hbm_gbs"], 3),
            "hbm_frac_nominal": round(hb / NOMINAL_HBM_GBS, 3),
            "tensor_frac": round(op.flops / s / 1e12 / (peaks["bf16_tflops"] * op.peak_ratio), 3),
            "roofline_frac": round(max(t_bw, t_fl) / s, 3)}


def gemm_kernel_name(rows_per_tile):
    """The GEMM kernel the library picks for a token tile of this many rows."""
    return "dec_gemm_kernel" if rows_per_tile <= 32 else "tc_gemm_kernel"


KERNEL_SOURCES = ("quantized_gemm_02_b200/csrc/hq_gemm_tc.cu", "quantized_gemm_02_b200/csrc/hq_gemm_small.cu",
                  "quantized_gemm_02_b200/csrc/hq_internal.cuh")


def kernel_source_digest():
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(op_name):
    """DRAM bytes per launch (read + write) of the op's GEMM kernel from the
    committed ncu capture in profiles/traffic.md, or None when there is none
    or the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(p):
        return None
    digest = kernel_source_digest()
    for line in open(p):
        f = [x.strip() for x in line.strip().strip("|").split("|")]
        if len(f) >= 6 and f[0] == op_name and f[5] == digest:
            try:
                return float(f[4])
            except ValueError:
                return None
    return None


def packed_bytes_int4(N, K, group, zero):
    G = K // group
    return N * K // 2 + N * G * 2 + (N * G // 2 if zero else 0)


CONFIG_TITLES = {
    1: "dense W4A16 INT4 sym g128, M=16, N=K=4096",
    2: "dense W4A16 UINT4 asym g128, (N,K) in {(8192,8192),(28672,8192),(8192,28672)}, M in {1,4,16,64,256,1024,"
       "4096,8192}",
    3: "MoE W4A16 MXFP4, E=256 top-8 softmax routing, H=7168, I=2048, T in {1,16,128,1024,4096}, grouped + indexed",
    4: "MoE W4A8 MXFP4 x MXFP8 (quantised on the fly), Zipf(1.2) routing, E=256 top-8, H=7168, I=2048, "
       "T in {1,64,512,4096}, grouped + indexed, fused weighted sum",
    5: "dense W4A4 NVFP4 x NVFP4 and W8A8 FP8 (per-channel x per-token), N=K=7168, M in {1,32,256,2048,8192}, "
       "activation quantisation inside the step; NVFP4 MoE at T=4096, grouped + indexed",
    "silu": "MoE gate-up GEMM + SiLU-and-mul at the config-3 shapes (MXFP4, bf16 activations, grouped), "
            "T in {16, 4096}: two calls versus the fused epilogue",
    "lowbit": "dense WnA16 at the other widths (INT2, INT3 g128; MXFP6 E2M3; float4e0m3 g128), N=28672, "
              "K=8192, M in {1, 16}",
    "fp8b": "block-scaled FP8 W8A8 (128 x 128 weight blocks, per token and 128 k activation scales): dense "
            "N=K=7168, M in {1,32,256,2048,8192}; MoE at the config-3 shapes, T in {64, 4096}, grouped + indexed",
    "mxint4": "MoE W4A16 MXINT4 (INT4 elements, E8M0 per 32) at the config-3 shapes and routing, T in {16, 4096}, "
              "grouped + indexed",
}

# Workload titles shared by the library arm's config and the reference arm's config.
WORKLOAD_TITLE = {
    "all": "all five configurations and the next-row formats: " +
           "; ".join(f"({i}) {t}" for i, t in CONFIG_TITLES.items()),
    "w4a16_asym_sweep": CONFIG_TITLES[2],
    "w4a16_dense_m16": CONFIG_TITLES[1],
    "moe_w4a16_mxfp4": CONFIG_TITLES[3],
    "moe_w4a8_mxfp8": CONFIG_TITLES[4],
    "moe_nvfp4": "MoE W4A4 NVFP4 x NVFP4 (activations quantised on the fly), E=256 top-8, H=7168, I=2048, T=4096, "
                 "grouped + indexed",
    "w4a4_nvfp4": "dense W4A4 NVFP4 x NVFP4, N=K=7168, M in {1,32,256,2048,8192}",
    "w8a8_fp8": "dense W8A8 FP8 per-channel x per-token, N=K=7168, M in {1,32,256,2048,8192}",
    "moe_silu": "MoE gate-up GEMM + SiLU-and-mul at the config-3 shapes, T in {16, 4096}: unfused and fused",
    "moe_indexed_gate_up_profile": "MoE W4A16 MXFP4 gate-up GEMM alone, indexed mode (config-3 MoE: E=256, top-8 "
                                   "softmax routing, T=4096, N=4096, K=7168), only the gate-up weights resident",
    "moe_nvfp4_down_profile": "MoE NVFP4 x NVFP4 down GEMM alone (config-5 MoE: E=256, top-8 softmax routing, "
                              "T=4096, N=7168, K=2048, grouped), only the down weights resident",
    "moe_profile_e64": "MoE W4A16 MXFP4 at the config-3 expert shapes with E=64, T=1024 (about 128 rows per "
                       "expert), grouped + indexed: a small case of the T=4096 calls for profiling",
    "lowbit": "dense WnA16 INT2, INT3, MXFP6 E2M3, float4e0m3 at N=28672, K=8192, M in {1, 16}",
    "w8a8_fp8_block": "block-scaled FP8 W8A8: dense N=K=7168, M in {1,32,256,2048,8192}, and MoE at the config-3 "
                      "shapes, T in {64, 4096}, grouped + indexed",
    "moe_w4a16_mxint4": "MoE W4A16 MXINT4 (INT4 elements, E8M0 per 32), config-3 shapes and routing, T in "
                        "{16, 4096}, grouped + indexed",
    "moe_masked_nvfp4": "masked-layout MoE W4A4 NVFP4 x NVFP4 (activations quantised on the fly), E=256 slabs of "
                        "256 rows, counts from a softmax top-8 routing of T=4096, H=7168, I=2048, gate-up + down",
}


def ops_w4a16_asym_sweep(hq, gen):
    shapes = [(8192, 8192), (28672, 8192), (8192, 28672)]
    Ms = [1, 4, 16, 64, 256, 1024, 4096, 8192]
    d = desc_of(hq, hq.HQ_UINT4, 128, hq.HQ_BF16, 1, 0, hq.HQ_BF16)
    ops, keep = [], []
    for (N, K) in shapes:
        w = synth.int4_weights(1, N, K, 128, True, gen, device="cuda")
        packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device="cuda")
        hq.hq_pack_weights(d, 1, N, K, w["codes"], w["scales"], w["zeros"], None, packed)
        keep.append(packed)
        wb = packed_bytes_int4(N, K, 128, True)
        for M in Ms:
            ops.append(dense_op(hq, d, f"N{N}_K{K}_M{M}", M, N, K, packed, wb, gen, 2))
    return ops, keep


def ops_w4a16_dense_m16(hq, gen):
    N = K = 4096
    M = 16
    d = desc_of(hq, hq.HQ_INT4, 128, hq.HQ_BF16, 0, 0, hq.HQ_BF16)
    w = synth.int4_weights(1, N, K, 128, False, gen, device="cuda")
    packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device="cuda")
    hq.hq_pack_weights(d, 1, N, K, w["codes"], w["scales"], None, None, packed)
    return [dense_op(hq, d, "cfg1_N4096_K4096_M16", M, N, K, packed, packed_bytes_int4(N, K, 128, False), gen,
                     1)], [packed]


def ops_shape(hq, M, N, K, gen):
    """One dense W4A16 UINT4-asymmetric GEMM of the given shape (profiling)."""
    d = desc_of(hq, hq.HQ_UINT4, 128, hq.HQ_BF16, 1, 0, hq.HQ_BF16)
    w = synth.int4_weights(1, N, K, 128, True, gen, device="cuda")
    packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device="cuda")
    hq.hq_pack_weights(d, 1, N, K, w["codes"], w["scales"], w["zeros"], None, packed)
    return [dense_op(hq, d, f"N{N}_K{K}_M{M}", M, N, K, packed, packed_bytes_int4(N, K, 128, True), gen, 2)], [packed]


def ops_lowbit(hq, gen, N=28672, K=8192, Ms=(1, 16)):
    """The other WnA16 widths on the largest config-2 shape with bf16
    activations: INT2 and INT3 (symmetric, bf16 scales per 128), MXFP6
    (E2M3, E8M0 per 32) and float4e0m3 (the zero-exponent view of symmetric
    INT4, bf16 scales per 128); weight GB/s at decode sizes."""
    kinds = [("int2_g128", hq.HQ_INT2, 128, hq.HQ_BF16, 2, False),
             ("int3_g128", hq.HQ_INT3, 128, hq.HQ_BF16, 3, False),
             ("mxfp6_e2m3", hq.HQ_E2M3, 32, hq.HQ_E8M0, 6, True),
             ("e0m3_g128", hq.HQ_E0M3, 128, hq.HQ_BF16, 4, False)]
    ops, keep = [], []
    for name, wd, grp, sd, bits, e8 in kinds:
        d = desc_of(hq, wd, grp, sd, 0, 0, hq.HQ_BF16)
        w = synth.lowbit_weights(1, N, K, bits, grp, False, e8, gen, device="cuda")
        packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device="cuda")
        hq.hq_pack_weights(d, 1, N, K, w["codes"], w["scales"], None, None, packed)
        keep.append(packed)
        wb = N * K * bits // 8 + N * (K // grp) * (1 if e8 else 2)
        for M in Ms:
            ops.append(dense_op(hq, d, f"{name}_N{N}_K{K}_M{M}", M, N, K, packed, wb, gen, "lowbit"))
    return ops, keep


def moe_call_kernels(hq, wdesc, a_dtype, mode, combine):
    """Library kernel launches of one hq_moe_gemm call: on-the-fly
    quantisation (MXFP8, per-token FP8: one kernel; NVFP4: tensor amax +
    quantise), the grouped mode's row copy, the block-scaled MMA's scale
    relayout or the dequantisation path's exact decode, the GEMM, and the
    weighted combine."""
    quant = a_dtype not in (None, hq.HQ_BF16)
    block_scaled = ((wdesc.w_dtype == hq.HQ_E2M1 and
                     ((wdesc.w_scale_dtype == hq.HQ_E8M0 and a_dtype == hq.HQ_MXFP8) or
                      (wdesc.w_scale_dtype == hq.HQ_UE4M3 and a_dtype == hq.HQ_NVFP4))) or
                    (wdesc.w_dtype == hq.HQ_E4M3 and wdesc.w_group == 128))
    n = 1  # the GEMM
    if quant:
        n += 2 if a_dtype == hq.HQ_NVFP4 else 1
        n += 1  # scale relayout (block-scaled) or exact decode to bf16
        if block_scaled and mode == hq.HQ_MOE_GROUPED:
            n += 1  # row copy of the codes
    elif mode == hq.HQ_MOE_GROUPED:
        n += 1  # row copy
    return n + (1 if combine else 0), block_scaled


def ops_moe(hq, config, name, wdesc, E, topk, H, I, Ts, routing, gen, a_dtype, modes=("grouped", "indexed"),
            parts=("gate_up", "down")):
    """MoE calls per T: the routing prepare, then per mode the gate-up GEMM
    (N = 2I, K = H, one activation row per token) and the down GEMM (N = H,
    K = I, one row per routed slot) with the fused weighted top-k sum; a MoE
    layer's time is the sum, as the pages time MoE (gate-up + down)."""
    dev = "cuda"
    weights = {}
    for part, (N, K) in (("gate_up", (2 * I, H)), ("down", (H, I))):
        if part not in parts:
            weights[part] = (None, N, K, 0)
            continue
        if wdesc.w_dtype == hq.HQ_E2M1 and wdesc.w_scale_dtype == hq.HQ_E8M0:
            w = synth.mxfp4_weights(E, N, K, gen, device=dev)
            glob = None
            bytes_per = N * K // 2 + N * K // 32
        elif wdesc.w_dtype == hq.HQ_INT4 and wdesc.w_scale_dtype == hq.HQ_E8M0:
            w = synth.mxint4_weights(E, N, K, gen, device=dev)
            glob = None
            bytes_per = N * K // 2 + N * K // 32
        elif wdesc.w_dtype == hq.HQ_E4M3 and wdesc.w_group == 128:
            w = synth.fp8_block_weights(E, N, K, gen, device=dev)
            glob = None
            bytes_per = N * K + ((N + 127) // 128) * (K // 128) * 4
        else:
            w = synth.nvfp4_weights_random(E, N, K, gen, device=dev)
            glob = w["global"]
            bytes_per = N * K // 2 + N * K // 16
        packed = torch.empty(hq.hq_packed_weights_bytes(wdesc, E, N, K), dtype=torch.uint8, device=dev)
        hq.hq_pack_weights(wdesc, E, N, K, w["codes"], w["scales"], None, glob, packed)
        del w
        weights[part] = (packed, N, K, bytes_per)
    pg, Ng, Kg, bg = weights["gate_up"]
    pd, Nd, Kd, bd = weights["down"]
    ratio = 1.0
    ops, keep = [], [weights]
    for T in Ts:
        ids, wts = routing(T, gen)
        touched = int(torch.unique(ids).numel())
        x_gate = synth.bf16_normal((T, H), gen, device=dev)
        x_down = synth.bf16_normal((T * topk, I), gen, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * topk, dtype=torch.int32, device=dev)
        inv = torch.empty(T * topk, dtype=torch.int32, device=dev)
        ids_h = ids.cpu().pin_memory()
        x_gate_h = x_gate.cpu().pin_memory()
        x_down_h = x_down.cpu().pin_memory()
        keep += [ids, wts, x_gate, x_down, off, perm, inv, ids_h, x_gate_h, x_down_h]

        def run_perm(T=T, ids=ids, off=off, perm=perm, inv=inv):
            hq.hq_moe_permute(T, topk, E, ids, off, perm, inv)

        def e2e_perm(run_perm=run_perm, ids=ids, ids_h=ids_h):
            ids.copy_(ids_h, non_blocking=True)
            run_perm()

        ops.append(Op(f"{name}_T{T}_routing", run_perm, 0.0, 0, T * topk * 4 * 3 + (E + 1) * 4, 1, T * topk * 4, 0,
                      e2e_perm, kernel="moe_permute_kernel", config=config))
        for mode_name in modes:
            mode = hq.HQ_MOE_GROUPED if mode_name == "grouped" else hq.HQ_MOE_INDEXED
            wsg = hq.hq_moe_workspace_bytes(mode, wdesc, T, topk, E, Ng, Kg, 0, 0)
            wsd = hq.hq_moe_workspace_bytes(mode, wdesc, T, topk, E, Nd, Kd, 1, 1)
            ws = torch.zeros(max(wsg, wsd), dtype=torch.uint8, device=dev)
            y = torch.empty(T * topk, Ng, dtype=torch.bfloat16, device=dev)
            out = torch.empty(T, Nd, dtype=torch.bfloat16, device=dev)
            out_h = torch.empty(T, Nd, dtype=torch.bfloat16).pin_memory()
            keep += [ws, y, out, out_h]

            def run_gate(mode=mode, ws=ws, y=y, x_gate=x_gate, wts=wts, off=off, perm=perm, T=T, wsg=wsg):
                hq.hq_moe_gemm(mode, wdesc, T, topk, E, Ng, Kg, pg, x_gate, None, None, 0, None, wts, off, perm, 0,
                               1.0, y, ws, wsg)

            def e2e_gate(run_gate=run_gate, x_gate=x_gate, x_gate_h=x_gate_h):
                x_gate.copy_(x_gate_h, non_blocking=True)
                run_gate()

            def run_down(mode=mode, ws=ws, out=out, x_down=x_down, wts=wts, off=off, perm=perm, T=T, wsd=wsd):
                hq.hq_moe_gemm(mode, wdesc, T, topk, E, Nd, Kd, pd, x_down, None, None, 1, None, wts, off, perm, 1,
                               1.0, out, ws, wsd)

            def e2e_down(run_down=run_down, x_down=x_down, x_down_h=x_down_h, out=out, out_h=out_h):
                x_down.copy_(x_down_h, non_blocking=True)
                run_down()
                out_h.copy_(out, non_blocking=True)

            kg, bs = moe_call_kernels(hq, wdesc, a_dtype, mode, 0)
            kd, _ = moe_call_kernels(hq, wdesc, a_dtype, mode, 1)
            if bs:
                ratio = 4.0 if wdesc.w_scale_dtype == hq.HQ_UE4M3 else 2.0
            kern = "bs_gemm_kernel" if bs else ("dec_gemm_kernel / tc_gemm_kernel")
            if "gate_up" in parts:
                ops.append(Op(f"{name}_T{T}_{mode_name}_gate_up", run_gate, 2.0 * T * topk * Ng * Kg, touched * bg,
                              T * Kg * 2 + T * topk * Ng * 2, kg, T * Kg * 2, 0, e2e_gate, kernel=kern,
                              peak_ratio=ratio, config=config))
            if "down" in parts:
                ops.append(Op(f"{name}_T{T}_{mode_name}_down", run_down, 2.0 * T * topk * Nd * Kd, touched * bd,
                              T * topk * Kd * 2 + T * Nd * 2, kd, T * topk * Kd * 2, T * Nd * 2, e2e_down,
                              kernel=kern, peak_ratio=ratio, config=config))
    return ops, keep


E_MOE, TOPK, H_MOE, I_MOE = 256, 8, 7168, 2048


def ops_moe_w4a16_mxfp4(hq, gen, Ts=(1, 16, 128, 1024, 4096)):
    d = desc_of(hq, hq.HQ_E2M1, 32, hq.HQ_E8M0, 0, 0, hq.HQ_BF16)
    routing = lambda T, g: synth.routing_softmax_topk(T, E_MOE, TOPK, g, device="cuda")
    return ops_moe(hq, 3, "cfg3_moe_w4a16", d, E_MOE, TOPK, H_MOE, I_MOE, list(Ts), routing, gen, hq.HQ_BF16)


def ops_moe_w4a16_mxint4(hq, gen, Ts=(16, 4096)):
    """MoE W4A16 with MXINT4 weights (INT4 elements, E8M0 per 32) at the
    config-3 shapes and routing."""
    d = desc_of(hq, hq.HQ_INT4, 32, hq.HQ_E8M0, 0, 0, hq.HQ_BF16)
    routing = lambda T, g: synth.routing_softmax_topk(T, E_MOE, TOPK, g, device="cuda")
    return ops_moe(hq, "mxint4", "moe_w4a16_mxint4", d, E_MOE, TOPK, H_MOE, I_MOE, list(Ts), routing, gen,
                   hq.HQ_BF16)


def ops_moe_silu(hq, gen, Ts=(16, 4096)):
    """The gate-up GEMM followed by SiLU-and-mul at the config-3 shapes
    (MXFP4 weights, bf16 activations, grouped mode): the two-call form
    (hq_moe_gemm writing the [T * 8, 2I] gate-up rows, then hq_silu_and_mul)
    and the fused form (hq_moe_gemm_gated on gate/up-interleaved weights)."""
    dev = "cuda"
    E, topk, H, I = E_MOE, TOPK, H_MOE, I_MOE
    d = desc_of(hq, hq.HQ_E2M1, 32, hq.HQ_E8M0, 0, 0, hq.HQ_BF16)
    w = synth.mxfp4_weights(E, 2 * I, H, gen, device=dev)
    nb = hq.hq_packed_weights_bytes(d, E, 2 * I, H)
    plain = torch.empty(nb, dtype=torch.uint8, device=dev)
    gated = torch.empty(nb, dtype=torch.uint8, device=dev)
    hq.hq_pack_weights(d, E, 2 * I, H, w["codes"], w["scales"], None, None, plain)
    hq.hq_pack_weights_gated(d, E, 2 * I, H, w["codes"], w["scales"], None, None, gated)
    del w
    bytes_per = 2 * I * H // 2 + 2 * I * H // 32
    ops, keep = [], [plain, gated]
    for T in Ts:
        ids, wts = synth.routing_softmax_topk(T, E, topk, gen, device=dev)
        touched = int(torch.unique(ids).numel())
        x = synth.bf16_normal((T, H), gen, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * topk, dtype=torch.int32, device=dev)
        inv = torch.empty(T * topk, dtype=torch.int32, device=dev)
        hq.hq_moe_permute(T, topk, E, ids, off, perm, inv)
        mode = hq.HQ_MOE_GROUPED
        wsb = max(hq.hq_moe_workspace_bytes(mode, d, T, topk, E, 2 * I, H, 0, 0),
                  hq.hq_moe_gated_workspace_bytes(mode, d, T, topk, E, I, H))
        ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
        y = torch.empty(T * topk, 2 * I, dtype=torch.bfloat16, device=dev)
        h = torch.empty(T * topk, I, dtype=torch.bfloat16, device=dev)
        x_h = x.cpu().pin_memory()
        h_h = torch.empty(T * topk, I, dtype=torch.bfloat16).pin_memory()
        keep += [ids, wts, x, off, perm, inv, ws, y, h, x_h, h_h]

        def run_two(T=T, x=x, off=off, perm=perm, ws=ws, y=y, h=h, wsb=wsb):
            hq.hq_moe_gemm(mode, d, T, topk, E, 2 * I, H, plain, x, None, None, 0, None, None, off, perm, 0, 1.0, y,
                           ws, wsb)
            hq.hq_silu_and_mul(T * topk, I, y, h)

        def run_fused(T=T, x=x, off=off, perm=perm, ws=ws, h=h, wsb=wsb):
            hq.hq_moe_gemm_gated(mode, d, T, topk, E, I, H, gated, x, None, None, None, off, perm, h, ws, wsb)

        for nm, run, nk in (("gate_up_then_silu", run_two, 3), ("gate_up_silu_fused", run_fused, 2)):
            def e2e(run=run, x=x, x_h=x_h, h=h, h_h=h_h):
                x.copy_(x_h, non_blocking=True)
                run()
                h_h.copy_(h, non_blocking=True)
            io = T * H * 2 + T * topk * I * 2 + (2 * T * topk * 2 * I * 2 if nm == "gate_up_then_silu" else 0)
            ops.append(Op(f"silu_mxfp4_T{T}_{nm}", run, 2.0 * T * topk * 2 * I * H, touched * bytes_per, io, nk,
                          T * H * 2, T * topk * I * 2, e2e, kernel="dec_gemm_kernel / tc_gemm_kernel",
                          config="silu"))
    return ops, keep


def ops_moe_fp8_block(hq, gen, Ts=(64, 4096)):
    """Block-scaled FP8 W8A8 MoE (128 x 128 weight blocks, per token and 128
    k activation scales quantised on the fly) at the config-3 shapes."""
    d = desc_of(hq, hq.HQ_E4M3, 128, hq.HQ_FP32, 0, 0, hq.HQ_E4M3)
    d.a_group = 128
    routing = lambda T, g: synth.routing_softmax_topk(T, E_MOE, TOPK, g, device="cuda")
    return ops_moe(hq, "fp8b", "moe_w8a8_fp8_block", d, E_MOE, TOPK, H_MOE, I_MOE, list(Ts), routing, gen,
                   hq.HQ_E4M3)


def ops_moe_profile_e64(hq, gen):
    """A profiling case of the config-3 MoE calls at a quarter of the experts:
    E = 64, T = 1024, top-8 (about 128 routed rows per expert, as at T = 4096
    with 256 experts), MXFP4 W4A16, grouped and indexed; 1.4 GB of weights."""
    d = desc_of(hq, hq.HQ_E2M1, 32, hq.HQ_E8M0, 0, 0, hq.HQ_BF16)
    routing = lambda T, g: synth.routing_softmax_topk(T, 64, TOPK, g, device="cuda")
    return ops_moe(hq, 3, "moe_w4a16_e64", d, 64, TOPK, H_MOE, I_MOE, [1024], routing, gen, hq.HQ_BF16)


def ops_moe_w4a8_mxfp8(hq, gen, Ts=(1, 64, 512, 4096)):
    d = desc_of(hq, hq.HQ_E2M1, 32, hq.HQ_E8M0, 0, 0, hq.HQ_MXFP8)
    routing = lambda T, g: synth.routing_zipf(T, E_MOE, TOPK, 1.2, g, device="cuda")
    return ops_moe(hq, 4, "cfg4_moe_w4a8", d, E_MOE, TOPK, H_MOE, I_MOE, list(Ts), routing, gen, hq.HQ_MXFP8)


def ops_moe_nvfp4(hq, gen, Ts=(4096,)):
    d = desc_of(hq, hq.HQ_E2M1, 16, hq.HQ_UE4M3, 0, 1, hq.HQ_NVFP4)
    routing = lambda T, g: synth.routing_softmax_topk(T, E_MOE, TOPK, g, device="cuda")
    return ops_moe(hq, 5, "cfg5_moe_nvfp4", d, E_MOE, TOPK, H_MOE, I_MOE, list(Ts), routing, gen, hq.HQ_NVFP4)


def ops_moe_nvfp4_down_profile(hq, gen):
    """A profiling case: the config-5 NVFP4 MoE down GEMM alone (E = 256,
    top-8 softmax routing of T = 4096 tokens, N = 7168, K = 2048, grouped,
    with the weighted top-k sum), only the down weights on the device
    (1.9 GB)."""
    d = desc_of(hq, hq.HQ_E2M1, 16, hq.HQ_UE4M3, 0, 1, hq.HQ_NVFP4)
    routing = lambda T, g: synth.routing_softmax_topk(T, E_MOE, TOPK, g, device="cuda")
    return ops_moe(hq, 5, "moe_nvfp4_down", d, E_MOE, TOPK, H_MOE, I_MOE, [4096], routing, gen, hq.HQ_NVFP4,
                   modes=("grouped",), parts=("down",))


def ops_moe_w4a16_indexed_gate_up_profile(hq, gen):
    """A profiling case: the config-3 MoE W4A16 MXFP4 gate-up GEMM alone in
    indexed mode at T = 4096 (E = 256, top-8 softmax routing, N = 4096,
    K = 7168), only the gate-up weights on the device (3.8 GB)."""
    d = desc_of(hq, hq.HQ_E2M1, 32, hq.HQ_E8M0, 0, 0, hq.HQ_BF16)
    routing = lambda T, g: synth.routing_softmax_topk(T, E_MOE, TOPK, g, device="cuda")
    return ops_moe(hq, 3, "cfg3_moe_w4a16", d, E_MOE, TOPK, H_MOE, I_MOE, [4096], routing, gen, hq.HQ_BF16,
                   modes=("indexed",), parts=("gate_up",))


def ops_moe_masked_nvfp4(hq, gen):
    """Masked-layout MoE (expert slabs with per-expert valid counts), NVFP4 x
    NVFP4, config-5 MoE shapes: the counts come from a softmax top-8 routing
    of T = 4096 tokens over E = 256 experts, slabs of 256 rows, expected_m =
    the mean count.  Step = gate-up (N = 2I, K = H) + down (N = H, K = I)."""
    dev = "cuda"
    E, topk, H, I, T, slab = E_MOE, TOPK, H_MOE, I_MOE, 4096, 256
    d = desc_of(hq, hq.HQ_E2M1, 16, hq.HQ_UE4M3, 0, 1, hq.HQ_NVFP4)
    ids, _ = synth.routing_softmax_topk(T, E, topk, gen, device=dev)
    counts = torch.bincount(ids.flatten().long(), minlength=E).clamp(max=slab).to(torch.int32)
    touched = int((counts > 0).sum())
    rows = int(counts.sum())
    expected_m = max(1, rows // E)
    parts = {}
    for part, (N, K) in (("gate_up", (2 * I, H)), ("down", (H, I))):
        w = synth.nvfp4_weights_random(E, N, K, gen, device=dev)
        packed = torch.empty(hq.hq_packed_weights_bytes(d, E, N, K), dtype=torch.uint8, device=dev)
        hq.hq_pack_weights(d, E, N, K, w["codes"], w["scales"], None, w["global"], packed)
        del w
        parts[part] = (packed, N, K, N * K // 2 + N * K // 16)
    pg, Ng, Kg, bg = parts["gate_up"]
    pd, Nd, Kd, bd = parts["down"]
    x_gate = synth.bf16_normal((E * slab, Kg), gen, device=dev)
    x_down = synth.bf16_normal((E * slab, Kd), gen, device=dev)
    y = torch.empty(E * slab, Ng, dtype=torch.bfloat16, device=dev)
    out = torch.empty(E * slab, Nd, dtype=torch.bfloat16, device=dev)
    wsb = max(hq.hq_moe_masked_workspace_bytes(d, E, slab, Ng, Kg, expected_m),
              hq.hq_moe_masked_workspace_bytes(d, E, slab, Nd, Kd, expected_m))
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    counts_h = counts.cpu().pin_memory()
    counts_e = torch.empty_like(counts)
    x_h = x_gate.cpu().pin_memory()
    out_h = torch.empty(E * slab, Nd, dtype=torch.bfloat16).pin_memory()

    def run():
        hq.hq_moe_gemm_masked(d, E, slab, Ng, Kg, pg, x_gate, counts, expected_m, y, ws, wsb)
        hq.hq_moe_gemm_masked(d, E, slab, Nd, Kd, pd, x_down, counts, expected_m, out, ws, wsb)

    def e2e():
        counts_e.copy_(counts_h, non_blocking=True)
        x_gate.copy_(x_h, non_blocking=True)
        run()
        out_h.copy_(out, non_blocking=True)

    flops = 2.0 * rows * (Ng * Kg + Nd * Kd)
    io = rows * (Kg // 2 + Ng * 2 + Kd // 2 + Nd * 2)
    # per GEMM: routing prepare, amax + quantise, gather codes, scale relayout, GEMM
    op = Op(f"moe_masked_nvfp4_T{T}_slab{slab}", run, flops, touched * (bg + bd), io, 2 * 6,
            E * slab * Kg * 2 + E * 4, E * slab * Nd * 2, e2e, kernel="bs_gemm_kernel", peak_ratio=4.0, config=5)
    return [op], [parts, x_gate, x_down, y, out, ws, counts]


def ops_dense_quantised(hq, fmt, gen, N=7168, K=7168, Ms=(1, 32, 256, 2048, 8192)):
    """Config 5 dense: N = K = 7168, both operands N(0,1) quantised by the
    library's own quantiser (weights per output row), M swept; each call
    quantises its activations and multiplies."""
    dev = "cuda"
    if fmt == "nvfp4":
        d = desc_of(hq, hq.HQ_E2M1, 16, hq.HQ_UE4M3, 0, 1, hq.HQ_NVFP4)
        wbytes = N * K // 2 + N * K // 16
    elif fmt == "fp8b":
        d = desc_of(hq, hq.HQ_E4M3, 128, hq.HQ_FP32, 0, 0, hq.HQ_E4M3)
        d.a_group = 128
        wbytes = N * K + ((N + 127) // 128) * (K // 128) * 4
    else:
        d = desc_of(hq, hq.HQ_E4M3, 0, hq.HQ_FP32, 0, 0, hq.HQ_E4M3)
        wbytes = N * K + N * 4
    Wf = synth.bf16_normal((N, K), gen, device=dev)

    def quant(x):
        M = x.shape[0]
        if fmt == "nvfp4":
            c = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
            s = torch.empty(M, K // 16, dtype=torch.uint8, device=dev)
        elif fmt == "fp8b":
            c = torch.empty(M, K, dtype=torch.uint8, device=dev)
            s = torch.empty(M, K // 128, dtype=torch.float32, device=dev)
        else:
            c = torch.empty(M, K, dtype=torch.uint8, device=dev)
            s = torch.empty(M, dtype=torch.float32, device=dev)
        g = torch.zeros(1, dtype=torch.float32, device=dev)
        wsq = torch.zeros(64, dtype=torch.uint8, device=dev)
        return c, s, g, wsq

    packed = torch.empty(hq.hq_packed_weights_bytes(d, 1, N, K), dtype=torch.uint8, device=dev)
    if fmt == "fp8b":
        # random E4M3 codes with 128 x 128 block scales (no weight quantiser for blocks)
        wb = synth.fp8_block_weights(1, N, K, gen, device=dev)
        hq.hq_pack_weights(d, 1, N, K, wb["codes"], wb["scales"], None, None, packed)
        wg = None
    else:
        wc, wsc, wg, wq = quant(Wf)
        hq.hq_quant_act(d, N, K, Wf, wc, wsc, wg, None, wq, 64)
        hq.hq_pack_weights(d, 1, N, K, wc, wsc, None, wg if fmt == "nvfp4" else None, packed)
    ops = []
    keep = [packed, wg]
    for M in Ms:
        x = synth.bf16_normal((M, K), gen, device=dev)
        c, s, g, wq2 = quant(x)
        C = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        wsb = hq.hq_gemm_workspace_bytes(d, M, N, K)
        ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device=dev)
        x_h = x.cpu().pin_memory()
        C_h = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
        keep += [x, c, s, g, wq2, C, ws, x_h, C_h]

        def run(M=M, x=x, c=c, s=s, g=g, wq2=wq2, C=C, ws=ws, wsb=wsb):
            hq.hq_quant_act(d, M, K, x, c, s, g, None, wq2, 64)
            hq.hq_gemm(d, M, N, K, packed, c, s, g if fmt == "nvfp4" else None, C, ws, wsb)

        def e2e(run=run, x=x, x_h=x_h, C=C, C_h=C_h):
            x.copy_(x_h, non_blocking=True)
            run()
            C_h.copy_(C, non_blocking=True)

        kern = (2 if fmt == "nvfp4" else 1) + (1 if fmt == "fp8" else 2)
        tag = 5 if fmt != "fp8b" else "fp8b"
        ops.append(Op(f"{'cfg5_' if tag == 5 else ''}{fmt}_N{N}_K{K}_M{M}", run, 2.0 * M * N * K, wbytes,
                      M * K * 2 + M * N * 2, kern, M * K * 2, M * N * 2, e2e,
                      kernel="bsf_gemm_kernel" if fmt == "fp8b" else "bs_gemm_kernel",
                      peak_ratio=4.0 if fmt == "nvfp4" else 2.0, config=tag))
    return ops, keep


def _workload(builders, title):
    def build(hq, gen_seed=0):
        gen = synth.generator(gen_seed, "cuda")
        ops, keep = [], []
        for b in builders:
            o, k = b(hq, gen)
            ops += o
            keep += k
        return ops, {"workload": title, "l2": L2_NOTE}, keep
    return build


WORKLOADS = {
    "all": _workload([ops_w4a16_dense_m16, ops_w4a16_asym_sweep, ops_moe_w4a16_mxfp4, ops_moe_w4a8_mxfp8,
                      lambda hq, g: ops_dense_quantised(hq, "nvfp4", g), lambda hq, g: ops_dense_quantised(hq, "fp8", g),
                      ops_moe_nvfp4, ops_moe_w4a16_mxint4, ops_moe_silu, ops_lowbit,
                      lambda hq, g: ops_dense_quantised(hq, "fp8b", g), ops_moe_fp8_block], WORKLOAD_TITLE["all"]),
    "w8a8_fp8_block": _workload([lambda hq, g: ops_dense_quantised(hq, "fp8b", g), ops_moe_fp8_block],
                                WORKLOAD_TITLE["w8a8_fp8_block"]),
    "lowbit": _workload([ops_lowbit], WORKLOAD_TITLE["lowbit"]),
    "moe_silu": _workload([ops_moe_silu], WORKLOAD_TITLE["moe_silu"]),
    "moe_profile_e64": _workload([ops_moe_profile_e64], WORKLOAD_TITLE["moe_profile_e64"]),
    "moe_nvfp4_down_profile": _workload([ops_moe_nvfp4_down_profile], WORKLOAD_TITLE["moe_nvfp4_down_profile"]),
    "moe_indexed_gate_up_profile": _workload([ops_moe_w4a16_indexed_gate_up_profile],
                                             WORKLOAD_TITLE["moe_indexed_gate_up_profile"]),
    "moe_w4a16_mxint4": _workload([ops_moe_w4a16_mxint4], WORKLOAD_TITLE["moe_w4a16_mxint4"]),
    "w4a16_asym_sweep": _workload([ops_w4a16_asym_sweep], WORKLOAD_TITLE["w4a16_asym_sweep"]),
    "w4a16_dense_m16": _workload([ops_w4a16_dense_m16], WORKLOAD_TITLE["w4a16_dense_m16"]),
    "moe_w4a16_mxfp4": _workload([ops_moe_w4a16_mxfp4], WORKLOAD_TITLE["moe_w4a16_mxfp4"]),
    "moe_w4a8_mxfp8": _workload([ops_moe_w4a8_mxfp8], WORKLOAD_TITLE["moe_w4a8_mxfp8"]),
    "moe_nvfp4": _workload([ops_moe_nvfp4], WORKLOAD_TITLE["moe_nvfp4"]),
    "moe_masked_nvfp4": _workload([ops_moe_masked_nvfp4], WORKLOAD_TITLE["moe_masked_nvfp4"]),
    "w4a4_nvfp4": _workload([lambda hq, g: ops_dense_quantised(hq, "nvfp4", g)], WORKLOAD_TITLE["w4a4_nvfp4"]),
    "w8a8_fp8": _workload([lambda hq, g: ops_dense_quantised(hq, "fp8", g)], WORKLOAD_TITLE["w8a8_fp8"]),
}

# configurations each workload covers (for the CPU samples)
WORKLOAD_CONFIGS = {"all": (1, 2, 3, 4, 5), "moe_profile_e64": (3,), "moe_nvfp4_down_profile": (5,), "moe_indexed_gate_up_profile": (3,), "w8a8_fp8_block": (5,), "moe_w4a16_mxint4": (3,), "moe_silu": (3,), "lowbit": (2,), "w4a16_asym_sweep": (2,), "w4a16_dense_m16": (1,),
                    "moe_w4a16_mxfp4": (3,), "moe_w4a8_mxfp8": (4,), "moe_nvfp4": (5,), "moe_masked_nvfp4": (5,),
                    "w4a4_nvfp4": (5,), "w8a8_fp8": (5,)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded samples)
# ---------------------------------------------------------------------------
# One sample per configuration: (weight kind, activation format, N, K, M):
# decode one weight matrix of the configuration's format and shape, quantise
# and decode M activation rows where the configuration quantises them, and
# multiply in fp64 (the MoE samples are one expert's gate-up matrix).
CPU_SAMPLES = {
    1: [("int4", "bf16", 4096, 4096, 16)],
    2: [("uint4", "bf16", 8192, 8192, 16)],
    3: [("mxfp4", "bf16", 4096, 7168, 16)],
    4: [("mxfp4", "mxfp8", 4096, 7168, 64)],
    5: [("nvfp4", "nvfp4", 7168, 7168, 32), ("fp8", "fp8", 7168, 7168, 32)],
}


def _cpu_sample(O, wk, ak, N, K, M, budget_s, gen):
    """Times the oracle on one sample until ``budget_s``; returns (flops, s, n)."""
    if wk in ("int4", "uint4"):
        w = synth.int4_weights(1, N, K, 128, wk == "uint4", gen)
        desc = O.Desc(wk, 128, "bf16", w_zero=(wk == "uint4"))
        args = (synth.to_np_bits(w["codes"][0]), synth.to_np_bits(w["scales"][0]),
                None if w["zeros"] is None else synth.to_np_bits(w["zeros"][0]))
    elif wk == "mxfp4":
        w = synth.mxfp4_weights(1, N, K, gen)
        desc = O.Desc("e2m1", 32, "e8m0")
        args = (synth.to_np_bits(w["codes"][0]), synth.to_np_bits(w["scales"][0]), None)
    elif wk == "nvfp4":
        w = synth.nvfp4_weights_random(1, N, K, gen)
        desc = O.Desc("e2m1", 16, "ue4m3", w_global=True)
        args = (synth.to_np_bits(w["codes"][0]), synth.to_np_bits(w["scales"][0]), None,
                synth.to_np_bits(w["global"])[0])
    else:
        w = synth.fp8_weights_random(1, N, K, gen)
        desc = O.Desc("e4m3", 0, "fp32")
        args = (synth.to_np_bits(w["codes"][0]), synth.to_np_bits(w["scales"][0]), None)
    xb = synth.to_np_bits(synth.bf16_normal((M, K), gen))
    flops, n = 0.0, 0
    t0 = time.perf_counter()
    while True:
        if ak == "bf16":
            A, row = O.decode_act("bf16", M, K, xb)
        elif ak == "fp8":
            q, sc = O.quant_fp8_per_token(xb)
            A, row = O.decode_act("fp8", M, K, q, sc)
        elif ak == "mxfp8":
            q, sc = O.quant_mxfp8(xb)
            A, row = O.decode_act("mxfp8", M, K, q, sc)
        else:
            q, sc, g = O.quant_nvfp4(xb)
            A, row = O.decode_act("nvfp4", M, K, q, sc, g)
        W, col = O.decode_weights(desc, N, K, *args)
        O.gemm(A, W, row, col)
        flops += 2.0 * M * N * K
        n += 1
        if time.perf_counter() - t0 > budget_s or n >= 50:
            break
    return flops, time.perf_counter() - t0, n


def cpu_baseline(workload: str, budget_s: float = 15.0):
    """Times the oracle as it stands on bounded samples of the workload, one
    per configuration it covers (all host threads numpy's BLAS uses), plus
    the first sample again on one thread.  ``value`` = sampled flops / time."""
    import oracle as O
    gen = synth.generator(0)
    cfgs = WORKLOAD_CONFIGS.get(workload, (2,))
    samples = [(c, s) for c in cfgs for s in CPU_SAMPLES[c]]
    per = max(1.0, budget_s / len(samples))
    tot_f = tot_s = 0.0
    per_cfg = {}
    descr = []
    for c, (wk, ak, N, K, M) in samples:
        f, s, n = _cpu_sample(O, wk, ak, N, K, M, per, gen)
        tot_f += f
        tot_s += s
        e = per_cfg.setdefault(str(c), {"flops": 0.0, "seconds": 0.0})
        e["flops"] += f
        e["seconds"] += s
        act = "" if ak == "bf16" else f" + {ak} quantise/decode of A"
        descr.append(f"cfg{c}: {n} x (decode {wk} W[{N},{K}]{act} + fp64 GEMM M={M})")
    for e in per_cfg.values():
        e["tflops"] = e["flops"] / e["seconds"] / 1e12
    one = None
    try:
        from threadpoolctl import threadpool_limits
        c, (wk, ak, N, K, M) = samples[0]
        with threadpool_limits(limits=1):
            f, s, n = _cpu_sample(O, wk, ak, N, K, M, min(per, 5.0), gen)
        one = {"tflops": f / s / 1e12, "cores": 1, "sample": f"cfg{c}: {n} x decode {wk} W[{N},{K}] + GEMM M={M}"}
    except Exception as exc:  # threadpoolctl unavailable: no 1-thread figure
        one = {"unavailable": type(exc).__name__}
    cores = len(os.sched_getaffinity(0))
    return {"value": tot_f / tot_s / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "sample": "; ".join(descr) + f"; {tot_s:.1f} s on numpy BLAS threads", "seconds": tot_s,
            "per_config": per_cfg, "one_core": one}


# ---------------------------------------------------------------------------
def init_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            # host-only runs (the reference arm's ranks, the CPU tests of this plumbing)
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
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
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.median([s["seconds"] for s in steps]) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_TITLE.get(args.workload, args.workload), "sample": cb["sample"],
                       "note": "CPU fp64 oracle on the host cores, bounded samples of the workload"},
            "cpu_baseline": {"value": v, "unit": "TFLOPS", "cores": cb["cores"], "kind": "oracle",
                             "sample": cb["sample"], "per_config": cb.get("per_config"),
                             "one_core": cb.get("one_core")},
            "e2e": {"value": v, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="hq", choices=["hq", "reference"])
    ap.add_argument("--workload", default="all", choices=list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time plain calls instead of replayed CUDA graphs")
    ap.add_argument("--shape", default=None, help="M,N,K: one dense GEMM instead of a workload")
    ap.add_argument("--shape-fmt", default="uint4", choices=["uint4", "nvfp4", "fp8"],
                    help="--shape weights: W4A16 UINT4 asym g128, or NVFP4 x NVFP4 / FP8 x FP8 quantised in the step")
    args = ap.parse_args()
    ws, rank, local = init_dist()
    if args.impl == "reference":
        return run_reference(args, ws, rank)

    hq = _hq()
    peaks = load_peaks()
    if args.shape:
        M, N, K = (int(x) for x in args.shape.split(","))
        gen = synth.generator(0, "cuda")
        if args.shape_fmt == "uint4":
            ops, keep = ops_shape(hq, M, N, K, gen)
            cfg = {"workload": f"dense W4A16 UINT4 asym g128, M={M}, N={N}, K={K}"}
        else:
            ops, keep = ops_dense_quantised(hq, args.shape_fmt, gen, N=N, K=K, Ms=(M,))
            cfg = {"workload": f"dense {args.shape_fmt} x {args.shape_fmt}, M={M}, N={N}, K={K}"}
        cfg["l2"] = L2_NOTE
    else:
        ops, cfg, keep = WORKLOADS[args.workload](hq)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    flush_sink = torch.empty((), dtype=torch.int64, device="cuda")
    stream = torch.cuda.current_stream()
    n_ops = len(ops)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ops]

    # Each device-resident call is captured once in a CUDA graph and replayed,
    # as a serving loop would, so that the timed region holds the GPU work and
    # not the Python launch path; --eager times the plain calls instead.
    graphs = [None] * n_ops
    if not args.eager:
        try:
            for op in ops:  # first calls (per-device kernel attributes) happen outside capture
                op.run()
            torch.cuda.synchronize()
            for i, op in enumerate(ops):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    op.run()
                graphs[i] = g
            torch.cuda.synchronize()
            cfg["launch"] = "one CUDA graph per call, replayed"
        except Exception as exc:  # capture unsupported: fall back to eager calls
            graphs = [None] * n_ops
            cfg["launch"] = "eager (graph capture failed: %s)" % type(exc).__name__
    else:
        cfg["launch"] = "eager"

    def one_step(timed: bool, e2e: bool = False):
        times = []
        for i, op in enumerate(ops):
            flush.zero_()
            flush_sink.copy_(flush.view(torch.int64).sum())  # leaves the L2 holding clean lines only
            a, b = ev[i]
            a.record(stream)
            if e2e:
                op.e2e()
            elif graphs[i] is not None:
                graphs[i].replay()
            else:
                op.run()
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

    # roofline of the dominant call: the one that takes the most time per step
    # among the five benchmark configurations' calls (the extra rows of the
    # default workload, other formats and modes, are reported in `sweep` only)
    in_cfg = [i for i, op in enumerate(ops) if op.config in (1, 2, 3, 4, 5)]
    i_dom = max(in_cfg, key=lambda i: per_op[i]) if in_cfg else int(np.argmax(per_op))
    dom = ops[i_dom]
    t_dom = per_op[i_dom] / 1e3
    hbm_t = dom.bytes / (peaks["hbm_gbs"] * 1e9)
    peak_fmt = peaks["bf16_tflops"] * dom.peak_ratio
    flop_t = dom.flops / (peak_fmt * 1e12)
    if flop_t >= hbm_t:
        roof = {"bound": "tensor", "achieved": dom.flops / t_dom / 1e12, "peak": peak_fmt, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": dom.bytes / t_dom / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(dom.name)
    roof["algorithmic_bytes"] = dom.bytes
    roof["kernel"] = (dom.kernel or "hq") + " (" + dom.name + ")"
    roof["peak_source"] = peaks["source"] + (" burst" if roof["bound"] == "tensor" else "") + (
        " bf16 x %g (nominal ratio of the MMA kind)" % dom.peak_ratio if roof["bound"] == "tensor" and dom.peak_ratio != 1
        else "")

    sweep = [sweep_entry(op, t, peaks) for op, t in zip(ops, per_op)]
    per_config = {}
    for op, t, e in zip(ops, per_op, sweep):
        pc = per_config.setdefault(str(op.config), {"title": CONFIG_TITLES.get(op.config, ""), "calls": 0,
                                                    "ms": 0.0, "flops": 0.0, "fracs": []})
        pc["calls"] += 1
        pc["ms"] += t
        pc["flops"] += op.flops
        if op.flops > 0:
            pc["fracs"].append(e["roofline_frac"])
    for pc in per_config.values():
        pc["tflops"] = round(pc["flops"] / (pc["ms"] / 1e3) / 1e12, 2) if pc["ms"] > 0 else 0.0
        pc["ms"] = round(pc["ms"], 4)
        fr = pc.pop("fracs")
        pc["roofline_frac_min"] = min(fr) if fr else None
        pc["roofline_frac_max"] = max(fr) if fr else None
        del pc["flops"]
    line = {
        "metric": METRIC,
        "value": value, "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": cfg,
        "e2e": {"value": flops_step * ws / (e2e_ms / 1e3) / 1e12, "unit": "TFLOPS",
                "h2d_bytes_per_step": sum(op.h2d for op in ops), "d2h_bytes_per_step": sum(op.d2h for op in ops)},
        "gpu_launches": sum(op.kernels for op in ops) * args.steps,
        "roofline": roof, "clocks": clk, "per_config": per_config, "sweep": sweep,
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
