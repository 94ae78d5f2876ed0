"""Test helpers: format catalogue, seeded inputs, and the two sides of a
parity check (the CUDA path through the C-ABI binding, the oracle on CPU).

The two sides meet only here, in the tests; they share nothing but the
seeded inputs from ``synth``.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import synth

# weight formats: name -> (C desc fields, oracle Desc kwargs)
WFORMATS = {
    "int4_g128": (dict(w_dtype=2, w_group=128, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                  dict(w_dtype="int4", w_group=128, w_scale="bf16")),
    "int4_g32": (dict(w_dtype=2, w_group=32, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                 dict(w_dtype="int4", w_group=32, w_scale="bf16")),
    "int4_ch": (dict(w_dtype=2, w_group=0, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                dict(w_dtype="int4", w_group=0, w_scale="bf16")),
    "uint4_g128": (dict(w_dtype=3, w_group=128, w_scale_dtype=0, w_has_zero=1, w_has_global=0),
                   dict(w_dtype="uint4", w_group=128, w_scale="bf16", w_zero=True)),
    "uint4_g64": (dict(w_dtype=3, w_group=64, w_scale_dtype=0, w_has_zero=1, w_has_global=0),
                  dict(w_dtype="uint4", w_group=64, w_scale="bf16", w_zero=True)),
    "mxfp4": (dict(w_dtype=4, w_group=32, w_scale_dtype=6, w_has_zero=0, w_has_global=0),
              dict(w_dtype="e2m1", w_group=32, w_scale="e8m0")),
    "nvfp4": (dict(w_dtype=4, w_group=16, w_scale_dtype=7, w_has_zero=0, w_has_global=1),
              dict(w_dtype="e2m1", w_group=16, w_scale="ue4m3", w_global=True)),
    "fp8": (dict(w_dtype=5, w_group=0, w_scale_dtype=1, w_has_zero=0, w_has_global=0),
            dict(w_dtype="e4m3", w_group=0, w_scale="fp32")),
    "mxint4": (dict(w_dtype=2, w_group=32, w_scale_dtype=6, w_has_zero=0, w_has_global=0),
               dict(w_dtype="int4", w_group=32, w_scale="e8m0")),
    "int1_g128": (dict(w_dtype=17, w_group=128, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                  dict(w_dtype="int1", w_group=128, w_scale="bf16")),
    "uint1_g64": (dict(w_dtype=18, w_group=64, w_scale_dtype=0, w_has_zero=1, w_has_global=0),
                  dict(w_dtype="uint1", w_group=64, w_scale="bf16", w_zero=True)),
    "int2_g64": (dict(w_dtype=10, w_group=64, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                 dict(w_dtype="int2", w_group=64, w_scale="bf16")),
    "uint2_g32": (dict(w_dtype=11, w_group=32, w_scale_dtype=0, w_has_zero=1, w_has_global=0),
                  dict(w_dtype="uint2", w_group=32, w_scale="bf16", w_zero=True)),
    "int3_g128": (dict(w_dtype=12, w_group=128, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                  dict(w_dtype="int3", w_group=128, w_scale="bf16")),
    "uint3_g64": (dict(w_dtype=13, w_group=64, w_scale_dtype=0, w_has_zero=1, w_has_global=0),
                  dict(w_dtype="uint3", w_group=64, w_scale="bf16", w_zero=True)),
    "e2m3": (dict(w_dtype=14, w_group=32, w_scale_dtype=6, w_has_zero=0, w_has_global=0),
             dict(w_dtype="e2m3", w_group=32, w_scale="e8m0")),
    "e3m2": (dict(w_dtype=15, w_group=32, w_scale_dtype=6, w_has_zero=0, w_has_global=0),
             dict(w_dtype="e3m2", w_group=32, w_scale="e8m0")),
    "e0m3_g128": (dict(w_dtype=16, w_group=128, w_scale_dtype=0, w_has_zero=0, w_has_global=0),
                  dict(w_dtype="e0m3", w_group=128, w_scale="bf16")),
    # block-scaled FP8 (128 x 128 weight blocks); only with "fp8g" activations
    "fp8b": (dict(w_dtype=5, w_group=128, w_scale_dtype=1, w_has_zero=0, w_has_global=0),
             dict(w_dtype="e4m3", w_group=128, w_scale="fp32")),
}
PAIR_ONLY = {"fp8b": "fp8g"}  # weight formats that exist with one activation format only
LOWBIT = {"int1_g128": 1, "uint1_g64": 1, "int2_g64": 2, "uint2_g32": 2, "int3_g128": 3, "uint3_g64": 3, "e2m3": 6, "e3m2": 6, "e0m3_g128": 4}
AFORMATS = {"bf16": 0, "fp8": 5, "mxfp8": 8, "nvfp4": 9, "fp8g": 5}
AGROUP = {"fp8g": 128}  # E4M3 with an fp32 scale per token and 128 k


def cdesc(wname: str, aname: str = "bf16"):
    import quantized_gemm_02_b200 as hq
    d = hq.QuantDesc(**WFORMATS[wname][0])
    d.a_dtype = AFORMATS[aname]
    d.a_group = AGROUP.get(aname, 0)
    return d


def odesc(wname: str, aname: str = "bf16") -> O.Desc:
    return O.Desc(**WFORMATS[wname][1], a_dtype=aname)


def make_weights(wname: str, E: int, N: int, K: int, seed: int = 0, device: str = "cpu") -> dict:
    """Standard-format weights for E experts (torch tensors on ``device``)."""
    g = synth.generator(seed, device)
    fields, _ = WFORMATS[wname]
    if wname == "mxint4":
        w = synth.mxint4_weights(E, N, K, g, device=device)
        return {"codes": w["codes"], "scales": w["scales"], "zeros": None, "global": None}
    if wname == "fp8b":
        w = synth.fp8_block_weights(E, N, K, g, device)
        return {"codes": w["codes"], "scales": w["scales"], "zeros": None, "global": None}
    if wname in LOWBIT:
        w = synth.lowbit_weights(E, N, K, LOWBIT[wname], fields["w_group"], bool(fields["w_has_zero"]),
                                 fields["w_scale_dtype"] == 6, g, device)
        return {"codes": w["codes"], "scales": w["scales"], "zeros": w["zeros"], "global": None}
    if fields["w_dtype"] in (2, 3):
        w = synth.int4_weights(E, N, K, fields["w_group"], fields["w_dtype"] == 3, g, device)
        return {"codes": w["codes"], "scales": w["scales"], "zeros": w["zeros"], "global": None}
    if wname == "mxfp4":
        w = synth.mxfp4_weights(E, N, K, g, device=device)
        return {"codes": w["codes"], "scales": w["scales"], "zeros": None, "global": None}
    if wname == "nvfp4":
        w = synth.nvfp4_weights_random(E, N, K, g, device)
        return {"codes": w["codes"], "scales": w["scales"], "zeros": None, "global": w["global"]}
    w = synth.fp8_weights_random(E, N, K, g, device)
    return {"codes": w["codes"], "scales": w["scales"], "zeros": None, "global": None}


def np_bits(t):
    return None if t is None else synth.to_np_bits(t)


def oracle_decoder(wname: str, w: dict, N: int, K: int):
    """decode_expert(e) for the oracle, from CPU copies of the inputs."""
    d = odesc(wname)
    codes = np_bits(w["codes"])
    scales = np_bits(w["scales"])
    zeros = np_bits(w["zeros"])
    glob = np_bits(w["global"])

    def dec(e, rows=None):
        if wname == "fp8b":
            # block scales: the rows' own scale rows
            rr = np.arange(N) if rows is None else np.asarray(rows)
            return O.decode_fp8_block_weights(codes[e][rr], scales[e][rr // 128], 128, row_block=1), None
        c, s = codes[e], scales[e]
        z = None if zeros is None else zeros[e]
        if rows is not None:
            c, s = c[rows], s[rows]
            z = None if z is None else z[rows]
        n = N if rows is None else len(rows)
        return O.decode_weights(d, n, K, c, s, z, None if glob is None else glob[e])

    return dec


def gpu_pack(wname: str, w: dict, E: int, N: int, K: int, aname: str = "bf16"):
    """Packs for the description the GEMM will use: the packed layout depends
    on the activation format (block-scaled layouts for MXFP4 x MXFP8 and
    NVFP4 x NVFP4)."""
    import quantized_gemm_02_b200 as hq
    d = cdesc(wname, aname)
    nbytes = hq.hq_packed_weights_bytes(d, E, N, K)
    assert nbytes > 0
    packed = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    cu = {k: (None if v is None else v.cuda()) for k, v in w.items()}
    hq.hq_pack_weights(d, E, N, K, cu["codes"], cu["scales"], cu["zeros"], cu["global"], packed)
    return packed


def act_storage(aname: str, M: int, K: int, device="cuda"):
    """Empty code / scale tensors for a quantised activation format."""
    if aname == "fp8g":
        return (torch.empty(M, K, dtype=torch.uint8, device=device),
                torch.empty(M, K // 128, dtype=torch.float32, device=device))
    if aname == "fp8":
        return (torch.empty(M, K, dtype=torch.uint8, device=device), torch.empty(M, dtype=torch.float32, device=device))
    if aname == "mxfp8":
        return (torch.empty(M, K, dtype=torch.uint8, device=device),
                torch.empty(M, K // 32, dtype=torch.uint8, device=device))
    return (torch.empty(M, K // 2, dtype=torch.uint8, device=device),
            torch.empty(M, K // 16, dtype=torch.uint8, device=device))


def gpu_quant(aname: str, x: torch.Tensor, static_global=None):
    """hq_quant_act on a bf16 CUDA tensor; returns (codes, scales, global)."""
    import quantized_gemm_02_b200 as hq
    M, K = x.shape
    codes, scales = act_storage(aname, M, K)
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    hq.hq_quant_act(cdesc("int4_g128", aname), M, K, x, codes, scales, g, static_global, ws, ws.numel())
    return codes, scales, g


def oracle_quant(aname: str, x_bits: np.ndarray):
    if aname == "fp8g":
        q, s = O.quant_fp8_block(x_bits)
        return q, s, None
    if aname == "fp8":
        q, s = O.quant_fp8_per_token(x_bits)
        return q, s, None
    if aname == "mxfp8":
        q, s = O.quant_mxfp8(x_bits)
        return q, s, None
    return O.quant_nvfp4(x_bits)


def assert_close(gpu_bf16: torch.Tensor, ref: np.ndarray, bound: np.ndarray, rel=4e-3, abs_=1e-5, what=""):
    g = gpu_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    tol = rel * bound + abs_
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at {tuple(i)}: "
            f"gpu={g[tuple(i)]!r} oracle={ref[tuple(i)]!r} tol={tol[tuple(i)]!r}; max err/bound "
            f"{float(np.max(err / np.maximum(bound, 1e-30))):.3e}")
    return float(np.max(err / np.maximum(bound, 1e-30)))
