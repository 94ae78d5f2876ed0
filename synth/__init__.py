"""Seeded synthetic inputs in the library's standard caller-facing formats.

This module is the only code shared by the CPU oracle and the CUDA path. It
draws random numbers and lays them out in the formats the C-ABI accepts; it
contains none of the method's arithmetic (no decoding, scaling, quantisation
or GEMM).  Every generator takes a ``torch.Generator`` and a device, so the
same recipe produces small CPU tensors for parity tests and multi-GB device
tensors for benchmarks.

Standard formats (the independent parameters of "Announcing Humming",
section "Unified quantization representation": weight format, scale
granularity, scale dtype, zero point, second-level scale):

* INT4 / UINT4 codes: int32 ``[E, N, K/8]``; nibble ``j`` (bits 4j..4j+3, LSB
  first) of word ``w`` holds the code for ``k = 8w + j``.  INT4 nibbles are
  two's complement, UINT4 nibbles are raw 0..15.
* INT4 zero points (asymmetric): int32 ``[E, N, ceil(G/8)]`` packed the same
  way along the group axis (``G = K / group``).
* INT4 scales: bf16 ``[E, N, G]``.
* E2M1 codes: uint8 ``[E, N, K/2]``; low nibble = even ``k``.
* E8M0 scales (MX, block 32): uint8 ``[E, N, K/32]``.
* NVFP4: E2M1 codes + UE4M3 scales uint8 ``[E, N, K/16]`` + fp32 global ``[E]``.
* FP8 E4M3: uint8 ``[E, N, K]`` + fp32 per-channel scales ``[E, N]``.
* Activations: bf16 ``[M, K]``.
* Routing: ``topk_ids`` int32 ``[T, k]``, ``topk_weights`` fp32 ``[T, k]``.

Uniform 4-bit codes are drawn as uniform random bytes: each byte is two
independent uniform nibbles, so a uniform byte stream is exactly "codes
uniform over all 16 values" for INT4 ([-8, 7]), UINT4 ([0, 15]) and E2M1.
"""
from __future__ import annotations

import numpy as np
import torch

__all__ = [
    "generator", "bf16_normal", "random_bytes", "int4_weights", "lowbit_weights", "mxint4_weights",
    "mxfp4_weights",
    "nvfp4_weights_random", "fp8_weights_random", "fp8_block_weights", "routing_softmax_topk", "routing_zipf",
    "pack_nibbles_i32", "pack_nibbles_u8", "to_np_bits",
]


def generator(seed: int = 0, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def bf16_normal(shape, gen: torch.Generator, std: float = 1.0, device: str = "cpu") -> torch.Tensor:
    """bf16 N(0, std^2) samples."""
    x = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def random_bytes(shape, gen: torch.Generator, device: str = "cpu") -> torch.Tensor:
    """Uniform random uint8."""
    return torch.randint(0, 256, tuple(shape), generator=gen, dtype=torch.uint8, device=device)


def to_np_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a tensor as a numpy array (bf16 -> uint16)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def pack_nibbles_i32(nib: np.ndarray) -> np.ndarray:
    """Pack 4-bit fields (0..15, last axis a multiple of 8) into int32 words.

    Field ``j`` of word ``w`` sits at bits ``4j..4j+3`` and holds element ``8w+j``.
    """
    nib = np.asarray(nib, dtype=np.uint32) & 0xF
    *lead, n = nib.shape
    assert n % 8 == 0
    v = nib.reshape(*lead, n // 8, 8)
    out = np.zeros((*lead, n // 8), dtype=np.uint32)
    for j in range(8):
        out |= v[..., j] << np.uint32(4 * j)
    return out.view(np.int32)


def pack_nibbles_u8(nib: np.ndarray) -> np.ndarray:
    """Pack 4-bit fields into bytes: low nibble = even index."""
    nib = np.asarray(nib, dtype=np.uint8) & 0xF
    *lead, n = nib.shape
    assert n % 2 == 0
    v = nib.reshape(*lead, n // 2, 2)
    return (v[..., 0] | (v[..., 1] << 4)).astype(np.uint8)


def _scales_bf16(shape, gen, device):
    # |N(0, 0.02)| + 1e-3, rounded to bf16
    s = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device).abs() * 0.02 + 1e-3
    return s.to(torch.bfloat16)


def int4_weights(E: int, N: int, K: int, group: int, asym: bool, gen: torch.Generator,
                 device: str = "cpu") -> dict:
    """INT4 weights with bf16 group scales (+ UINT4 zero points if ``asym``).

    Codes are uniform over the 16 nibble values: [-8, 7] read as INT4,
    [0, 15] read as UINT4.  Zero points are uniform in [0, 15].
    ``group == 0`` means one scale per output channel.
    """
    G = 1 if group == 0 else K // group
    codes = random_bytes((E, N, K // 2), gen, device).view(torch.int32)
    scales = _scales_bf16((E, N, G), gen, device)
    zeros = None
    if asym:
        gw = (G + 7) // 8
        z = random_bytes((E, N, gw * 4), gen, device).view(torch.int32)
        if G % 8:
            # unused trailing nibbles are zero
            keep = (1 << (4 * (G % 8))) - 1
            z[..., -1] &= keep
        zeros = z
    return {"codes": codes, "scales": scales, "zeros": zeros}


def lowbit_weights(E: int, N: int, K: int, bits: int, group: int, zero: bool, e8m0: bool, gen: torch.Generator,
                   device: str = "cpu") -> dict:
    """b-bit codes (b = 2, 3, 6, or 4 for float4e0m3) as the standard
    little-endian bit stream: uniform random bytes are uniform codes.
    Scales: bf16 |N(0, 0.02)| + 1e-3 per group, or (e8m0) E8M0 exponents
    uniform over [-8, -4] per 32; zero points uint8 uniform in [0, 2^b)."""
    codes = random_bytes((E, N, K * bits // 8), gen, device)
    G = 1 if group == 0 else K // group
    if e8m0:
        scales = torch.randint(119, 124, (E, N, K // 32), generator=gen, dtype=torch.int32, device=device)
        scales = scales.to(torch.uint8)
    else:
        scales = _scales_bf16((E, N, G), gen, device)
    zeros = None
    if zero:
        zeros = torch.randint(0, 1 << bits, (E, N, G), generator=gen, dtype=torch.int32, device=device)
        zeros = zeros.to(torch.uint8)
    return {"codes": codes, "scales": scales, "zeros": zeros}


def mxint4_weights(E: int, N: int, K: int, gen: torch.Generator, exp_lo: int = -8, exp_hi: int = -4,
                   device: str = "cpu") -> dict:
    """MXINT4: INT4 codes uniform over all 16 nibbles (int32 words as for
    INT4); E8M0 scale exponents uniform over the integers [exp_lo, exp_hi]."""
    codes = random_bytes((E, N, K // 2), gen, device).view(torch.int32)
    e = torch.randint(exp_lo + 127, exp_hi + 128, (E, N, K // 32), generator=gen,
                      dtype=torch.int32, device=device)
    return {"codes": codes, "scales": e.to(torch.uint8)}


def mxfp4_weights(E: int, N: int, K: int, gen: torch.Generator, exp_lo: int = -8, exp_hi: int = -4,
                  device: str = "cpu") -> dict:
    """E2M1 codes uniform over all 16 codes (incl. -0); E8M0 scale exponents
    uniform over the integers [exp_lo, exp_hi] (codes exp + 127)."""
    codes = random_bytes((E, N, K // 2), gen, device)
    e = torch.randint(exp_lo + 127, exp_hi + 128, (E, N, K // 32), generator=gen,
                      dtype=torch.int32, device=device)
    return {"codes": codes, "scales": e.to(torch.uint8)}


def nvfp4_weights_random(E: int, N: int, K: int, gen: torch.Generator, device: str = "cpu") -> dict:
    """NVFP4 weights drawn directly as codes (for expert sets too large to
    quantise from a float tensor): E2M1 codes uniform over 16 codes; UE4M3
    scale codes uniform over [0x28, 0x4F] (0.25 .. 3.75); global scale 1/64."""
    codes = random_bytes((E, N, K // 2), gen, device)
    sc = torch.randint(0x28, 0x50, (E, N, K // 16), generator=gen, dtype=torch.int32, device=device)
    g = torch.full((E,), 1.0 / 64.0, dtype=torch.float32, device=device)
    return {"codes": codes, "scales": sc.to(torch.uint8), "global": g}


def fp8_weights_random(E: int, N: int, K: int, gen: torch.Generator, device: str = "cpu") -> dict:
    """E4M3 codes uniform over the 254 finite codes (the two NaN codes
    0x7F / 0xFF are never drawn); fp32 per-channel scales |N(0, 0.01)| + 1e-3."""
    r = torch.randint(0, 254, (E, N, K), generator=gen, dtype=torch.int32, device=device)
    codes = (r + (r >= 0x7F).to(torch.int32)).to(torch.uint8)
    sc = torch.randn(E, N, generator=gen, dtype=torch.float32, device=device).abs() * 0.01 + 1e-3
    return {"codes": codes, "scales": sc}


def fp8_block_weights(E: int, N: int, K: int, gen: torch.Generator, device: str = "cpu") -> dict:
    """E4M3 codes uniform over the 254 finite codes; one fp32 scale per 128
    rows x 128 k, |N(0, 0.01)| + 1e-3: scales [E, ceil(N / 128), K / 128]."""
    r = torch.randint(0, 254, (E, N, K), generator=gen, dtype=torch.int32, device=device)
    codes = (r + (r >= 0x7F).to(torch.int32)).to(torch.uint8)
    sc = torch.randn(E, (N + 127) // 128, K // 128, generator=gen, dtype=torch.float32, device=device).abs() * 0.01
    return {"codes": codes, "scales": sc + 1e-3}


def routing_softmax_topk(T: int, E: int, k: int, gen: torch.Generator, device: str = "cpu"):
    """Router: N(0,1) logits [T, E], softmax, top-k by probability (ties to
    the lower expert index).  The selected probabilities are the weights, not
    renormalised."""
    logits = torch.randn(T, E, generator=gen, dtype=torch.float32, device=device)
    p = torch.softmax(logits, dim=-1)
    w, ids = torch.topk(p, k, dim=-1, largest=True, sorted=True)
    return ids.to(torch.int32), w.to(torch.float32)


def routing_zipf(T: int, E: int, k: int, s: float, gen: torch.Generator, device: str = "cpu"):
    """Zipf(s) expert popularity: a fixed random permutation ranks the
    experts, p_e is proportional to rank^-s; each token draws k distinct
    experts by Gumbel-top-k on log p_e (sampling without replacement);
    weights are a softmax of fresh N(0,1) logits over the k selected."""
    perm = torch.randperm(E, generator=gen, device=device)
    rank = torch.empty(E, dtype=torch.float32, device=device)
    rank[perm] = torch.arange(1, E + 1, dtype=torch.float32, device=device)
    logp = -s * torch.log(rank)
    u = torch.rand(T, E, generator=gen, dtype=torch.float32, device=device).clamp_(1e-12, 1.0 - 1e-7)
    gumbel = -torch.log(-torch.log(u))
    _, ids = torch.topk(logp[None, :] + gumbel, k, dim=-1)
    wl = torch.randn(T, k, generator=gen, dtype=torch.float32, device=device)
    w = torch.softmax(wl, dim=-1)
    return ids.to(torch.int32), w.to(torch.float32)
