"""CPU oracle for the quantised-weight GEMM path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this module.  The product
(``quantized_gemm_02_b200``) never imports it and shares no code with it;
both sides see the same inputs through ``synth`` only.

What it computes, and from where (all pages are about the Humming kernel
library; citations name the page and its section):

* Formats are only named by the pages ("Announcing Humming", section
  "Quantization support"; SGLang PR #23754 digest, section "Mxfp4HummingMoEMethod").
  Their values are decoded here from the bit fields of the public format
  definitions: OCP Microscaling v1.0 (E2M1, E8M0, the MX block rule), OCP
  8-bit floating point (E4M3 "fn": bias 7, no infinities, S.1111.111 = NaN)
  and NVIDIA's NVFP4 (E2M1 values, UE4M3 per-16 scale, FP32 second-level scale).
* Weight semantics follow the unified quantisation description ("Announcing
  Humming", section "Unified quantization representation"): weight format,
  scale granularity, scale dtype, zero point and second-level scale are
  independent.  w = (q - z) * s for integer weights (z = 0 when symmetric);
  w = e2m1 * 2^(c-127) for MXFP4; w = e2m1 * ue4m3 * g for NVFP4;
  w = e4m3 for FP8 with the per-channel scale applied to the output.
* The GEMM is C[m, n] = sum_k a[m, k] * w[n, k] times the per-token /
  per-channel / global scales, in fp64 (numpy matmul as the library step).
* MoE ("Announcing Humming", section "Performance"/WnA16 on Indexed and
  Grouped paths; SGLang PR #23754 digest, humming_moe_runner_core_run and
  moe_fused_mul_sum): out[t] = s_r * sum_j w[t, j] * (a[t] . W_{ids[t, j]}^T).
  The masked layout (same digest, gemm type "grouped_masked" with
  expert_num_tokens and expected_m): expert e multiplies the first
  expert_num_tokens[e] rows of its own fixed-size slab of activation rows.
* Activation quantisers (per-token FP8, MXFP8, NVFP4) use fp32 IEEE
  operations in the stated order with round-to-nearest-even and saturation;
  the pages name the activation formats ("Announcing Humming", sections
  "W8A8 / W4A8 / W4A4" and the usage section's MXFP8 MoE activation
  override) but give no recipe, so the recipes below are the plain readings
  listed in the design notes.

Parity pins live in ``tests/test_oracle_*.py``.  Functions without an
independent pin say "parity unpinned" in their docstring.  The functions of
the last section (FP6, INT1-3, MXINT4 and block-scaled FP8) serve rows that
have no GPU path yet; their element values and reductions are pinned, while
the MXINT4 and INT1-3 code conventions are readings (the pages only name
those formats).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Desc", "e2m1_value", "e4m3_value", "e8m0_value", "E2M1", "E4M3", "E8M0",
    "bf16_to_f64", "e4m3_rn_sat", "e2m1_rn_sat", "unpack_nibbles_i32", "unpack_nibbles_u8",
    "decode_weights", "quant_fp8_per_token", "quant_mxfp8", "quant_nvfp4", "decode_act",
    "gemm", "moe_permute", "moe", "moe_expert_outputs", "moe_masked", "silu_and_mul", "nvfp4_global_scale",
    "fp6_value", "E2M3", "E3M2", "decode_int_weights", "decode_fp6_weights", "decode_mxint4_weights",
    "decode_fp8_block_weights", "quant_fp8_block", "decode_fp8_block_act",
    "unpack_bits", "e0m_value", "E0M3", "E0M7", "int_to_e0m", "decode_lowbit_weights",
]


# ---------------------------------------------------------------------------
# Format definitions (value of every code, from its bit fields)
# ---------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    """E2M1 (OCP MX v1.0 FP4): sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0.  Exponent 0 is subnormal: 0.5 * m."""
    s = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * 0.5 * m
    return s * 2.0 ** (e - 1) * (1.0 + m / 2.0)


def e4m3_value(code: int) -> float:
    """E4M3 "fn" (OCP FP8): sign bit 7, exponent bits 6..3 (bias 7), mantissa
    bits 2..0.  Exponent 0 is subnormal (m/8 * 2^-6).  S.1111.111 is NaN; there
    are no infinities, so the largest finite magnitude is 1.75 * 2^8 = 448."""
    s = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e8m0_value(code: int) -> float:
    """E8M0 (OCP MX v1.0 shared scale): 2^(code - 127); code 255 is NaN."""
    if code == 255:
        return math.nan
    return 2.0 ** (code - 127)


E2M1 = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3 = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
E8M0 = np.array([e8m0_value(c) for c in range(256)], dtype=np.float64)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (bf16 is the top half of an fp32)."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


# ---------------------------------------------------------------------------
# Rounding to a narrow format: round to nearest, ties to even, saturate
# ---------------------------------------------------------------------------

def _round_nonneg(ax: np.ndarray, vals: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of ``vals`` (sorted non-negative magnitudes
    indexed by code) to each ``ax >= 0``; ties go to the even code (the code
    whose mantissa LSB is 0); values above the largest magnitude saturate."""
    ax = np.asarray(ax, dtype=np.float64)
    top = len(vals) - 1
    idx = np.searchsorted(vals, ax, side="left")
    idx = np.clip(idx, 1, top)
    lo = idx - 1
    d_lo = ax - vals[lo]
    d_hi = vals[idx] - ax
    pick = np.where(d_hi < d_lo, idx, lo)
    tie = d_hi == d_lo
    even = np.where(idx % 2 == 0, idx, lo)
    pick = np.where(tie, even, pick)
    pick = np.where(ax >= vals[top], top, pick)
    pick = np.where(ax <= 0.0, 0, pick)
    return pick.astype(np.int64)


def e4m3_rn_sat(x: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 code, RNE, saturating to +-448, IEEE sign kept (so a value
    that rounds to zero keeps its sign bit)."""
    x = np.asarray(x, dtype=np.float32)
    mag = _round_nonneg(np.abs(x), E4M3[:127])
    return (mag | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def e2m1_rn_sat(x: np.ndarray) -> np.ndarray:
    """fp32 -> E2M1 code, RNE, saturating to +-6, IEEE sign kept."""
    x = np.asarray(x, dtype=np.float32)
    mag = _round_nonneg(np.abs(x), E2M1[:8])
    return (mag | np.where(np.signbit(x), 0x8, 0)).astype(np.uint8)


# ---------------------------------------------------------------------------
# Standard-format unpacking
# ---------------------------------------------------------------------------

def unpack_nibbles_i32(words: np.ndarray, n: int) -> np.ndarray:
    """int32 words -> 4-bit fields (uint8 0..15); field j of word w is element 8w+j."""
    w = np.asarray(words).view(np.uint32) if np.asarray(words).dtype == np.int32 else np.asarray(words, dtype=np.uint32)
    out = np.empty((*w.shape, 8), dtype=np.uint8)
    for j in range(8):
        out[..., j] = (w >> np.uint32(4 * j)) & np.uint32(0xF)
    return out.reshape(*w.shape[:-1], w.shape[-1] * 8)[..., :n]


def unpack_nibbles_u8(b: np.ndarray, n: int) -> np.ndarray:
    """bytes -> 4-bit fields; the low nibble is the even element."""
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty((*b.shape, 2), dtype=np.uint8)
    out[..., 0] = b & 0xF
    out[..., 1] = b >> 4
    return out.reshape(*b.shape[:-1], b.shape[-1] * 2)[..., :n]


# ---------------------------------------------------------------------------
# Quantisation description
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Desc:
    """Independent quantisation parameters ("Announcing Humming", section
    "Unified quantization representation").

    w_dtype: 'int4' | 'uint4' | 'e2m1' | 'e4m3'
    w_group: 0 (per output channel) or the K-group size (16, 32, 64, 128)
    w_scale: 'bf16' | 'fp32' | 'e8m0' | 'ue4m3'
    w_zero:  asymmetric zero points (UINT4, same grouping as the scales)
    w_global: FP32 second-level (tensor) scale
    a_dtype: 'bf16' | 'fp8' (per token) | 'mxfp8' | 'nvfp4'
    """
    w_dtype: str
    w_group: int
    w_scale: str
    w_zero: bool = False
    w_global: bool = False
    a_dtype: str = "bf16"


def _signed4(n: np.ndarray) -> np.ndarray:
    """4-bit two's complement field -> integer in [-8, 7]."""
    n = n.astype(np.int64)
    return np.where(n >= 8, n - 16, n)


def decode_weights(d: Desc, N: int, K: int, codes, scales, zeros=None, global_scale=None):
    """Decode one expert's standard-format weights to fp64 ``W [N, K]``.

    Returns ``(W, col_scale)``; ``col_scale`` is the FP8 per-output-channel
    scale that multiplies the output (None for the other formats, whose
    scales are folded into W).
    """
    col = None
    if d.w_dtype in ("int1", "uint1", "int2", "uint2", "int3", "uint3", "e0m3", "e2m3", "e3m2"):
        # the other widths, from the standard b-bit code stream
        z = None if zeros is None else np.asarray(zeros).reshape(N, -1)
        return decode_lowbit_weights(d.w_dtype, np.asarray(codes).reshape(N, -1), scales, K, d.w_group, z), None
    if d.w_dtype in ("int4", "uint4"):
        q = unpack_nibbles_i32(codes, K)
        q = _signed4(q) if d.w_dtype == "int4" else q.astype(np.int64)
        g = K if d.w_group == 0 else d.w_group
        G = K // g
        if d.w_scale == "bf16":
            s = bf16_to_f64(np.asarray(scales).reshape(N, G))
        elif d.w_scale == "fp32":
            s = np.asarray(scales, dtype=np.float32).reshape(N, G).astype(np.float64)
        elif d.w_scale == "e8m0" and d.w_dtype == "int4" and g == 32 and not d.w_zero:
            # MXINT4: the int32 words are the packed bytes (low nibble = even k)
            return decode_mxint4_weights(np.ascontiguousarray(codes).view(np.uint8), scales, K), None
        else:
            raise ValueError(d.w_scale)
        z = np.zeros((N, G), dtype=np.int64)
        if d.w_zero:
            z = unpack_nibbles_i32(zeros, G).astype(np.int64)
        grp = np.arange(K) // g
        W = (q - z[:, grp]).astype(np.float64) * s[:, grp]
    elif d.w_dtype == "e2m1":
        c = unpack_nibbles_u8(codes, K)
        v = E2M1[c]
        if d.w_scale == "e8m0":
            blk = np.arange(K) // 32
            W = v * E8M0[np.asarray(scales).reshape(N, K // 32)][:, blk]
        elif d.w_scale == "ue4m3":
            blk = np.arange(K) // 16
            W = v * E4M3[np.asarray(scales).reshape(N, K // 16)][:, blk]
            if d.w_global:
                W = W * float(np.float32(global_scale))
        else:
            raise ValueError(d.w_scale)
    elif d.w_dtype == "e4m3" and d.w_group == 128:
        # block-scaled FP8: scales [ceil(N / 128), K / 128]
        W = decode_fp8_block_weights(np.asarray(codes).reshape(N, K), np.asarray(scales).reshape(-1, K // 128))
    elif d.w_dtype == "e4m3":
        W = E4M3[np.asarray(codes).reshape(N, K)]
        col = np.asarray(scales, dtype=np.float32).reshape(N).astype(np.float64)
    else:
        raise ValueError(d.w_dtype)
    return W, col


# ---------------------------------------------------------------------------
# Activation quantisers (fp32 IEEE ops in the stated order)
# ---------------------------------------------------------------------------

def quant_fp8_per_token(x_bits: np.ndarray):
    """Per-token FP8: s = amax_row / 448 (fp32), q = e4m3(x / s) (fp32
    division, RNE, saturating).  An all-zero row gets s = 1.  Parity unpinned
    as a recipe (the pages name tokenwise FP8 activations without a recipe);
    its rounding steps are pinned."""
    x = bf16_to_f32(x_bits)
    amax = np.max(np.abs(x), axis=1).astype(np.float32)
    s = (amax / np.float32(448.0)).astype(np.float32)
    s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
    q = e4m3_rn_sat((x / s[:, None]).astype(np.float32))
    return q, s


def _floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for a > 0, exact for normal and subnormal fp32."""
    _, ex = np.frexp(np.asarray(a, dtype=np.float64))
    return ex.astype(np.int64) - 1


def quant_mxfp8(x_bits: np.ndarray):
    """MXFP8 (OCP MX v1.0 rule): per block of 32 along K, shared exponent
    e = floor(log2(amax)) - 8 (8 = emax of E4M3), clamped to [-127, 127],
    stored as E8M0 code e + 127; q = e4m3(x * 2^-e), RNE, saturating.  An
    all-zero block gets code 127 and q = 0."""
    x = bf16_to_f32(x_bits)
    M, K = x.shape
    xb = x.reshape(M, K // 32, 32)
    amax = np.max(np.abs(xb), axis=2)
    e = np.where(amax > 0, _floor_log2(np.where(amax > 0, amax, 1.0)) - 8, 0)
    e = np.clip(e, -127, 127)
    scaled = np.ldexp(xb, (-e)[..., None].astype(np.int32)).astype(np.float32)
    q = e4m3_rn_sat(scaled).reshape(M, K)
    return q, (e + 127).astype(np.uint8)


def nvfp4_global_scale(x_bits: np.ndarray) -> np.float32:
    """The NVFP4 tensor (second-level) scale of a bf16 tensor: g = amax / (448
    * 6) in fp32, 1 for an all-zero tensor.  ``quant_nvfp4`` uses it when no
    static scale is given; quantising some rows of a tensor with
    ``global_scale=nvfp4_global_scale(whole tensor)`` gives those rows' codes
    in the whole tensor's quantisation."""
    x = bf16_to_f32(x_bits)
    amax_t = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    return np.float32(amax_t / np.float32(2688.0)) if amax_t > 0 else np.float32(1.0)


def quant_nvfp4(x_bits: np.ndarray, global_scale=None):
    """NVFP4: g = amax_tensor / (448 * 6) (fp32; 1 if the tensor is zero)
    unless a static ``global_scale`` is given; per block of 16 along K,
    sb = ue4m3(((amax_blk / 6) / g)), d = decode(sb) * g (fp32),
    q = e2m1(x / d), with q = 0 when d == 0.  Returns packed E2M1 codes
    [M, K/2] (low nibble = even k), UE4M3 codes [M, K/16] and g."""
    x = bf16_to_f32(x_bits)
    M, K = x.shape
    g = nvfp4_global_scale(x_bits) if global_scale is None else np.float32(global_scale)
    xb = x.reshape(M, K // 16, 16)
    amax_b = np.max(np.abs(xb), axis=2).astype(np.float32)
    sbv = ((amax_b / np.float32(6.0)).astype(np.float32) / g).astype(np.float32)
    sb = e4m3_rn_sat(sbv)
    d = (E4M3[sb].astype(np.float32) * g).astype(np.float32)
    safe = np.where(d == 0, np.float32(1.0), d).astype(np.float32)
    q = e2m1_rn_sat((xb / safe[..., None]).astype(np.float32))
    q = np.where((d == 0)[..., None], 0, q).astype(np.uint8).reshape(M, K)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb, np.float32(g)


def decode_act(a_dtype: str, M: int, K: int, a, scales=None, global_scale=None):
    """Decode activations to fp64 ``[M, K]`` and the per-row scale (FP8
    per-token; None otherwise).  bf16 activations are taken as they are."""
    row = None
    if a_dtype == "bf16":
        A = bf16_to_f64(np.asarray(a).reshape(M, K))
    elif a_dtype == "fp8":
        A = E4M3[np.asarray(a).reshape(M, K)]
        row = np.asarray(scales, dtype=np.float32).reshape(M).astype(np.float64)
    elif a_dtype == "mxfp8":
        blk = np.arange(K) // 32
        A = E4M3[np.asarray(a).reshape(M, K)] * E8M0[np.asarray(scales).reshape(M, K // 32)][:, blk]
    elif a_dtype == "fp8g":
        # E4M3 with an fp32 scale per token and 128 k (quant_fp8_block)
        A = decode_fp8_block_act(np.asarray(a).reshape(M, K), np.asarray(scales).reshape(M, K // 128))
    elif a_dtype == "nvfp4":
        blk = np.arange(K) // 16
        c = unpack_nibbles_u8(np.asarray(a).reshape(M, K // 2), K)
        A = E2M1[c] * E4M3[np.asarray(scales).reshape(M, K // 16)][:, blk] * float(np.float32(global_scale))
    else:
        raise ValueError(a_dtype)
    return A, row


# ---------------------------------------------------------------------------
# GEMM and MoE
# ---------------------------------------------------------------------------

def gemm(A: np.ndarray, W: np.ndarray, row_scale=None, col_scale=None):
    """C = diag(row_scale) . A . W^T . diag(col_scale) in fp64, plus the
    per-element error scale sum_k |a_k w_k| (with |scales|) used by the
    parity tolerance."""
    out = A @ W.T
    bound = np.abs(A) @ np.abs(W).T
    if row_scale is not None:
        out = out * row_scale[:, None]
        bound = bound * np.abs(row_scale)[:, None]
    if col_scale is not None:
        out = out * col_scale[None, :]
        bound = bound * np.abs(col_scale)[None, :]
    return out, bound


def moe_permute(topk_ids: np.ndarray, E: int):
    """Routing prepare (SGLang PR #23754 digest: moe_permute_prepare /
    moe_align_block_size): the T*k slots (slot = t*k + j) sorted by expert,
    stable in slot order.  Returns (expert_offsets [E+1], perm [T*k] = slot at
    each permuted position, inv_perm [T*k] = permuted position of each slot)."""
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm), dtype=np.int32)
    return offsets, perm, inv


def moe_expert_outputs(A_slots: np.ndarray, topk_ids: np.ndarray, decode_expert, row_scale=None):
    """Y[slot] = a_slot . W_{e(slot)}^T for every slot, in fp64, plus the
    matching error scale.  ``A_slots`` is [T*k, K] (the activation row each
    slot multiplies); ``decode_expert(e)`` returns (W_e [N, K], col_scale_e)."""
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    Y = None
    B = None
    for e in np.unique(flat):
        rows = np.nonzero(flat == e)[0]
        W, col = decode_expert(int(e))
        rs = None if row_scale is None else row_scale[rows]
        y, b = gemm(A_slots[rows], W, rs, col)
        if Y is None:
            Y = np.zeros((len(flat), W.shape[0]))
            B = np.zeros((len(flat), W.shape[0]))
        Y[rows] = y
        B[rows] = b
    return Y, B


def moe(A_slots: np.ndarray, topk_ids: np.ndarray, topk_weights: np.ndarray, decode_expert,
        routed_scale: float = 1.0, row_scale=None):
    """Combined MoE output out[t] = s_r * sum_j w[t, j] * Y[t*k + j] (fp64) and
    its error scale s_r * sum_j |w[t, j]| * B[t*k + j]."""
    T, k = np.asarray(topk_ids).shape
    Y, B = moe_expert_outputs(A_slots, topk_ids, decode_expert, row_scale)
    w = np.asarray(topk_weights, dtype=np.float32).astype(np.float64)
    N = Y.shape[1]
    out = routed_scale * np.einsum("tj,tjn->tn", w, Y.reshape(T, k, N))
    bound = abs(routed_scale) * np.einsum("tj,tjn->tn", np.abs(w), B.reshape(T, k, N))
    return out, bound, Y, B


def moe_masked(A_slab: np.ndarray, counts, slab: int, decode_expert, row_scale=None):
    """Masked-layout MoE expert outputs (SGLang PR #23754 digest:
    humming_moe_runner_core_run, gemm type "grouped_masked"): ``A_slab`` is
    [E * slab, K] (fp64, already decoded); expert e's rows are
    [e * slab, e * slab + c_e) with c_e = clamp(counts[e], 0, slab), and
    Y[e * slab + i] = a . W_e^T for those rows.  Returns (Y, B, valid) with
    Y and B NaN on the rows that are not valid, ``valid`` their mask.  The
    reading that a count outside [0, slab] is clamped is this oracle's (the
    pages state no rule)."""
    E = len(counts)
    R = E * slab
    Y = None
    B = None
    valid = np.zeros(R, dtype=bool)
    for e in range(E):
        c = min(max(int(counts[e]), 0), slab)
        rows = np.arange(e * slab, e * slab + c)
        valid[rows] = True
        W, col = decode_expert(e)
        if Y is None:
            Y = np.full((R, W.shape[0]), np.nan)
            B = np.full((R, W.shape[0]), np.nan)
        if c == 0:
            continue
        rs = None if row_scale is None else row_scale[rows]
        Y[rows], B[rows] = gemm(A_slab[rows], W, rs, col)
    return Y, B, valid


def silu_and_mul(Y: np.ndarray) -> np.ndarray:
    """Gated activation between an MoE layer's gate-up and down GEMMs, in
    fp64: for Y [R, 2I] (gate columns first, then up), out[r, i] =
    silu(Y[r, i]) * Y[r, I + i] with silu(g) = g / (1 + exp(-g)).  The pages
    name no activation; this is the usual gated-MLP form (a reading)."""
    Y = np.asarray(Y, dtype=np.float64)
    I = Y.shape[1] // 2
    g, u = Y[:, :I], Y[:, I:]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u


# ---------------------------------------------------------------------------
# Formats of the rows that come next (oracle first; no GPU path yet): FP6
# and INT1/2/3 weights ("Announcing Humming", section "Performance":
# WnA16 with INT1, INT2, INT3 and FP4 to FP8 weights), MXINT4 weights (same
# section, MoE on B300), FP8 with block scales (section "W8A8 / W4A8 /
# W4A4": block-scaled FP8 W8A8 as on Hopper).
# ---------------------------------------------------------------------------

def fp6_value(code: int, kind: str) -> float:
    """OCP MX v1.0 FP6.  'e2m3': sign bit 5, exponent bits 4..3 (bias 1),
    mantissa bits 2..0; 'e3m2': exponent bits 4..2 (bias 3), mantissa bits
    1..0.  Exponent 0 is subnormal; there are no infinities or NaNs."""
    s = -1.0 if (code >> 5) & 1 else 1.0
    if kind == "e2m3":
        e, m, mb, bias = (code >> 3) & 3, code & 7, 3, 1
    elif kind == "e3m2":
        e, m, mb, bias = (code >> 2) & 7, code & 3, 2, 3
    else:
        raise ValueError(kind)
    if e == 0:
        return s * (m / 2.0 ** mb) * 2.0 ** (1 - bias)
    return s * (1.0 + m / 2.0 ** mb) * 2.0 ** (e - bias)


E2M3 = np.array([fp6_value(c, "e2m3") for c in range(64)], dtype=np.float64)
E3M2 = np.array([fp6_value(c, "e3m2") for c in range(64)], dtype=np.float64)


def decode_int_weights(bits: int, codes, scales, group: int, zeros=None):
    """b-bit integer weights (b in 1..8) from unpacked codes u [N, K] in
    [0, 2^b): w = (u - z) * s with z the per-group zero point when given
    (unsigned codes, as UINT4), else w = q * s with q the b-bit two's
    complement value of u (signed codes, as INT4); s bf16 bits
    [N, K / group] (group 0 = per channel).  The code-level form is this
    oracle's reading: the pages name INT1/2/3 without a packing or a
    signedness rule, so the INT4 rules are carried over."""
    u = np.asarray(codes).astype(np.int64)
    if u.min(initial=0) < 0 or u.max(initial=0) >= (1 << bits):
        raise ValueError("code out of range")
    N, K = u.shape
    g = K if group == 0 else group
    s = bf16_to_f64(np.asarray(scales).reshape(N, K // g))
    grp = np.arange(K) // g
    if zeros is None:
        q = np.where(u >= (1 << (bits - 1)), u - (1 << bits), u)
        return q.astype(np.float64) * s[:, grp]
    z = np.asarray(zeros).astype(np.int64).reshape(N, K // g)
    return (u - z[:, grp]).astype(np.float64) * s[:, grp]


def decode_fp6_weights(kind: str, codes, e8m0_scales):
    """MXFP6 weights (OCP MX v1.0): FP6 codes [N, K] (one per byte, low 6
    bits) with an E8M0 scale per 32 along K: w = fp6 * 2^(c - 127)."""
    c = np.asarray(codes).astype(np.int64)
    N, K = c.shape
    table = E2M3 if kind == "e2m3" else E3M2
    blk = np.arange(K) // 32
    return table[c & 63] * E8M0[np.asarray(e8m0_scales).reshape(N, K // 32)][:, blk]


def decode_mxint4_weights(codes, e8m0_scales, K: int):
    """MXINT4 weights: packed 4-bit two's complement codes [N, K/2] (low
    nibble = even k) with an E8M0 scale per 32 along K: w = q * 2^(c - 127).
    Reading: the pages name MXINT4 only; this is MXFP4's layout with INT4
    elements and no further element scale."""
    q = _signed4(unpack_nibbles_u8(codes, K)).astype(np.float64)
    N = q.shape[0]
    blk = np.arange(K) // 32
    return q * E8M0[np.asarray(e8m0_scales).reshape(N, K // 32)][:, blk]


def decode_fp8_block_weights(codes, scales, block: int = 128, row_block=None):
    """FP8 weights with block scales: E4M3 codes [N, K] and fp32 scales
    [ceil(N / row_block), K / block], one per row_block x block tile
    (row_block defaults to block: square blocks):
    w[n, k] = e4m3(code) * s[n // row_block, k // block].  row_block = 1
    takes one scale row per weight row (a block's scale row repeated), for
    decoding some rows of a matrix."""
    c = np.asarray(codes)
    N, K = c.shape
    rb = block if row_block is None else row_block
    s = np.asarray(scales, dtype=np.float32).astype(np.float64)
    return E4M3[c] * s[np.arange(N)[:, None] // rb, np.arange(K)[None, :] // block]


def quant_fp8_block(x_bits: np.ndarray, group: int = 128):
    """FP8 activations with a scale per token and per `group` along K:
    s = amax_group / 448 (fp32), q = e4m3(x / s), RNE, saturating; an
    all-zero group gets s = 1 (the per-token recipe applied to each group).
    Returns codes [M, K] and fp32 scales [M, K / group]."""
    x = bf16_to_f32(x_bits)
    M, K = x.shape
    xg = x.reshape(M, K // group, group)
    amax = np.max(np.abs(xg), axis=2).astype(np.float32)
    s = (amax / np.float32(448.0)).astype(np.float32)
    s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
    q = e4m3_rn_sat((xg / s[..., None]).astype(np.float32)).reshape(M, K)
    return q, s


def decode_fp8_block_act(codes, scales, group: int = 128):
    """Decode block-scaled FP8 activations to fp64 [M, K]."""
    c = np.asarray(codes)
    M, K = c.shape
    s = np.asarray(scales, dtype=np.float32).astype(np.float64).reshape(M, K // group)
    return E4M3[c] * s[:, np.arange(K) // group]


# ---------------------------------------------------------------------------
# Standard format of b-bit weight codes and the zero-exponent float view
# ("Announcing Humming", section "Quantization support": a float format with
# no exponent bits whose values are the symmetric integers of its width,
# e.g. float8e0m7 and INT8 without -128 both hold -127..127; symmetric INT
# weights that fit are converted to it; section "Performance", WnA16:
# INT1/2/3 and FP4 to FP8 weights)
# ---------------------------------------------------------------------------

def unpack_bits(packed, bits: int, K: int) -> np.ndarray:
    """b-bit codes from a little-endian bit stream per row: element k of a row
    occupies bits [b*k, b*k + b) of the row's bytes (bit 0 = the least
    significant bit of byte 0).  For b = 4 this is the INT4 / E2M1 nibble
    order.  Reading: the pages give no packing for INT1/2/3 or FP6; this is
    the plain stream."""
    by = np.asarray(packed, dtype=np.uint8)
    bitsarr = np.unpackbits(by, axis=-1, bitorder="little")[..., :bits * K]
    bitsarr = bitsarr.reshape(*by.shape[:-1], K, bits).astype(np.int64)
    return (bitsarr << np.arange(bits, dtype=np.int64)).sum(axis=-1)


def e0m_value(code: int, bits: int) -> float:
    """Float with zero exponent bits and (bits - 1) mantissa bits
    (float4e0m3, float8e0m7): the sign bit, then the magnitude m read as an
    integer; the value is -m or m (code 1 << (bits - 1) is -0)."""
    m = code & ((1 << (bits - 1)) - 1)
    return -float(m) if (code >> (bits - 1)) & 1 else float(m)


E0M3 = np.array([e0m_value(c, 4) for c in range(16)], dtype=np.float64)
E0M7 = np.array([e0m_value(c, 8) for c in range(256)], dtype=np.float64)


def int_to_e0m(q, bits: int) -> np.ndarray:
    """Symmetric integers |q| <= 2^(bits - 1) - 1 to their zero-exponent
    codes (sign bit and magnitude); q = 0 gives +0."""
    q = np.asarray(q, dtype=np.int64)
    lim = (1 << (bits - 1)) - 1
    if np.any(np.abs(q) > lim):
        raise ValueError("not a symmetric integer of this width")
    return (np.where(q < 0, 1 << (bits - 1), 0) | np.abs(q)).astype(np.int64)


def decode_lowbit_weights(kind: str, packed, scales, K: int, group: int = 0, zeros=None):
    """Weights of the other WnA16 widths from the standard bit stream
    (``unpack_bits``) [N, K * b / 8] bytes:
      'int1' / 'int2' / 'int3': signed b-bit two's complement times bf16
          group scales (INT1: codes 0 and -1);
      'uint1' / 'uint2' / 'uint3': (u - z) times bf16 group scales, z uint8
          [N, K/group];
      'e0m3': float4e0m3 times bf16 group scales;
      'e2m3' / 'e3m2': MXFP6 with an E8M0 scale per 32."""
    if kind in ("int1", "uint1", "int2", "int3", "uint2", "uint3"):
        b = int(kind[-1])
        u = unpack_bits(packed, b, K)
        return decode_int_weights(b, u, scales, group, zeros if kind.startswith("u") else None)
    if kind == "e0m3":
        c = unpack_bits(packed, 4, K)
        N = c.shape[0]
        g = K if group == 0 else group
        s = bf16_to_f64(np.asarray(scales).reshape(N, K // g))
        return E0M3[c] * s[:, np.arange(K) // g]
    if kind in ("e2m3", "e3m2"):
        return decode_fp6_weights(kind, unpack_bits(packed, 6, K), scales)
    raise ValueError(kind)
