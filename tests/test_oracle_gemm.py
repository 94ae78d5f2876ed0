"""Pins for the oracle's weight decoding, GEMM and MoE.

* Closed forms: when every weight decodes to the same value c, every output
  is c * sum_k a[m, k] (the "K * scale * sum(a)" reading).
* One-hot activations pick single decoded weights, compared with values
  worked out by hand from the standard format.
* Brute force on tiny shapes: a second decoder written with different
  primitives (hex digits, the golden E2M1 table, torch float8 casts) and
  pure-Python fsum dot products.
* MoE: E = 1 with top-1 and weight 1 is the dense GEMM; relabelling experts
  changes nothing; the permutation matches a brute-force listing.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from conftest import read_golden

E2M1_GOLD = {int(c): float(v) for c, v in read_golden("e2m1_values.txt")}


def _a(M, K, seed=0):
    g = synth.generator(seed)
    x = synth.bf16_normal((M, K), g)
    return synth.to_np_bits(x), x.to(torch.float64).numpy()


def _rowsum(af):
    return np.array([math.fsum(r) for r in af])


@pytest.mark.parametrize("case", ["int4", "uint4", "mxfp4", "nvfp4", "fp8"])
def test_constant_weight_closed_form(case):
    M, N, K = 5, 7, 256
    ab, af = _a(M, K)
    if case == "int4":
        d = O.Desc("int4", 128, "bf16")
        codes = np.full((N, K // 8), 0x33333333, dtype=np.int64).astype(np.int32)  # q = 3
        scales = np.full((N, 2), 0x3F00, dtype=np.uint16)  # bf16 0.5
        c = 1.5
        W, col = O.decode_weights(d, N, K, codes, scales)
    elif case == "uint4":
        d = O.Desc("uint4", 64, "bf16", w_zero=True)
        codes = np.full((N, K // 8), 0x99999999 - 2 ** 32, dtype=np.int64).astype(np.int32)  # q = 9
        scales = np.full((N, 4), 0x3E80, dtype=np.uint16)  # bf16 0.25
        zeros = np.full((N, 1), 0x4444, dtype=np.int32)  # z = 4 for the 4 groups
        c = (9 - 4) * 0.25
        W, col = O.decode_weights(d, N, K, codes, scales, zeros)
    elif case == "mxfp4":
        d = O.Desc("e2m1", 32, "e8m0")
        codes = np.full((N, K // 2), 0x33, dtype=np.uint8)  # 1.5
        scales = np.full((N, K // 32), 125, dtype=np.uint8)  # 2^-2
        c = 0.375
        W, col = O.decode_weights(d, N, K, codes, scales)
    elif case == "nvfp4":
        d = O.Desc("e2m1", 16, "ue4m3", w_global=True)
        codes = np.full((N, K // 2), 0x55, dtype=np.uint8)  # 3.0
        scales = np.full((N, K // 16), 0x38, dtype=np.uint8)  # 1.0
        c = 0.75
        W, col = O.decode_weights(d, N, K, codes, scales, global_scale=0.25)
    else:
        d = O.Desc("e4m3", 0, "fp32")
        codes = np.full((N, K), 0x40, dtype=np.uint8)  # 2.0
        scales = np.full((N,), 1.5, dtype=np.float32)
        c = 3.0
        W, col = O.decode_weights(d, N, K, codes, scales)
    out, bound = O.gemm(af, W, None, col)
    want = c * _rowsum(af)
    assert np.allclose(out, want[:, None], rtol=1e-12, atol=1e-12)
    assert np.allclose(bound, abs(c) * _rowsum(np.abs(af))[:, None], rtol=1e-12)


def test_one_hot_picks_hand_decoded_weights():
    K = 32
    eye = np.eye(K)
    # INT4 symmetric: nibbles 0..15 read as 0..7, -8..-1; one scale of 2.0
    d = O.Desc("int4", 0, "bf16")
    codes = np.array([[0x76543210, np.uint32(0xFEDCBA98).view(np.int32), 0, 0x11111111]], dtype=np.int32)
    W, _ = O.decode_weights(d, 1, K, codes, np.array([[0x4000]], dtype=np.uint16))
    out, _ = O.gemm(eye, W)
    want = [2.0 * v for v in list(range(8)) + list(range(-8, 0)) + [0] * 8 + [1] * 8]
    assert out[:, 0].tolist() == want
    # UINT4 with zero point 3 in group 0 and 12 in group 1 (group 16), scale 1
    d = O.Desc("uint4", 16, "bf16", w_zero=True)
    zeros = np.array([[0xC3]], dtype=np.int32)
    sc = np.array([[0x3F80, 0x3F80]], dtype=np.uint16)
    W, _ = O.decode_weights(d, 1, K, codes, sc, zeros)
    out, _ = O.gemm(eye, W)
    want = [v - 3 for v in range(16)] + [0 - 12] * 8 + [1 - 12] * 8
    assert out[:, 0].tolist() == want
    # MXFP4: byte 0x4F = (k0: code 15 = -6, k1: code 4 = 2) with scale 2^3
    d = O.Desc("e2m1", 32, "e8m0")
    b = np.zeros((1, 16), dtype=np.uint8)
    b[0, 0] = 0xF4
    b[0, 1] = 0x9A
    W, _ = O.decode_weights(d, 1, K, b, np.array([[130]], dtype=np.uint8))
    out, _ = O.gemm(eye, W)
    assert out[:4, 0].tolist() == [2.0 * 8, -6.0 * 8, -1.0 * 8, -0.5 * 8]


def _indep_decode(desc, N, K, codes, scales, zeros=None, gscale=None):
    """Second decoder: hex digits, golden tables, torch casts, Python loops."""
    f8 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).tolist()
    e8 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64).tolist()

    def bf16(bits):
        return torch.tensor([int(bits)], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).item()

    def nib_word(word, j):
        h = "%08x" % (int(word) & 0xFFFFFFFF)
        return int(h[7 - j], 16)

    W = [[0.0] * K for _ in range(N)]
    for n in range(N):
        for k in range(K):
            if desc.w_dtype in ("int4", "uint4"):
                v = nib_word(codes[n][k // 8], k % 8)
                if desc.w_dtype == "int4" and v > 7:
                    v -= 16
                g = K if desc.w_group == 0 else desc.w_group
                z = nib_word(zeros[n][(k // g) // 8], (k // g) % 8) if desc.w_zero else 0
                W[n][k] = (v - z) * bf16(scales[n][k // g])
            elif desc.w_dtype == "e2m1":
                byte = int(codes[n][k // 2])
                v = E2M1_GOLD[(byte >> 4) if k % 2 else (byte & 15)]
                if desc.w_scale == "e8m0":
                    W[n][k] = v * e8[int(scales[n][k // 32])]
                else:
                    W[n][k] = v * f8[int(scales[n][k // 16])] * gscale
    return W


@pytest.mark.parametrize("case", ["int4", "uint4", "mxfp4", "nvfp4"])
def test_bruteforce_tiny(case):
    M, N, K = 3, 5, 64
    ab, af = _a(M, K, seed=7)
    g = synth.generator(11)
    zeros = None
    gs = None
    if case in ("int4", "uint4"):
        grp = 32
        w = synth.int4_weights(1, N, K, grp, case == "uint4", g)
        d = O.Desc(case, grp, "bf16", w_zero=case == "uint4")
        codes = w["codes"][0].numpy()
        scales = synth.to_np_bits(w["scales"][0])
        zeros = None if w["zeros"] is None else w["zeros"][0].numpy()
    elif case == "mxfp4":
        w = synth.mxfp4_weights(1, N, K, g)
        d = O.Desc("e2m1", 32, "e8m0")
        codes, scales = w["codes"][0].numpy(), w["scales"][0].numpy()
    else:
        w = synth.nvfp4_weights_random(1, N, K, g)
        d = O.Desc("e2m1", 16, "ue4m3", w_global=True)
        codes, scales = w["codes"][0].numpy(), w["scales"][0].numpy()
        gs = float(w["global"][0])
    W, col = O.decode_weights(d, N, K, codes, scales, zeros, gs)
    out, _ = O.gemm(af, W)
    Wi = _indep_decode(d, N, K, codes, scales, zeros, gs)
    for m in range(M):
        for n in range(N):
            ref = math.fsum(af[m][k] * Wi[n][k] for k in range(K))
            assert abs(out[m, n] - ref) <= 1e-12 * (1 + abs(ref)), (m, n)


def test_moe_single_expert_top1_is_dense():
    T, N, K = 9, 16, 64
    ab, af = _a(T, K, seed=2)
    g = synth.generator(3)
    w = synth.mxfp4_weights(1, N, K, g)
    d = O.Desc("e2m1", 32, "e8m0")
    dec = lambda e: O.decode_weights(d, N, K, w["codes"][e].numpy(), w["scales"][e].numpy())
    ids = np.zeros((T, 1), dtype=np.int32)
    wts = np.ones((T, 1), dtype=np.float32)
    out, bound, _, _ = O.moe(af, ids, wts, dec)
    W, _ = dec(0)
    dense, dbound = O.gemm(af, W)
    assert np.array_equal(out, dense) and np.array_equal(bound, dbound)


def test_moe_relabel_invariance_and_manual_sum():
    T, E, k, N, K = 6, 5, 2, 8, 32
    ab, af = _a(T, K, seed=4)
    g = synth.generator(5)
    w = synth.mxfp4_weights(E, N, K, g)
    d = O.Desc("e2m1", 32, "e8m0")
    dec = lambda e: O.decode_weights(d, N, K, w["codes"][e].numpy(), w["scales"][e].numpy())
    ids, wts = synth.routing_softmax_topk(T, E, k, g)
    ids, wts = ids.numpy(), wts.numpy()
    A_slots = np.repeat(af, k, axis=0)
    out, _, Y, _ = O.moe(A_slots, ids, wts, dec, routed_scale=2.5)
    # manual: per token, per choice, decode that expert and dot
    for t in range(T):
        acc = np.zeros(N)
        for j in range(k):
            W, _ = dec(int(ids[t, j]))
            acc += float(wts[t, j]) * (W @ af[t])
        assert np.allclose(out[t], 2.5 * acc, rtol=1e-12, atol=1e-12)
    # relabel experts by a permutation; decoded weights follow the labels
    p = np.array([3, 0, 4, 1, 2])
    inv = np.argsort(p)
    dec2 = lambda e: dec(int(inv[e]))
    out2, _, _, _ = O.moe(A_slots, p[ids].astype(np.int32), wts, dec2, routed_scale=2.5)
    assert np.allclose(out, out2, rtol=1e-12, atol=1e-12)


def test_moe_permute_bruteforce():
    g = synth.generator(9)
    T, E, k = 50, 16, 4
    ids, _ = synth.routing_zipf(T, E, k, 1.2, g)
    ids = ids.numpy()
    off, perm, inv = O.moe_permute(ids, E)
    listing = []
    for e in range(E):
        for slot in range(T * k):
            if ids.reshape(-1)[slot] == e:
                listing.append(slot)
    assert perm.tolist() == listing
    assert off[-1] == T * k and off[0] == 0
    for e in range(E):
        assert off[e + 1] - off[e] == int((ids == e).sum())
    assert np.array_equal(perm[inv], np.arange(T * k))
    # each token's k experts are distinct
    assert all(len(set(r)) == k for r in ids.tolist())


@pytest.mark.parametrize("T", [64, 512, 4096])
def test_zipf_routing_spans_empty_to_more_than_an_eighth(T):
    # the config-4 input recipe: Zipf(1.2) popularity over 256 experts, top-8
    # distinct per token; per-expert counts must reach from 0 (T = 64) to more
    # than T / 8, so the MoE tests and bench see both empty and crowded experts
    g = synth.generator(900 + T)
    ids, wts = synth.routing_zipf(T, 256, 8, 1.2, g)
    counts = np.bincount(ids.numpy().reshape(-1), minlength=256)
    assert counts.sum() == T * 8
    assert counts.max() > T // 8
    if T <= 512:
        assert counts.min() == 0
    assert np.allclose(wts.sum(dim=-1).numpy(), 1.0, atol=1e-6)


def test_moe_masked_matches_routed_top1_and_ignores_invalid_rows():
    # a top-1 routing laid out as slabs (expert e's tokens in token order,
    # padded to the slab) gives the routed MoE's per-slot outputs exactly;
    # NaN in the padding rows reaches no valid row; counts past the slab clamp
    T, E, N, K, slab = 11, 4, 8, 64, 6
    ab, af = _a(T, K, seed=6)
    g = synth.generator(7)
    w = synth.mxfp4_weights(E, N, K, g)
    d = O.Desc("e2m1", 32, "e8m0")
    dec = lambda e: O.decode_weights(d, N, K, w["codes"][e].numpy(), w["scales"][e].numpy())
    ids = np.array([[2], [0], [2], [3], [2], [0], [2], [2], [0], [3], [2]], dtype=np.int32)
    Y_routed, B_routed = O.moe_expert_outputs(af, ids, dec)
    A_slab = np.full((E * slab, K), np.nan)
    counts = np.zeros(E, dtype=np.int64)
    where = {}
    for t in range(T):
        e = int(ids[t, 0])
        if counts[e] < slab:
            where[t] = e * slab + counts[e]
            A_slab[where[t]] = af[t]
        counts[e] += 1
    Y, B, valid = O.moe_masked(A_slab, counts, slab, dec)
    assert counts[2] == 6 and counts[0] == 3 and counts[1] == 0
    assert valid.sum() == sum(min(int(c), slab) for c in counts)
    for t, r in where.items():
        assert valid[r]
        assert np.array_equal(Y[r], Y_routed[t]) and np.array_equal(B[r], B_routed[t])
    assert np.isnan(Y[~valid]).all() and not np.isnan(Y[valid]).any()
    # a count above the slab takes the slab; a negative count none
    Y2, _, valid2 = O.moe_masked(A_slab, np.array([3, -4, 99, 2]), slab, dec)
    assert valid2.sum() == 3 + 0 + slab + 2


def test_silu_and_mul_closed_forms():
    g = np.array([0.0, 1.0, -1.0, 2.5, -2.5, 40.0, -40.0, -800.0])
    u = np.array([3.0, 1.0, 1.0, -2.0, 0.5, 1.0, 1.0, 2.0])
    out = O.silu_and_mul(np.concatenate([g, u])[None, :])[0]
    assert out[0] == 0.0
    assert out[1] == pytest.approx(0.7310585786300049, abs=1e-15)  # sigma(1) = 1 / (1 + 1/e)
    # silu(-x) = silu(x) - x (sigma(-x) = 1 - sigma(x)), times the up value
    assert out[2] == pytest.approx(0.7310585786300049 - 1.0, abs=1e-15)
    assert out[4] / 0.5 == pytest.approx(out[3] / -2.0 - 2.5, abs=1e-12)
    # large |g|: silu(g) -> g, silu(-g) -> 0 (no overflow trouble)
    assert out[5] == pytest.approx(40.0, rel=1e-15)
    assert abs(out[6]) < 1e-15 and out[7] == 0.0
