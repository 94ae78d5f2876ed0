"""Pins for the oracle paths that quantised activations take.

* ``decode_act`` for per-token FP8 and MXFP8: hand-built codes and scales
  whose decoded values are worked out by hand here (E4M3 "fn" and E8M0 from
  the OCP 8-bit floating point and OCP Microscaling v1.0 definitions), with
  two 32-element blocks of different E8M0 codes so that a wrong block index
  (k // 16 for k // 32) or a dropped scale factor fails.
* ``gemm`` with a per-row (per-token) scale: constant weights c give the
  closed form out[m, n] = s_m * c * sum_k a[m, k].
* ``quant_nvfp4``'s UE4M3 block-scale step: bit-exact against torch's
  fp32 -> float8_e4m3fn cast (an independent library routine) of
  fp32(fp32(amax / 6) / g), and two hand-built blocks whose scale lands
  exactly on a midpoint between neighbouring UE4M3 values (round to nearest
  even goes down on one, up on the other).
"""
import math

import numpy as np
import torch

import oracle as O
import synth


def _bits(t):
    return synth.to_np_bits(t.to(torch.bfloat16))


def test_decode_act_fp8_hand_values():
    # E4M3: 0x38 = 1.0 (exponent 7 = bias), 0x40 = 2.0, 0x3C = 1.5,
    # 0xB8 = -1.0, 0x7E = 448 (1.75 * 2^8), 0x01 = 2^-9 (subnormal 1/8 * 2^-6),
    # 0x08 = 2^-6 (smallest normal), 0x00 = 0
    codes = np.array([[0x38, 0x40, 0x3C, 0xB8, 0x7E, 0x01, 0x08, 0x00],
                      [0x40, 0x40, 0x40, 0x40, 0xC4, 0x39, 0x30, 0x80]], dtype=np.uint8)
    want = np.array([[1.0, 2.0, 1.5, -1.0, 448.0, 2.0 ** -9, 2.0 ** -6, 0.0],
                     [2.0, 2.0, 2.0, 2.0, -3.0, 1.125, 0.5, -0.0]])
    scales = np.array([0.25, 3.0], dtype=np.float32)
    A, row = O.decode_act("fp8", 2, 8, codes, scales)
    assert np.array_equal(A, want)
    # the per-token scale is returned apart (it multiplies the output row)
    assert row.tolist() == [0.25, 3.0]


def test_decode_act_mxfp8_block_index_and_scale():
    # K = 64: two MX blocks of 32.  Row 0: block 0 code 127 (2^0), block 1
    # code 130 (2^3).  Row 1: block 0 code 120 (2^-7), block 1 code 127.
    M, K = 2, 64
    codes = np.zeros((M, K), dtype=np.uint8)
    codes[:, :] = 0x38  # 1.0 everywhere
    codes[0, 20] = 0x44  # 3.0 at k = 20 (block 0, but k // 16 = 1)
    codes[0, 40] = 0xC0  # -2.0 at k = 40 (block 1)
    codes[1, 31] = 0x30  # 0.5 at the last k of block 0
    codes[1, 32] = 0x7E  # 448 at the first k of block 1
    scales = np.array([[127, 130], [120, 127]], dtype=np.uint8)
    A, row = O.decode_act("mxfp8", M, K, codes, scales)
    assert row is None
    want = np.ones((M, K))
    want[0, :32] *= 1.0
    want[0, 32:] *= 8.0
    want[1, :32] *= 2.0 ** -7
    want[0, 20] = 3.0
    want[0, 40] = -2.0 * 8.0
    want[1, 31] = 0.5 * 2.0 ** -7
    want[1, 32] = 448.0
    assert np.array_equal(A, want)


def test_gemm_row_scale_closed_form():
    # every weight decodes to c = 0.75 (NVFP4 code 0x5 = 3.0 times UE4M3 1.0
    # times global 0.25); per-row scales s_m of either sign
    M, N, K = 6, 5, 128
    g = synth.generator(17)
    x = synth.bf16_normal((M, K), g)
    af = x.to(torch.float64).numpy()
    W, col = O.decode_weights(O.Desc("e2m1", 16, "ue4m3", w_global=True), N, K,
                              np.full((N, K // 2), 0x55, dtype=np.uint8), np.full((N, K // 16), 0x38, dtype=np.uint8),
                              global_scale=0.25)
    assert col is None and np.all(W == 0.75)
    s = np.array([0.5, -2.0, 1e-3, 3.0, 1.0, 0.125])
    out, bound = O.gemm(af, W, s, None)
    for m in range(M):
        want = s[m] * 0.75 * math.fsum(af[m])
        assert np.allclose(out[m], want, rtol=1e-12, atol=1e-14)
        assert np.allclose(bound[m], abs(s[m]) * 0.75 * math.fsum(np.abs(af[m])), rtol=1e-12)
    # row and column scales together: s_m * c * t_n * sum_k a[m, k]
    t = np.array([1.0, -0.5, 2.0, 4.0, 0.25])
    out2, _ = O.gemm(af, W, s, t)
    for m in range(M):
        for n in range(N):
            assert math.isclose(out2[m, n], s[m] * 0.75 * t[n] * math.fsum(af[m]), rel_tol=1e-12, abs_tol=1e-14)


def test_nvfp4_scale_codes_match_torch_cast():
    g = synth.generator(23)
    M, K = 40, 512
    x = synth.bf16_normal((M, K), g) * 3
    x[1, 32:48] = 0
    x[2] = x[2] * 1e-3
    for static in (None, 0.01, 1.0):
        packed, sb, gsc = O.quant_nvfp4(_bits(x), global_scale=static)
        xf = x.float()
        amax_t = xf.abs().max()
        gt = (amax_t / 2688.0) if static is None else torch.tensor(static, dtype=torch.float32)
        assert np.float32(gt.item()) == gsc
        amax_b = xf.reshape(M, K // 16, 16).abs().amax(dim=2)
        sbv = (amax_b / 6.0) / gt  # fp32 ops in the recipe's order
        assert sbv.max() < 464  # inside torch's cast range
        ref = sbv.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(sb, ref), static


def test_nvfp4_scale_midpoints_round_to_even():
    # g = 1.  Block 0: amax 6.375 -> 6.375 / 6 = 1.0625, the midpoint of
    # UE4M3 1.0 (0x38) and 1.125 (0x39): ties to even -> 0x38 (rounding up
    # would give 0x39).  Block 1: amax 7.125 -> 1.1875, the midpoint of
    # 1.125 (0x39) and 1.25 (0x3A): ties to even -> 0x3A (truncation would
    # give 0x39).  Block 2: amax 1.59375 * 6 = 9.5625 -> 1.59375, above the
    # midpoint 1.5625 of 1.5 / 1.625 -> 0x3D.
    K = 48
    x = np.zeros((1, K), dtype=np.float32)
    x[0, 3] = 6.375
    x[0, 16 + 7] = -7.125
    x[0, 32 + 0] = 9.5625
    xb = torch.tensor(x).to(torch.bfloat16)
    assert xb.float().numpy().tolist() == x.tolist()  # all three are bf16 values
    packed, sb, gsc = O.quant_nvfp4(_bits(xb), global_scale=1.0)
    assert sb[0].tolist() == [0x38, 0x3A, 0x3D]
    # and the element step uses the rounded scale: 6.375 / 1.0 -> E2M1 6 (code 7)
    q = O.unpack_nibbles_u8(packed, K)
    assert q[0, 3] == 7
    assert O.E2M1[q[0, 16 + 7]] == -6.0  # -7.125 / 1.25 = -5.7 -> -6
