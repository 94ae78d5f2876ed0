"""Pins of the oracle functions for the rows that come next (no GPU path
yet): FP6 element values, MXFP6 / MXINT4 / INT1-3 weight decoding, and FP8
with block scales.  Each is checked against the published format values or
against an already pinned oracle function, never against a retyped copy of
its own formula."""
import numpy as np
import pytest

import oracle as O
import synth
from conftest import read_golden


def test_fp6_landmarks_and_symmetry():
    for kind, code, value in read_golden("fp6_landmarks.txt"):
        assert O.fp6_value(int(code), kind) == float(value), (kind, code)
    for table in (O.E2M3, O.E3M2):
        pos = table[:32]
        assert np.all(np.diff(pos) > 0)              # magnitudes increase with the code
        assert np.array_equal(table[32:], -pos)      # the sign bit mirrors
        assert np.signbit(table[32]) and table[32] == 0.0
    # every value is a multiple of the smallest subnormal (no rounding in the table)
    assert np.all(np.mod(O.E2M3[:32] / 0.125, 1) == 0)
    assert np.all(np.mod(O.E3M2[:32] / 0.0625, 1) == 0)


def test_mxfp6_weights_scale_and_layout():
    N, K = 3, 64
    g = np.random.default_rng(1)
    codes = g.integers(0, 64, size=(N, K))
    sc = np.array([[127, 128], [120, 127], [130, 125]], dtype=np.uint8)
    for kind, table in (("e2m3", O.E2M3), ("e3m2", O.E3M2)):
        W = O.decode_fp6_weights(kind, codes, sc)
        for n in range(N):
            for k in (0, 31, 32, 63):
                assert W[n, k] == table[codes[n, k]] * 2.0 ** (int(sc[n, k // 32]) - 127)


def test_mxint4_is_mxfp4_layout_with_int4_elements():
    # one-hot rows decoded by hand: nibble 0x7 = 7, 0x8 = -8, 0xF = -1
    K = 64
    codes = np.zeros((3, K // 2), dtype=np.uint8)
    codes[0, 0] = 0x07          # k = 0 -> 7
    codes[1, 0] = 0x80          # k = 1 -> -8
    codes[2, 16] = 0xF0         # k = 33 -> -1
    sc = np.array([[127, 127], [128, 127], [127, 125]], dtype=np.uint8)
    W = O.decode_mxint4_weights(codes, sc, K)
    assert W[0, 0] == 7.0 and W[1, 1] == -16.0 and W[2, 33] == -0.25
    assert np.count_nonzero(W) == 3
    # same nibble order and scale blocks as MXFP4: swap the element table
    g = synth.generator(3)
    w = synth.mxfp4_weights(1, 4, K, g)
    c, s = w["codes"][0].numpy(), w["scales"][0].numpy()
    Wi = O.decode_mxint4_weights(c, s, K)
    Wf, _ = O.decode_weights(O.Desc("e2m1", 32, "e8m0"), 4, K, c, s)
    q = O.unpack_nibbles_u8(c, K)
    ints = np.where(q >= 8, q.astype(np.int64) - 16, q).astype(np.float64)
    ratio = np.divide(Wi, ints, out=np.zeros_like(Wi), where=ints != 0)
    ratio_f = np.divide(Wf, O.E2M1[q], out=np.zeros_like(Wf), where=O.E2M1[q] != 0)
    both = (ints != 0) & (O.E2M1[q] != 0)
    assert np.array_equal(ratio[both], ratio_f[both])   # the same per-block power of two


def test_int_weights_reduce_to_the_int4_path():
    # b = 4 signed is the INT4 decoder (two's complement); with zero points
    # it is the UINT4 decoder
    N, K, G = 4, 128, 64
    g = synth.generator(5)
    w = synth.int4_weights(1, N, K, G, True, g)
    codes_i32, scales, zeros_i32 = w["codes"][0].numpy(), synth.to_np_bits(w["scales"][0]), w["zeros"][0].numpy()
    u = O.unpack_nibbles_i32(codes_i32, K)
    z = O.unpack_nibbles_i32(zeros_i32, K // G)
    W_asym = O.decode_int_weights(4, u, scales, G, zeros=z)
    ref, _ = O.decode_weights(O.Desc("uint4", G, "bf16", w_zero=True), N, K, codes_i32, scales, zeros_i32)
    assert np.array_equal(W_asym, ref)
    W_sym = O.decode_int_weights(4, u, scales, G)
    ref2, _ = O.decode_weights(O.Desc("int4", G, "bf16"), N, K, codes_i32, scales)
    assert np.array_equal(W_sym, ref2)


def test_int1_int2_int3_hand_values():
    s = synth.to_np_bits(synth.bf16_normal((1, 1), synth.generator(0)).abs() + 1)  # one scale, per channel
    sv = O.bf16_to_f64(s)[0, 0]
    # signed codes are b-bit two's complement (the INT4 rule)
    for bits, codes, expect in ((1, [0, 1], [0, -1]), (2, [0, 1, 2, 3], [0, 1, -2, -1]),
                                (3, [0, 3, 4, 7], [0, 3, -4, -1])):
        W = O.decode_int_weights(bits, np.array([codes]), s, 0)
        assert np.array_equal(W[0], np.array(expect, dtype=np.float64) * sv), bits
    with pytest.raises(ValueError):
        O.decode_int_weights(2, np.array([[4]]), s, 0)


def test_fp8_block_scales_reduce_to_per_channel_and_per_token():
    # weights: one scale per 128 x 128 block, all blocks of a row-block equal
    # -> the per-channel FP8 decode with that channel scale
    N, K = 256, 256
    w = synth.fp8_weights_random(1, N, K, synth.generator(8))
    codes = w["codes"][0].numpy()
    bs = np.array([[0.5, 0.5], [0.25, 0.25]], dtype=np.float32)
    Wb = O.decode_fp8_block_weights(codes, bs)
    Wc, col = O.decode_weights(O.Desc("e4m3", 0, "fp32"), N, K, codes, np.repeat(bs[:, 0], 128))
    assert np.array_equal(Wb, Wc * col[:, None])
    # activations: the grouped recipe is the per-token recipe on each group
    x = synth.to_np_bits(synth.bf16_normal((5, 384), synth.generator(9)))
    x[2, 128:256] = 0  # an all-zero group
    q, s = O.quant_fp8_block(x)
    q2, s2 = O.quant_fp8_per_token(x.reshape(15, 128))
    assert np.array_equal(q, q2.reshape(5, 384)) and np.array_equal(s, s2.reshape(5, 3))
    assert s[2, 1] == 1.0
    A = O.decode_fp8_block_act(q, s)
    A2, row = O.decode_act("fp8", 15, 128, q2, s2)
    assert np.array_equal(A, (A2 * row[:, None]).reshape(5, 384))


def test_mxint4_through_decode_weights_equals_int4_with_power_of_two_scales():
    # the unified description routes INT4 + E8M0 per 32 to the MXINT4
    # decoder, reading the INT4 int32 words as their bytes; with bf16 group
    # scales equal to the same powers of two (bf16 bits = code << 7) the
    # plain INT4 g32 decoder gives the same weights
    N, K = 6, 128
    g = synth.generator(11)
    w = synth.mxint4_weights(1, N, K, g, exp_lo=-20, exp_hi=10)
    codes = w["codes"][0].numpy()
    sc = w["scales"][0].numpy()
    Wm, col = O.decode_weights(O.Desc("int4", 32, "e8m0"), N, K, codes, sc)
    assert col is None
    assert np.array_equal(Wm, O.decode_mxint4_weights(codes.view(np.uint8), sc, K))
    bf16_scales = (sc.astype(np.uint16) << 7).astype(np.uint16)
    Wi, _ = O.decode_weights(O.Desc("int4", 32, "bf16"), N, K, codes, bf16_scales)
    assert np.array_equal(Wm, Wi)


def test_fp8_block_weights_by_rows_and_through_decode_weights():
    # decoding chosen rows with their own block-scale rows (row_block = 1)
    # gives those rows of the whole-matrix decode; the unified description
    # (E4M3, group 128, fp32 scales) routes to the block decoder
    N, K = 300, 256
    g = synth.generator(12)
    w = synth.fp8_block_weights(1, N, K, g)
    c, s = w["codes"][0].numpy(), w["scales"][0].numpy()
    assert s.shape == (3, 2)
    full = O.decode_fp8_block_weights(c, s)
    rows = np.array([0, 127, 128, 299])
    part = O.decode_fp8_block_weights(c[rows], s[rows // 128], 128, row_block=1)
    assert np.array_equal(part, full[rows])
    Wd, col = O.decode_weights(O.Desc("e4m3", 128, "fp32"), N, K, c, s)
    assert col is None and np.array_equal(Wd, full)
    assert full[200, 130] == O.E4M3[c[200, 130]] * float(s[1, 1])
