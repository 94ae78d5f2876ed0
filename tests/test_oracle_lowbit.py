"""Pins for the oracle's other WnA16 widths and the zero-exponent view.

* ``unpack_bits`` (the b-bit standard stream) against hand-packed bytes for
  b = 1, 2, 3, 6 and against the nibble / byte readers for b = 4, 8;
* the zero-exponent floats (float4e0m3, float8e0m7) against a generic
  minifloat decoder written here (exponent 0 = subnormal: (m / 2^M) *
  2^(1 - bias), with bias = 1 - M), which also reproduces the E2M1, E4M3,
  E2M3 and E3M2 tables, and against the pages' statement that float8e0m7
  and INT8 without -128 hold the same integers -127..127;
* the view itself: symmetric INT4 weights that avoid -8, converted to
  float4e0m3 codes, decode to the same weights;
* INT2 / INT3 / UINT2 / UINT3 and MXFP6 from the stream agree with the
  unpacked-code decoders.
"""
import numpy as np
import pytest

import oracle as O
import synth


def _pack_stream(codes, bits):
    """Hand packing (independent of the oracle): bit i of code k goes to bit
    b*k + i of the row, least significant first."""
    codes = np.asarray(codes, dtype=np.int64)
    N, K = codes.shape
    out = np.zeros((N, K * bits // 8), dtype=np.uint8)
    for n in range(N):
        for k in range(K):
            for i in range(bits):
                if (codes[n, k] >> i) & 1:
                    pos = bits * k + i
                    out[n, pos // 8] |= 1 << (pos % 8)
    return out


def test_unpack_bits_hand_examples():
    # 3-bit codes 0..7: 000 100 010 110 001 101 011 111 (LSB first) -> bytes
    assert O.unpack_bits(np.array([[0b10001000, 0b11000110, 0b11111010]], dtype=np.uint8), 3, 8).tolist() == \
        [[0, 1, 2, 3, 4, 5, 6, 7]]
    # 2-bit codes 3, 0, 1, 2 -> 0b10_01_00_11
    assert O.unpack_bits(np.array([[0b10010011]], dtype=np.uint8), 2, 4).tolist() == [[3, 0, 1, 2]]
    # 1-bit
    assert O.unpack_bits(np.array([[0b00000101]], dtype=np.uint8), 1, 8).tolist() == [[1, 0, 1, 0, 0, 0, 0, 0]]
    # 6-bit codes 63, 1, 32, 5 -> 24 bits (LSB first): 111111 100000 000001 101000
    assert O.unpack_bits(np.array([[0b01111111, 0b00000000, 0b00010110]], dtype=np.uint8), 6, 4).tolist() == \
        [[63, 1, 32, 5]]


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 6, 8])
def test_unpack_bits_random_round_trip(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(5, 64))
    assert np.array_equal(O.unpack_bits(_pack_stream(codes, bits), bits, 64), codes)
    if bits == 4:
        assert np.array_equal(O.unpack_nibbles_u8(_pack_stream(codes, 4), 64), codes)
    if bits == 8:
        assert np.array_equal(_pack_stream(codes, 8), codes.astype(np.uint8))


def _minifloat(code, e_bits, m_bits, bias):
    s = -1.0 if (code >> (e_bits + m_bits)) & 1 else 1.0
    e = (code >> m_bits) & ((1 << e_bits) - 1)
    m = code & ((1 << m_bits) - 1)
    if e == 0:
        return s * (m / 2.0 ** m_bits) * 2.0 ** (1 - bias)
    return s * (1.0 + m / 2.0 ** m_bits) * 2.0 ** (e - bias)


def test_zero_exponent_floats_are_symmetric_integers():
    assert [_minifloat(c, 0, 3, -2) for c in range(16)] == O.E0M3.tolist()
    assert [_minifloat(c, 0, 7, -6) for c in range(256)] == O.E0M7.tolist()
    # the same generic decoder gives the other tables (a pin of the decoder itself)
    assert [_minifloat(c, 2, 1, 1) for c in range(16)] == O.E2M1.tolist()
    assert [_minifloat(c, 2, 3, 1) for c in range(64)] == O.E2M3.tolist()
    assert [_minifloat(c, 3, 2, 3) for c in range(64)] == O.E3M2.tolist()
    e4 = [_minifloat(c, 4, 3, 7) for c in range(256)]
    fin = ~np.isnan(O.E4M3)
    assert np.array_equal(np.array(e4)[fin], O.E4M3[fin])
    # float8e0m7 and INT8 without -128 hold the same integers
    assert sorted(set(O.E0M7.tolist())) == list(range(-127, 128))
    assert sorted(set(O.E0M3.tolist())) == list(range(-7, 8))
    assert O.E0M3[8] == 0.0 and np.signbit(O.E0M3[8])  # the -0 code


@pytest.mark.parametrize("bits", [4, 8])
def test_int_to_e0m_round_trip(bits):
    lim = (1 << (bits - 1)) - 1
    q = np.arange(-lim, lim + 1)
    c = O.int_to_e0m(q, bits)
    table = O.E0M3 if bits == 4 else O.E0M7
    assert np.array_equal(table[c], q.astype(np.float64))
    assert c[lim] == 0  # +0
    with pytest.raises(ValueError):
        O.int_to_e0m([-(lim + 1)], bits)


def test_symmetric_int4_view_as_e0m3_keeps_the_weights():
    # symmetric INT4 weights that avoid -8, converted code by code to
    # float4e0m3, decode to the same weights with the same scales
    N, K, G = 6, 128, 32
    rng = np.random.default_rng(3)
    q = rng.integers(-7, 8, size=(N, K))
    nib = np.where(q < 0, q + 16, q)
    codes_i32 = synth.pack_nibbles_i32(nib)
    scales = synth.to_np_bits(synth.bf16_normal((N, K // G), synth.generator(4)).abs())
    W_int, _ = O.decode_weights(O.Desc("int4", G, "bf16"), N, K, codes_i32, scales)
    e0 = _pack_stream(O.int_to_e0m(q, 4), 4)
    W_e0 = O.decode_lowbit_weights("e0m3", e0, scales, K, G)
    assert np.array_equal(W_int, W_e0)


@pytest.mark.parametrize("kind,bits", [("int1", 1), ("int2", 2), ("int3", 3), ("uint1", 1), ("uint2", 2),
                                       ("uint3", 3)])
def test_lowbit_integers_from_the_stream(kind, bits):
    N, K, G = 4, 128, 64
    rng = np.random.default_rng(bits)
    u = rng.integers(0, 1 << bits, size=(N, K))
    scales = synth.to_np_bits(synth.bf16_normal((N, K // G), synth.generator(bits)).abs())
    zeros = rng.integers(0, 1 << bits, size=(N, K // G)).astype(np.uint8) if kind.startswith("u") else None
    W = O.decode_lowbit_weights(kind, _pack_stream(u, bits), scales, K, G, zeros)
    s = O.bf16_to_f64(scales)
    for n in range(N):
        for k in (0, 1, 63, 64, 127):
            if zeros is None:
                q = u[n, k] - (1 << bits) if u[n, k] >= (1 << (bits - 1)) else u[n, k]
            else:
                q = u[n, k] - int(zeros[n, k // G])
            assert W[n, k] == q * s[n, k // G]


@pytest.mark.parametrize("kind", ["e2m3", "e3m2"])
def test_mxfp6_from_the_stream(kind):
    N, K = 3, 64
    rng = np.random.default_rng(9)
    c = rng.integers(0, 64, size=(N, K))
    sc = np.array([[127, 130], [120, 127], [133, 126]], dtype=np.uint8)
    W = O.decode_lowbit_weights(kind, _pack_stream(c, 6), sc, K)
    table = O.E2M3 if kind == "e2m3" else O.E3M2
    for n in range(N):
        for k in range(K):
            assert W[n, k] == table[c[n, k]] * 2.0 ** (int(sc[n, k // 32]) - 127)
