"""Pins for the oracle's format decoders and rounding.

Each check compares the oracle with something other than itself: the
published format tables (``tests/golden``), torch's own float8 casts (an
independent library routine) and the IEEE rounding rule on hand-built ties.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from conftest import read_golden


def _same(a, b):
    return (math.isnan(a) and math.isnan(b)) or (a == b and math.copysign(1, a) == math.copysign(1, b))


def test_e2m1_table_matches_spec():
    rows = read_golden("e2m1_values.txt")
    assert len(rows) == 16
    for code, val in rows:
        assert _same(O.E2M1[int(code)], float(val)), code


def test_e4m3_all_codes_match_torch_cast():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        assert _same(O.E4M3[c], ref[c]), hex(c)


def test_e4m3_landmarks_match_spec():
    for code, val in read_golden("e4m3_landmarks.txt"):
        assert _same(O.E4M3[int(code, 16)], float(val)), code


def test_e8m0_all_codes_match_torch_cast():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    for c in range(256):
        assert _same(O.E8M0[c], ref[c]), c
    for code, val in read_golden("e8m0_landmarks.txt"):
        assert _same(O.E8M0[int(code)], float(val)), code


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(1)
    bits = torch.randint(0, 65536, (4096,), generator=g, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_to_f64(bits.numpy().view(np.uint16))
    ok = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert ok.all()


def test_rounding_ties_and_saturation():
    for fmt, x, want in read_golden("rounding_ties.txt"):
        x = np.float32(float(x))
        if fmt == "e2m1":
            got = O.E2M1[int(O.e2m1_rn_sat(np.array([x]))[0])]
        else:
            got = O.E4M3[int(O.e4m3_rn_sat(np.array([x]))[0])]
        assert _same(got, float(want)), (fmt, x, got, want)


def test_e4m3_rounding_matches_torch_in_range():
    g = torch.Generator().manual_seed(2)
    # magnitudes spanning the subnormal range up to just below 464 (where the
    # unsaturated torch cast starts to produce NaN)
    mant = torch.rand(200000, generator=g, dtype=torch.float32) + 1.0
    ex = torch.randint(-14, 9, (200000,), generator=g, dtype=torch.int32).to(torch.float32)
    sign = torch.where(torch.rand(200000, generator=g) < 0.5, -1.0, 1.0)
    x = sign * mant * torch.pow(2.0, ex)
    x = x[x.abs() < 464.0]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_rn_sat(x.numpy())
    assert np.array_equal(got, ref)


def test_e4m3_every_midpoint_rounds_to_even():
    vals = O.E4M3[:127]
    mids = (vals[:-1] + vals[1:]) / 2
    got = O.e4m3_rn_sat(mids.astype(np.float32))
    want = np.where(np.arange(126) % 2 == 0, np.arange(126), np.arange(1, 127))
    assert np.array_equal(got.astype(np.int64), want)


def test_decode_quant_idempotent_on_representable():
    finite = [c for c in range(256) if not math.isnan(O.E4M3[c])]
    x = O.E4M3[finite].astype(np.float32)
    assert np.array_equal(O.e4m3_rn_sat(x), np.array(finite, dtype=np.uint8))
    x2 = O.E2M1.astype(np.float32)
    assert np.array_equal(O.e2m1_rn_sat(x2), np.arange(16, dtype=np.uint8))


def test_nibble_unpack_order():
    # nibble j of a word holds element 8w + j; two's complement for INT4
    w = np.array([[0x76543210, np.uint32(0xFEDCBA98).view(np.int32)]], dtype=np.int32)
    n = O.unpack_nibbles_i32(w, 16)
    assert n.tolist() == [list(range(16))]
    b = np.array([[0x21, 0xF3]], dtype=np.uint8)
    assert O.unpack_nibbles_u8(b, 4).tolist() == [[1, 2, 3, 15]]
