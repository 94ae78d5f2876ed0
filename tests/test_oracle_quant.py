"""Pins for the oracle's activation quantisers.

The per-token FP8 and MXFP8 recipes are cross-checked against torch's own
fp32 arithmetic and float8 cast (independent library routines) where that
cast is defined (|v| < 464); saturation, zero blocks and the OCP MX shared
exponent rule are pinned with hand-built cases; NVFP4 is pinned through its
invariants (the tensor's largest block gets the largest scale, decode error
within half the local grid spacing, all-zero cases).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth


def _bits(t):
    return synth.to_np_bits(t.to(torch.bfloat16))


def test_fp8_per_token_matches_torch():
    g = synth.generator(3)
    x = synth.bf16_normal((37, 256), g)
    x[5] = 0  # all-zero row
    q, s = O.quant_fp8_per_token(_bits(x))
    xf = x.float()
    amax = xf.abs().amax(dim=1)
    s_ref = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    assert np.array_equal(s.view(np.uint32), s_ref.numpy().view(np.uint32))
    y = xf / s_ref[:, None]
    assert y.abs().max() < 464
    q_ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, q_ref)
    assert (q[5] == 0).all()
    # the row maximum always lands on +-448
    for m in range(37):
        if m == 5:
            continue
        assert np.max(O.E4M3[q[m]] * 0 + np.abs(O.E4M3[q[m]])) == 448.0


def test_mxfp8_shared_exponent_rule():
    # amax 1.0 -> floor(log2) = 0 -> e = -8 (code 119); amax 448 -> e = 0 (code 127);
    # amax 500 -> e = 0 and 500 saturates to 448; amax 2^-10 -> e = -18.
    rows = []
    for amax in (1.0, 448.0, 500.0, 2.0 ** -10, 3.0):
        r = np.zeros(32, dtype=np.float32)
        r[7] = amax
        r[8] = -amax / 4
        rows.append(r)
    x = torch.tensor(np.stack(rows)).to(torch.bfloat16)
    q, sc = O.quant_mxfp8(_bits(x))
    assert sc[:, 0].tolist() == [119, 127, 127, 127 - 18, 120]
    assert O.E4M3[q[0, 7]] == 256.0 and O.E4M3[q[0, 8]] == -64.0
    assert O.E4M3[q[1, 7]] == 448.0
    assert O.E4M3[q[2, 7]] == 448.0  # bf16(500) = 500 -> saturated
    assert O.E4M3[q[3, 7]] == 256.0
    assert O.E4M3[q[4, 7]] == 384.0  # 3 * 2^7


def test_mxfp8_matches_torch_where_cast_defined():
    g = synth.generator(4)
    x = synth.bf16_normal((64, 512), g)
    x[3, 32:64] = 0  # zero block
    q, sc = O.quant_mxfp8(_bits(x))
    xf = x.float().reshape(64, 16, 32)
    amax = xf.abs().amax(dim=2)
    _, ex = torch.frexp(torch.where(amax > 0, amax, torch.ones_like(amax)))
    e = torch.where(amax > 0, ex - 1 - 8, torch.zeros_like(ex)).clamp(-127, 127)
    assert np.array_equal(sc.astype(np.int64), (e + 127).numpy())
    y = torch.ldexp(xf, (-e)[..., None].to(torch.float32))
    ok = y.abs() < 464
    q_ref = torch.where(ok, y, torch.zeros_like(y)).to(torch.float8_e4m3fn).view(torch.uint8)
    qr = q.reshape(64, 16, 32)
    assert np.array_equal(qr[ok.numpy()], q_ref.numpy()[ok.numpy()])
    # outside the torch-cast range the oracle saturates
    assert np.all(np.isin(qr[~ok.numpy()], [0x7E, 0xFE]))
    assert (sc[3, 1] == 127) and (q[3, 32:64] == 0).all()


def _nvfp4_decode(packed, sb, gsc, M, K):
    A, _ = O.decode_act("nvfp4", M, K, packed, sb, gsc)
    return A


def test_nvfp4_invariants():
    g = synth.generator(5)
    M, K = 24, 256
    x = synth.bf16_normal((M, K), g)
    x[2, 16:32] = 0
    xb = _bits(x)
    packed, sb, gsc = O.quant_nvfp4(xb)
    xf = x.float().numpy().astype(np.float64)
    amax = np.abs(xf).max()
    assert gsc == np.float32(np.float32(amax) / np.float32(2688.0))
    # the block holding the tensor maximum gets scale code 448 (0x7E)
    r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    assert sb[r, c // 16] == 0x7E
    assert sb[2, 1] == 0
    assert np.all(sb < 0x80)  # scales are unsigned
    dec = _nvfp4_decode(packed, sb, gsc, M, K)
    d = O.E4M3[sb].astype(np.float32).astype(np.float64) * float(gsc)
    dd = np.repeat(d, 16, axis=1)
    # the E2M1 grid spacing is at most 2 (between 4 and 6); scaled values never
    # exceed 6 by more than the scale's own rounding (2^-4 relative)
    err = np.abs(dec - xf)
    assert np.all(err <= 1.0 * dd + 1e-30)
    assert np.all(np.abs(xf) <= 6.0 * dd * (1 + 2 ** -4) + 1e-30)
    assert np.all(dec[2, 16:32] == 0)


def test_nvfp4_exact_on_representable_blocks():
    # a block whose values are E2M1 grid points times a UE4M3-representable
    # scale (with g = 1) decodes back exactly
    vals = O.E2M1[[1, 2, 3, 4, 5, 6, 7, 7, 9, 10, 11, 12, 13, 14, 15, 0]]
    x = torch.tensor(np.tile(vals * 0.5, (4, 1)), dtype=torch.float32).to(torch.bfloat16)
    packed, sb, gsc = O.quant_nvfp4(_bits(x), global_scale=1.0)
    assert gsc == 1.0
    assert np.all(O.E4M3[sb] == 0.5)
    dec = _nvfp4_decode(packed, sb, gsc, 4, 16)
    assert np.array_equal(dec, x.float().numpy().astype(np.float64))


def test_zero_tensors():
    z = np.zeros((2, 64), dtype=np.uint16)
    q, s = O.quant_fp8_per_token(z)
    assert (q == 0).all() and (s == 1.0).all()
    q, sc = O.quant_mxfp8(z)
    assert (q == 0).all() and (sc == 127).all()
    p, sb, gsc = O.quant_nvfp4(z)
    assert (p == 0).all() and (sb == 0).all() and gsc == 1.0
