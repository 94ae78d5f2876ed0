"""GPU parity: weight repack identity and bit-exact activation quantisation."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import PAIR_ONLY, WFORMATS, cdesc, gpu_pack, gpu_quant, make_weights, np_bits, oracle_quant

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wname", [w for w in WFORMATS if w not in PAIR_ONLY])
def test_pack_unpack_identity(wname):
    import quantized_gemm_02_b200 as hq
    E, N, K = 2, 80, 384  # ragged N (pads to 128 rows), 6 k-blocks
    w = make_weights(wname, E, N, K, seed=3)
    packed = gpu_pack(wname, w, E, N, K)
    out = {k: (None if v is None else torch.empty_like(v, device="cuda")) for k, v in w.items()}
    if out["zeros"] is not None:
        out["zeros"].zero_()
    hq.hq_unpack_weights(cdesc(wname), E, N, K, packed, out["codes"], out["scales"], out["zeros"], out["global"])
    torch.cuda.synchronize()
    for k, v in w.items():
        if v is None:
            continue
        want = np_bits(v)
        if wname.startswith("e0m3") and k == "codes":
            # float4e0m3 is stored as the symmetric integer it is: -0 comes back as +0
            want = want.copy()
            want[(want & 0x0F) == 0x08] &= 0xF0
            want[(want & 0xF0) == 0x80] &= 0x0F
        assert np.array_equal(np_bits(out[k]), want), k


@pytest.mark.parametrize("wname,aname", [("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("fp8", "fp8"), ("fp8b", "fp8g")])
def test_pack_unpack_identity_block_scaled(wname, aname):
    # block-scaled layouts (chosen by the activation format): codes row-major,
    # scales in 512-byte chunks; FP8 x FP8: E4M3 bytes row-major, row scales
    import quantized_gemm_02_b200 as hq
    E, N, K = 2, 80, 512
    w = make_weights(wname, E, N, K, seed=5)
    packed = gpu_pack(wname, w, E, N, K, aname)
    out = {k: (None if v is None else torch.empty_like(v, device="cuda")) for k, v in w.items()}
    hq.hq_unpack_weights(cdesc(wname, aname), E, N, K, packed, out["codes"], out["scales"], out["zeros"],
                         out["global"])
    torch.cuda.synchronize()
    for k, v in w.items():
        if v is None:
            continue
        assert np.array_equal(np_bits(out[k]), np_bits(v)), k
    # the codes of each row sit in stage chunks (MXFP4: 64 bytes, else 128),
    # [chunk][128 rows][chunk bytes] per 128-row tile (4-bit: two per byte,
    # even k low), padded rows zero
    d = cdesc(wname, aname)
    per_e = hq.hq_packed_weights_bytes(d, 1, N, K)
    p0 = packed[:per_e].cpu().numpy()
    codes = w["codes"][0].numpy() if hasattr(w["codes"], "numpy") else w["codes"][0].cpu().numpy()
    rb = K if wname in ("fp8", "fp8b") else K // 2
    cb = 64 if wname == "mxfp4" else 128
    rows = p0[: 128 * rb].reshape(rb // cb, 128, cb).transpose(1, 0, 2).reshape(128, rb)
    assert np.array_equal(rows[:N], codes.reshape(N, rb))
    assert not rows[N:].any()


def test_pack_is_deterministic_and_pads_with_zero():
    E, N, K = 1, 70, 128
    w = make_weights("int4_g128", E, N, K, seed=4)
    p1 = gpu_pack("int4_g128", w, E, N, K)
    p2 = gpu_pack("int4_g128", w, E, N, K)
    assert torch.equal(p1, p2)


def _acts(M, K, seed):
    g = synth.generator(seed)
    x = synth.bf16_normal((M, K), g)
    x[1] = 0                       # all-zero row / blocks
    x[2, :64] = 0
    x[3, 5] = 3.0e4                # one large value
    x[4, :] = x[4, :] * 1e-30      # tiny row (subnormal scales in fp32)
    return x


@pytest.mark.parametrize("aname", ["fp8", "mxfp8", "nvfp4", "fp8g"])
@pytest.mark.parametrize("shape", [(37, 512), (5, 7168)])
def test_quant_act_bit_exact(aname, shape):
    M, K = shape
    x = _acts(M, K, seed=M + K)
    codes, scales, g = gpu_quant(aname, x.cuda())
    torch.cuda.synchronize()
    q, s, og = oracle_quant(aname, np_bits(x))
    assert np.array_equal(codes.cpu().numpy(), q)
    if aname in ("fp8", "fp8g"):
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), s.view(np.uint32))
    else:
        assert np.array_equal(scales.cpu().numpy(), s)
    if aname == "nvfp4":
        assert np.float32(g.cpu().numpy()[0]) == og


def test_quant_nvfp4_static_global():
    x = _acts(9, 256, seed=5)
    sg = torch.tensor([0.0125], dtype=torch.float32, device="cuda")
    codes, scales, g = gpu_quant("nvfp4", x.cuda(), static_global=sg)
    torch.cuda.synchronize()
    q, s, og = O.quant_nvfp4(np_bits(x), global_scale=np.float32(0.0125))
    assert np.array_equal(codes.cpu().numpy(), q) and np.array_equal(scales.cpu().numpy(), s)


def test_quant_signed_zero_and_ties():
    # values that round to zero keep their sign; exact E2M1 ties round to even
    K = 64
    row = np.zeros(K, dtype=np.float32)
    row[:8] = [-1e-6, 1e-6, 0.25, 0.75, 1.25, 2.5, 5.0, -7.0]
    row[8] = 6.0
    x = torch.tensor(row[None, :]).to(torch.bfloat16)
    for aname in ("fp8", "mxfp8", "nvfp4"):
        codes, scales, g = gpu_quant(aname, x.cuda())
        torch.cuda.synchronize()
        q, s, og = oracle_quant(aname, np_bits(x))
        assert np.array_equal(codes.cpu().numpy(), q), aname
