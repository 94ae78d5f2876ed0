"""GPU parity of the dense GEMM against the fp64 oracle.

Tolerance (stated by the method's target): |gpu - oracle| <= 4e-3 * sum_k
|a_k w_k| (times |scales|) + 1e-5 per element.  Quantised activations are
first checked bit-exact, then each side multiplies its own quantised copy.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import (PAIR_ONLY, WFORMATS, assert_close, cdesc, gpu_pack, gpu_quant, make_weights, np_bits, odesc,
                    oracle_decoder, oracle_quant)

pytestmark = pytest.mark.gpu


def run_gemm(wname, aname, packed, M, N, K, a_gpu, a_scales=None, a_global=None):
    import quantized_gemm_02_b200 as hq
    d = cdesc(wname, aname)
    ws_bytes = hq.hq_gemm_workspace_bytes(d, M, N, K)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    hq.hq_gemm(d, M, N, K, packed, a_gpu, a_scales, a_global, c, ws, ws_bytes)
    return c


def parity(wname, aname, M, N, K, seed=0, cols=None, rows=None):
    """Runs one GEMM on the GPU and checks it against the oracle (optionally on
    sampled output columns / rows).  Returns the max err/bound ratio."""
    w = make_weights(wname, 1, N, K, seed=seed)
    packed = gpu_pack(wname, w, 1, N, K, aname)
    x = synth.bf16_normal((M, K), synth.generator(seed + 1))
    xb = np_bits(x)
    if aname == "bf16":
        c = run_gemm(wname, aname, packed, M, N, K, x.cuda())
        A, row = O.decode_act("bf16", M, K, xb)
    else:
        codes, scales, g = gpu_quant(aname, x.cuda())
        q, s, og = oracle_quant(aname, xb)
        assert np.array_equal(codes.cpu().numpy(), q)
        c = run_gemm(wname, aname, packed, M, N, K, codes, scales, g if aname == "nvfp4" else None)
        A, row = O.decode_act(aname, M, K, q, s, og)
    torch.cuda.synchronize()
    dec = oracle_decoder(wname, w, N, K)
    cols = np.arange(N) if cols is None else np.asarray(cols)
    rows = np.arange(M) if rows is None else np.asarray(rows)
    W, col = dec(0, cols)
    ref, bound = O.gemm(A[rows], W, None if row is None else row[rows], col)
    got = c.cpu()[torch.as_tensor(rows)][:, torch.as_tensor(cols)]
    return assert_close(got, ref, bound, what=f"{wname}x{aname} M={M} N={N} K={K}")


@pytest.mark.parametrize("wname", [w for w in WFORMATS if w not in PAIR_ONLY])
@pytest.mark.parametrize("M", [1, 7, 16, 33])
def test_gemm_bf16_acts_small(wname, M):
    parity(wname, "bf16", M, 200, 512, seed=M)


@pytest.mark.parametrize("wname,aname", [
    ("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("fp8", "fp8"), ("int4_g128", "fp8"),
    ("uint4_g128", "mxfp8"), ("mxfp4", "nvfp4"), ("fp8", "mxfp8"), ("nvfp4", "fp8"), ("mxint4", "mxfp8"),
    ("int3_g128", "fp8"), ("e2m3", "mxfp8"), ("uint2_g32", "nvfp4"), ("e0m3_g128", "fp8"),
])
@pytest.mark.parametrize("M", [1, 16, 40])
def test_gemm_quantised_acts_small(wname, aname, M):
    parity(wname, aname, M, 136, 256, seed=10 + M)


@pytest.mark.parametrize("M,N,K", [(1, 200, 512), (16, 200, 512), (40, 136, 1024), (300, 200, 512),
                                   (129, 2048, 384), (5, 512, 8192)])
def test_gemm_fp8_block_scaled(M, N, K):
    # FP8 weights with 128 x 128 block scales x FP8 activations with per-(token,
    # 128 k) scales: per-stage accumulators promoted with both scales in fp32;
    # whole tiles, Stream-K pieces and the fixup (5 x 512 x 8192: many pieces)
    parity("fp8b", "fp8g", M, N, K, seed=80 + M)


def test_gemm_large_token_count():
    # many token tiles of the streaming kernel, ragged last tile
    parity("uint4_g128", "bf16", 300, 96, 384, seed=5)


def test_gemm_many_token_tiles():
    # 2100 tokens: eleven 256-token tiles (ragged last), grouped raster of token tiles
    parity("uint4_g128", "bf16", 2100, 136, 256, seed=6)
    parity("fp8", "fp8", 2100, 136, 256, seed=7)


@pytest.mark.parametrize("wname,aname", [("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("fp8", "fp8")])
@pytest.mark.parametrize("M", [129, 300])
def test_gemm_block_scaled_many_token_tiles(wname, aname, M):
    # more than 128 tokens: several 128-token tiles of the block-scaled
    # kernel (scale chunks of each token slot), ragged last tile; FP8 x FP8
    # runs 256-token tiles (no scale columns in tensor memory)
    parity(wname, aname, M, 136, 512, seed=20 + M)


def test_gemm_fp8_fp8_256_token_tiles():
    # enough 256-token tiles (2 x 148 weight tiles) for the FP8 kernel to use
    # them: 300 tokens = one full and one ragged tile; sampled columns
    N = 148 * 128
    cols = np.sort(np.random.default_rng(3).choice(N, 256, replace=False))
    parity("fp8", "fp8", 300, N, 256, seed=44, cols=cols)


@pytest.mark.parametrize("M", [16, 300])
def test_gemm_fp8_fp8_k_not_multiple_of_128(M):
    # K = 192: the FP8 x FP8 pair keeps the tiled layout and the kernels that
    # stage the E4M3 weights through tensor memory
    parity("fp8", "fp8", M, 136, 192, seed=40 + M)


def test_config1_full():
    # Dense W4A16: M=16, N=K=4096, INT4 symmetric, bf16 scales per 128 group
    r = parity("int4_g128", "bf16", 16, 4096, 4096, seed=0)
    assert r < 4e-3


@pytest.mark.parametrize("NK", [(8192, 8192), (28672, 8192), (8192, 28672)])
@pytest.mark.parametrize("M", [1, 16, 64])
def test_config2_sampled(NK, M):
    N, K = NK
    cols = np.sort(np.random.default_rng(M).choice(N, 256, replace=False))
    parity("uint4_g128", "bf16", M, N, K, seed=2, cols=cols)


@pytest.mark.parametrize("aname", ["nvfp4", "fp8"])
def test_config5_quantised_weights(aname):
    # W4A4 NVFP4 x NVFP4 and W8A8 FP8: both operands N(0,1) quantised.  The
    # weights are quantised on the GPU (per output channel = per row of W) and
    # checked bit-exact against the oracle's quantiser before the GEMM.
    import quantized_gemm_02_b200 as hq
    M, N, K = 32, 7168, 7168
    gen = synth.generator(7)
    Wf = synth.bf16_normal((N, K), gen)
    x = synth.bf16_normal((M, K), gen)
    wc, ws, wg = gpu_quant(aname, Wf.cuda())
    q, s, og = oracle_quant(aname, np_bits(Wf))
    torch.cuda.synchronize()
    assert np.array_equal(wc.cpu().numpy(), q)
    wname = "nvfp4" if aname == "nvfp4" else "fp8"
    w = {"codes": wc[None], "scales": ws[None], "zeros": None, "global": (wg if aname == "nvfp4" else None)}
    packed = gpu_pack(wname, w, 1, N, K, aname)
    ac, asc, ag = gpu_quant(aname, x.cuda())
    c = run_gemm(wname, aname, packed, M, N, K, ac, asc, ag if aname == "nvfp4" else None)
    torch.cuda.synchronize()
    qa, sa, oga = oracle_quant(aname, np_bits(x))
    A, row = O.decode_act(aname, M, K, qa, sa, oga)
    cols = np.sort(np.random.default_rng(1).choice(N, 512, replace=False))
    d = odesc(wname)
    W, col = O.decode_weights(d, len(cols), K, q[cols], s[cols], None, og)
    ref, bound = O.gemm(A, W, row, col)
    assert_close(c.cpu()[:, torch.as_tensor(cols)], ref, bound, what=f"config5 {aname}")


def test_split_k_deterministic_and_workspace_reusable():
    import quantized_gemm_02_b200 as hq
    M, N, K = 4, 512, 8192  # few tiles -> many splits
    w = make_weights("mxfp4", 1, N, K, seed=9)
    packed = gpu_pack("mxfp4", w, 1, N, K)
    x = synth.bf16_normal((M, K), synth.generator(10)).cuda()
    d = cdesc("mxfp4")
    wsb = hq.hq_gemm_workspace_bytes(d, M, N, K)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        hq.hq_gemm(d, M, N, K, packed, x, None, None, c, ws, wsb)
        outs.append(c)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    assert hq.hq_device_error() == 0


@pytest.mark.parametrize("wname,aname", [("uint4_g128", "bf16"), ("mxfp4", "bf16"), ("mxfp4", "mxfp8"),
                                         ("nvfp4", "nvfp4"), ("fp8", "fp8"), ("int4_g128", "fp8")])
def test_batch_invariant_rows_do_not_depend_on_m(wname, aname):
    # compute option batch_invariant: the first m rows of a 300-row call are
    # bit-identical to a call with only those m rows (same codes and scales);
    # the 300-row result also matches the oracle
    import quantized_gemm_02_b200 as hq
    N, K, Mmax = 136, 512, 300
    w = make_weights(wname, 1, N, K, seed=71)
    packed = gpu_pack(wname, w, 1, N, K, aname)
    x = synth.bf16_normal((Mmax, K), synth.generator(72))
    d = cdesc(wname, aname)
    cfg = hq.ComputeConfig()
    cfg.batch_invariant = 1
    if aname == "bf16":
        codes, scales, g = x.cuda(), None, None
    else:
        codes, scales, g = gpu_quant(aname, x.cuda())
        if aname != "nvfp4":
            g = None
    outs = {}
    for M in (Mmax, 1, 5, 64, 65, 200):
        wsb = hq.hq_gemm_config_workspace_bytes(d, cfg, M, N, K)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
        c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        hq.hq_gemm_config(d, cfg, M, N, K, packed, codes[:M].contiguous(),
                          None if scales is None else scales[:M].contiguous(), g, c, ws, wsb)
        outs[M] = c
    torch.cuda.synchronize()
    for M, c in outs.items():
        assert torch.equal(c, outs[Mmax][:M]), M
    xb = np_bits(x)
    if aname == "bf16":
        A, row = O.decode_act("bf16", Mmax, K, xb)
    else:
        q, s, og = oracle_quant(aname, xb)
        A, row = O.decode_act(aname, Mmax, K, q, s, og)
    W, col = oracle_decoder(wname, w, N, K)(0)
    ref, bound = O.gemm(A, W, row, col)
    assert_close(outs[Mmax].cpu(), ref, bound, what=f"batch-invariant {wname}x{aname}")
