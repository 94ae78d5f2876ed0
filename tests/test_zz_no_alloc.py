"""hq_gemm_noalloc: the dense GEMM for callers that cannot allocate device
memory (under an allocator that owns all device memory, as a plugin given no
allocator, or on a code path that must not allocate).  It must compute what
hq_gemm computes, using the library's fixed device scratch array instead of
a caller workspace: each call is compared with hq_gemm and with the oracle.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  It also passes when run alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import cdesc, gpu_pack, gpu_quant, make_weights, np_bits, oracle_decoder, oracle_quant

pytestmark = pytest.mark.gpu

REL, ABS = 4e-3, 1e-5  # the parity tolerance used by every GEMM test


def _reference_and_bound(wname, aname, w, x, M, N, K):
    xb = np_bits(x)
    if aname == "bf16":
        A, row = O.decode_act("bf16", M, K, xb)
    else:
        q, s, og = oracle_quant(aname, xb)
        A, row = O.decode_act(aname, M, K, q, s, og)
    W, col = oracle_decoder(wname, w, N, K)(0)
    return O.gemm(A, W, row, col)


@pytest.mark.parametrize("wname,aname,M,N,K", [
    ("mxfp4", "bf16", 4, 512, 8192),        # split-K: tile counters at the head of the scratch
    ("nvfp4", "nvfp4", 24, 320, 1024),      # block-scaled MMA, Stream-K tickets in the scratch
    ("nvfp4", "fp8", 24, 320, 1024),        # quantised activations: decoded copy in the scratch
    ("fp8", "fp8", 24, 320, 1024),          # FP8 MMA straight from TMA, per-token scales in the epilogue
    ("uint4_g128", "bf16", 40, 200, 2048),  # several token tiles
])
def test_noalloc_matches_hq_gemm_twice(wname, aname, M, N, K):
    import quantized_gemm_02_b200 as hq
    w = make_weights(wname, 1, N, K, seed=M + N)
    packed = gpu_pack(wname, w, 1, N, K, aname)
    x = synth.bf16_normal((M, K), synth.generator(M))
    d = cdesc(wname, aname)
    if aname == "bf16":
        a, a_s, a_g = x.cuda(), None, None
    else:
        a, a_s, a_g = gpu_quant(aname, x.cuda())
        if aname != "nvfp4":
            a_g = None
    wsb = hq.hq_gemm_workspace_bytes(d, M, N, K)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    ref_c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    hq.hq_gemm(d, M, N, K, packed, a, a_s, a_g, ref_c, ws, wsb)
    outs = []
    for _ in range(2):
        c = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        hq.hq_gemm_noalloc(d, M, N, K, packed, a, a_s, a_g, c)
        outs.append(c)
    torch.cuda.synchronize()
    assert hq.hq_device_error() == 0
    ref, bound = _reference_and_bound(wname, aname, w, x, M, N, K)
    tol = REL * bound + ABS
    r = ref_c.float().cpu().numpy()
    for c in outs:
        g = c.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g))
        assert np.all(np.abs(g - r) <= tol)    # against hq_gemm
        assert np.all(np.abs(g - ref) <= tol)  # against the oracle


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import quantized_gemm_02_b200 as hq
    # FP8 activations with NVFP4 weights need a decoded bf16 copy of A:
    # 4096 x 16384 x 2 B = 128 MiB > 64 MiB
    d = cdesc("nvfp4", "fp8")
    assert hq.hq_gemm_workspace_bytes(d, 4096, 256, 16384) > (64 << 20)
    with pytest.raises(hq.HQError) as e:
        hq.hq_gemm_noalloc(d, 4096, 256, 16384, 16, 16, 16, 16, 16)
    assert e.value.status == 3  # HQ_ERR_WORKSPACE
    # argument errors are reported as hq_gemm reports them
    with pytest.raises(hq.HQError) as e:
        hq.hq_gemm_noalloc(cdesc("uint4_g128"), 16, 256, 1024, 16, None, None, None, 16)
    assert e.value.status == 1  # HQ_ERR_INVALID_ARG
