"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point include/hq.h declares, and rejects bad arguments on the
host before touching a device."""
import ctypes
import os
import re

import pytest

import quantized_gemm_02_b200 as hq
from hqtest import cdesc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^HQ_API\s+[^(]*?\b(hq_\w+)\s*\(", txt, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    L = hq.lib()
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(hq.EXPORTS) <= set(names)


def test_status_strings():
    for s in range(8):
        assert hq.hq_status_string(s)
    assert hq.hq_status_string(99) == "unknown status"


def test_packed_size_queries():
    # INT4 g128, N=4096, K=4096: 8 MiB codes + 32 groups x 64 rows x 2 B per tile row
    n = hq.hq_packed_weights_bytes(cdesc("int4_g128"), 1, 4096, 4096)
    assert n >= 4096 * 4096 // 2 + 4096 * 32 * 2
    assert n < 4096 * 4096 // 2 * 1.05
    # E experts scale linearly
    assert hq.hq_packed_weights_bytes(cdesc("mxfp4"), 8, 256, 512) == 8 * hq.hq_packed_weights_bytes(cdesc("mxfp4"), 1, 256, 512)
    # ragged N pads to 64 rows
    assert hq.hq_packed_weights_bytes(cdesc("fp8"), 1, 65, 128) == hq.hq_packed_weights_bytes(cdesc("fp8"), 1, 128, 128)
    # K not a multiple of 64 and unsupported descriptions give 0
    assert hq.hq_packed_weights_bytes(cdesc("int4_g128"), 1, 64, 96) == 0
    bad = cdesc("mxfp4")
    bad.w_group = 16
    assert hq.hq_packed_weights_bytes(bad, 1, 64, 128) == 0


def test_workspace_queries_are_consistent():
    d = cdesc("uint4_g128")
    assert hq.hq_gemm_workspace_bytes(d, 16, 8192, 8192) > 0
    dq = cdesc("nvfp4", "nvfp4")
    # quantised activations need a decode buffer on top
    assert hq.hq_gemm_workspace_bytes(dq, 32, 7168, 7168) >= 32 * 7168 * 2
    m = hq.hq_moe_workspace_bytes(hq.HQ_MOE_GROUPED, cdesc("mxfp4"), 16, 8, 256, 4096, 7168, 0, 1)
    assert m >= 16 * 8 * 4096 * 2 + 16 * 8 * 7168 * 2
    assert hq.hq_moe_workspace_bytes(hq.HQ_MOE_INDEXED, cdesc("mxfp4"), 16, 8, 256, 4096, 7168, 0, 0) < m


def test_host_validation_without_device():
    d = cdesc("int4_g128")
    with pytest.raises(hq.HQError) as e:
        hq.hq_pack_weights(d, 1, 64, 100, 16, 16, None, None, 16, stream=0)
    assert e.value.status == 1  # K not a multiple of 64
    bad = cdesc("int4_g128")
    bad.w_dtype = 99
    with pytest.raises(hq.HQError) as e:
        hq.hq_gemm(bad, 1, 64, 128, 16, 16, None, None, 16, 16, 0, stream=0)
    assert e.value.status == 2
    with pytest.raises(hq.HQError) as e:
        hq.hq_gemm(d, 1, 64, 128, 16, 16, None, None, 16, None, 0, stream=0)
    assert e.value.status == 3  # no workspace
    with pytest.raises(hq.HQError) as e:
        hq.hq_moe_permute(4, 2, 2000, 16, 16, 16, 16, stream=0)
    assert e.value.status == 1  # E > 1024
    # a zero-row GEMM is a no-op that succeeds without a device
    hq.hq_gemm(d, 0, 64, 128, 16, 16, None, None, 16, None, 0, stream=0)


def test_moe_gemm_host_validation():
    d = cdesc("mxfp4")
    T, k, E, N, K = 4, 2, 8, 128, 256
    wsb = hq.hq_moe_workspace_bytes(hq.HQ_MOE_INDEXED, d, T, k, E, N, K, 0, 0)
    assert wsb > 0
    call = lambda desc, a_s=None, a_g=None, ids=None, off=None, perm=None, ws=16: hq.hq_moe_gemm(
        hq.HQ_MOE_INDEXED, desc, T, k, E, N, K, 16, 16, a_s, a_g, 0, ids, None, off, perm, 0, 1.0, 16, ws, wsb,
        stream=0)
    with pytest.raises(hq.HQError) as e:
        call(d)  # neither routing arrays nor topk_ids
    assert e.value.status == 1
    with pytest.raises(hq.HQError) as e:
        call(d, off=16)  # offsets without perm
    assert e.value.status == 1
    with pytest.raises(hq.HQError) as e:
        call(d, a_s=16, ids=16)  # scales for bf16 activations
    assert e.value.status == 1
    with pytest.raises(hq.HQError) as e:
        call(cdesc("nvfp4", "nvfp4"), a_s=16, ids=16)  # NVFP4 codes without their tensor scale
    assert e.value.status == 1
    with pytest.raises(hq.HQError) as e:
        call(cdesc("mxfp4", "mxfp8"), a_s=18, ids=16)  # scales not 4-byte aligned
    assert e.value.status == 1
    with pytest.raises(hq.HQError) as e:
        call(d, ids=16, ws=None)
    assert e.value.status == 3
    bad = cdesc("mxfp4", "mxfp8")
    bad.a_group = 16  # MXFP8 scales are per 32
    with pytest.raises(hq.HQError) as e:
        call(bad, ids=16)
    assert e.value.status == 2
    assert hq.hq_moe_workspace_bytes(hq.HQ_MOE_INDEXED, bad, T, k, E, N, K, 0, 0) == 0
    ok = cdesc("mxfp4", "mxfp8")
    ok.a_group = 32
    assert hq.hq_moe_workspace_bytes(hq.HQ_MOE_INDEXED, ok, T, k, E, N, K, 0, 0) > 0
    # indexed mode stages no rows for bf16 activations; grouped copies T * topk rows
    g = hq.hq_moe_workspace_bytes(hq.HQ_MOE_GROUPED, d, 64, 8, 256, 4096, 7168, 0, 0)
    i = hq.hq_moe_workspace_bytes(hq.HQ_MOE_INDEXED, d, 64, 8, 256, 4096, 7168, 0, 0)
    assert g - i >= 64 * 8 * 7168 * 2


def test_compute_config_queries():
    d = cdesc("uint4_g128")
    assert hq.hq_gemm_config_workspace_bytes(d, None, 16, 8192, 8192) == hq.hq_gemm_workspace_bytes(d, 16, 8192, 8192)
    c = hq.ComputeConfig()
    assert hq.hq_gemm_config_workspace_bytes(d, c, 16, 8192, 8192) == hq.hq_gemm_workspace_bytes(d, 16, 8192, 8192)
    c.batch_invariant = 1
    assert hq.hq_gemm_config_workspace_bytes(d, c, 16, 8192, 8192) > 0
    assert hq.hq_gemm_config_workspace_bytes(cdesc("nvfp4", "nvfp4"), c, 300, 7168, 7168) > 0
    c.reserved[3] = 1  # unknown options must stay zero
    assert hq.hq_gemm_config_workspace_bytes(d, c, 16, 8192, 8192) == 0


def test_masked_moe_and_silu_host_validation():
    d = cdesc("mxfp4")
    # size query: E slabs of `slab` rows; the routing arrays sit after the MoE workspace
    n = hq.hq_moe_masked_workspace_bytes(d, 8, 48, 96, 256, 24)
    assert n >= 8 * 48 * 256 * 2 + 8 * 48 * 4
    assert hq.hq_moe_masked_workspace_bytes(d, 8, 48, 96, 256, 0) > 0      # expected_m < 1: the slab
    assert hq.hq_moe_masked_workspace_bytes(d, 0, 48, 96, 256, 24) == 0    # no experts
    assert hq.hq_moe_masked_workspace_bytes(d, 2000, 48, 96, 256, 24) == 0  # E > 1024
    assert hq.hq_moe_masked_workspace_bytes(d, 8, 0, 96, 256, 24) == 0     # empty slab
    assert hq.hq_moe_masked_workspace_bytes(d, 8, 48, 96, 100, 24) == 0    # K not a multiple of 64
    with pytest.raises(hq.HQError) as e:
        hq.hq_moe_gemm_masked(d, 8, 48, 96, 256, 16, 16, None, 24, 16, 16, n, stream=0)
    assert e.value.status == 1  # no expert_num_tokens
    with pytest.raises(hq.HQError) as e:
        hq.hq_moe_gemm_masked(d, 8, 48, 96, 256, 16, 16, 16, 24, 16, None, 0, stream=0)
    assert e.value.status == 3  # no workspace
    with pytest.raises(hq.HQError) as e:
        hq.hq_silu_and_mul(4, 12, 16, 16, stream=0)
    assert e.value.status == 1  # I not a multiple of 8
    with pytest.raises(hq.HQError) as e:
        hq.hq_silu_and_mul(4, 16, 17, 32, stream=0)
    assert e.value.status == 1  # misaligned input
    hq.hq_silu_and_mul(0, 16, None, None, stream=0)  # zero rows: a no-op without a device


def test_host_dispatch_plans():
    # which kernel and tiling each call takes (host only; 148 SMs without a device)
    p = hq.hq_gemm_plan
    # W4A16: decode kernel up to 32 tokens, then the multi-stage kernel
    assert p(cdesc("uint4_g128"), None, 16, 28672, 8192) == {
        "kernel": 1, "layout": 0, "token_tile": 16, "weight_tiles": 224, "token_tiles": 1, "ctas": 148}
    assert p(cdesc("uint4_g128"), None, 32, 8192, 8192)["token_tile"] == 32
    big = p(cdesc("uint4_g128"), None, 8192, 28672, 8192)
    assert big["kernel"] == 0 and big["token_tile"] == 256 and big["token_tiles"] == 32
    assert p(cdesc("uint4_g128"), None, 64, 8192, 8192)["token_tile"] == 64
    # the microscaling pairs take their own layouts and the TMA-fed kernel, at most 128 tokens
    mx = p(cdesc("mxfp4", "mxfp8"), None, 8192, 7168, 7168)
    assert (mx["kernel"], mx["layout"], mx["token_tile"]) == (2, 1, 128)
    nv = p(cdesc("nvfp4", "nvfp4"), None, 1, 7168, 7168)
    assert (nv["kernel"], nv["layout"], nv["token_tile"]) == (2, 2, 16)
    # dense NVFP4 from 1024 rows: 192-token tiles (a ragged last one at M = 8192)
    nv8k = p(cdesc("nvfp4", "nvfp4"), None, 8192, 7168, 7168)
    assert (nv8k["token_tile"], nv8k["token_tiles"]) == (192, 43)
    assert p(cdesc("nvfp4", "nvfp4"), None, 256, 7168, 7168)["token_tile"] == 128
    # other quantised pairs decode the activations and keep the dequantisation layout
    assert p(cdesc("nvfp4", "fp8"), None, 8192, 7168, 7168)["layout"] == 0
    # FP8 x FP8: 256-token tiles only with at least two per SM, else 128; K % 128 != 0 keeps the old layout
    assert p(cdesc("fp8", "fp8"), None, 8192, 7168, 7168)["token_tile"] == 256
    assert p(cdesc("fp8", "fp8"), None, 256, 7168, 7168)["token_tile"] == 128
    assert p(cdesc("fp8", "fp8"), None, 300, 7168, 192)["layout"] == 0
    # batch invariance: 64-token tiles, no K split (CTAs <= tiles; TMA-fed kernel: CTAs divide tiles)
    c = hq.ComputeConfig()
    c.batch_invariant = 1
    bi = p(cdesc("uint4_g128"), c, 1, 8192, 8192)
    assert (bi["kernel"], bi["token_tile"], bi["ctas"]) == (0, 64, 64)
    bi2 = p(cdesc("nvfp4", "nvfp4"), c, 300, 7168, 7168)
    tiles = bi2["weight_tiles"] * bi2["token_tiles"]
    assert bi2["token_tile"] == 64 and tiles % bi2["ctas"] == 0 and bi2["ctas"] <= 148
    # MoE: NVFP4 takes 192-token tiles at ~128 rows per expert, MXFP4 x MXFP8 stays at 128
    assert hq.hq_moe_plan(cdesc("nvfp4", "nvfp4"), 4096, 8, 256, 4096, 7168, 0)["token_tile"] == 192
    assert hq.hq_moe_plan(cdesc("mxfp4", "mxfp8"), 4096, 8, 256, 4096, 7168, 0)["token_tile"] == 128
    assert hq.hq_moe_plan(cdesc("mxfp4"), 1, 8, 256, 4096, 7168, 0)["token_tile"] == 16
