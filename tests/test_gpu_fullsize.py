"""GPU parity at the full sizes of the benchmarked configurations, in the
launch configurations the benchmark times.

The oracle cannot multiply these sizes whole, so each case follows one
sampling rule: all N output columns of up to 256 random rows (decoded weight
rows taken in chunks), plus 4096 random (row, column) elements; MoE cases
check every routed row on a sample of output columns, every column of the
rows routed to a few experts, and 4096 random elements.  Inputs are drawn on
the GPU by the seeded generators (the same recipe as the benchmark) and
copied to the host for the oracle; quantised activations are quantised by the
oracle itself on the sampled rows (NVFP4 with the whole tensor's scale).

These paths are the ones small tests do not reach: whole tiles round-robin
over the persistent CTAs with token tiles rastered in groups (ragged last
group and tile included), Stream-K over thousands of tiles in the TMA-fed
kernel, and the MoE scheduler over 256 experts with uneven (Zipf) loads.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import (assert_close, cdesc, gpu_pack, gpu_quant, make_weights, np_bits, odesc, oracle_quant)

pytestmark = pytest.mark.gpu

N_ROWS, N_ELEMS, CHUNK = 256, 4096, 2048


def _rng(seed):
    return np.random.default_rng(seed)


def _oracle_rows(aname, x_bits_rows, glob=None):
    """The oracle's decoded activation rows (and per-row scales) for some rows
    of a tensor; NVFP4 rows use the whole tensor's scale ``glob``."""
    R, K = x_bits_rows.shape
    if aname == "bf16":
        return O.decode_act("bf16", R, K, x_bits_rows)
    if aname == "nvfp4":
        q, s, g = O.quant_nvfp4(x_bits_rows, global_scale=glob)
        return O.decode_act("nvfp4", R, K, q, s, g)
    q, s, _ = oracle_quant(aname, x_bits_rows)
    return O.decode_act(aname, R, K, q, s)


def _weight_rows(wname, w, rows, K):
    """Oracle decode of some weight rows (output columns) of expert 0 from the
    standard-format tensors (which may live on the GPU)."""
    idx = torch.as_tensor(np.asarray(rows), device=w["codes"].device)
    c = np_bits(w["codes"][0][idx])
    if wname == "fp8b":
        # block scales: each row's own 128-row block scale row
        s = np_bits(w["scales"][0][idx // 128])
        return O.decode_fp8_block_weights(c, s, 128, row_block=1), None
    s = np_bits(w["scales"][0][idx])
    z = None if w["zeros"] is None else np_bits(w["zeros"][0][idx])
    g = None if w["global"] is None else np_bits(w["global"])[0]
    return O.decode_weights(odesc(wname), len(rows), K, c, s, z, g)


def _check_dense(wname, aname, w, x, C, M, N, K, seed, glob=None):
    """All columns of sampled rows, then random elements.  Returns the worst
    err / bound ratio."""
    rng = _rng(seed)
    rows = np.arange(M) if M <= N_ROWS else np.sort(rng.choice(M, N_ROWS, replace=False))
    xb = np_bits(x[torch.as_tensor(rows, device=x.device)])
    A, rs = _oracle_rows(aname, xb, glob)
    got = C[torch.as_tensor(rows, device=C.device)].cpu()
    worst = 0.0
    for n0 in range(0, N, CHUNK):
        cols = np.arange(n0, min(N, n0 + CHUNK))
        W, col = _weight_rows(wname, w, cols, K)
        ref, bound = O.gemm(A, W, rs, col)
        worst = max(worst, assert_close(got[:, n0:n0 + len(cols)], ref, bound,
                                        what=f"{wname}x{aname} M={M} N={N} K={K} rows, cols {n0}.."))
    ms = rng.integers(0, M, N_ELEMS)
    ns = rng.integers(0, N, N_ELEMS)
    um, im = np.unique(ms, return_inverse=True)
    un, inn = np.unique(ns, return_inverse=True)
    Am, rsm = _oracle_rows(aname, np_bits(x[torch.as_tensor(um, device=x.device)]), glob)
    Wn, coln = _weight_rows(wname, w, un, K)
    ref = np.einsum("ik,ik->i", Am[im], Wn[inn])
    bound = np.einsum("ik,ik->i", np.abs(Am[im]), np.abs(Wn[inn]))
    if rsm is not None:
        ref, bound = ref * rsm[im], bound * np.abs(rsm[im])
    if coln is not None:
        ref, bound = ref * coln[inn], bound * np.abs(coln[inn])
    got_e = C[torch.as_tensor(ms, device=C.device), torch.as_tensor(ns, device=C.device)].cpu()
    worst = max(worst, assert_close(got_e, ref, bound, what=f"{wname}x{aname} M={M} elements"))
    return worst


def _run_dense(wname, aname, packed, a, a_s, a_g, M, N, K):
    import quantized_gemm_02_b200 as hq
    d = cdesc(wname, aname)
    wsb = hq.hq_gemm_workspace_bytes(d, M, N, K)
    ws = torch.zeros(max(wsb, 256), dtype=torch.uint8, device="cuda")
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    hq.hq_gemm(d, M, N, K, packed, a, a_s, a_g, C, ws, wsb)
    torch.cuda.synchronize()
    assert hq.hq_device_error() == 0
    return C


@pytest.mark.parametrize("M,N,K", [
    (4096, 8192, 8192),    # 1024 tiles: round-robin, two full raster groups of 8 token tiles
    (5000, 8192, 8192),    # raster groups 8 + 8 + 4 (ragged) and a ragged last token tile
    (8192, 28672, 8192),   # the benchmark's dominant call
    (256, 28672, 8192),    # one token tile, weights streamed once
    (1024, 8192, 28672),   # K = 28672
])
def test_w4a16_uint4_large_m(M, N, K):
    import quantized_gemm_02_b200 as hq
    plan = hq.hq_gemm_plan(cdesc("uint4_g128"), None, M, N, K)
    assert plan["kernel"] == 0 and plan["token_tile"] == 256
    assert plan["weight_tiles"] * plan["token_tiles"] >= plan["ctas"]  # whole tiles round-robin
    w = make_weights("uint4_g128", 1, N, K, seed=M + 1, device="cuda")
    packed = gpu_pack("uint4_g128", w, 1, N, K)
    x = synth.bf16_normal((M, K), synth.generator(M + 2, "cuda"), device="cuda")
    C = _run_dense("uint4_g128", "bf16", packed, x, None, None, M, N, K)
    assert _check_dense("uint4_g128", "bf16", w, x, C, M, N, K, seed=M) < 4e-3


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_w4a16_uint4_small_m_all_columns(M):
    # the decode kernel (Stream-K) and the two-CTA-per-SM multi-stage kernel
    # on the largest config-2 shape, every output column
    N, K = 28672, 8192
    w = make_weights("uint4_g128", 1, N, K, seed=100 + M, device="cuda")
    packed = gpu_pack("uint4_g128", w, 1, N, K)
    x = synth.bf16_normal((M, K), synth.generator(101 + M, "cuda"), device="cuda")
    C = _run_dense("uint4_g128", "bf16", packed, x, None, None, M, N, K)
    _check_dense("uint4_g128", "bf16", w, x, C, M, N, K, seed=M)


_QW = {}


def _quantised_weights(aname, N, K):
    """Config 5 weights: N(0,1) quantised per output row by the library and,
    bit-exact, by the oracle (cached per format)."""
    key = (aname, N, K)
    if key not in _QW:
        Wf = synth.bf16_normal((N, K), synth.generator(500, "cuda"), device="cuda")
        wc, wsc, wg = gpu_quant(aname, Wf)
        q, s, og = oracle_quant(aname, np_bits(Wf))
        torch.cuda.synchronize()
        assert np.array_equal(wc.cpu().numpy(), q)
        if aname == "fp8":
            assert np.array_equal(wsc.cpu().numpy().view(np.uint32), s.view(np.uint32))
        else:
            assert np.array_equal(wsc.cpu().numpy(), s)
        w = {"codes": wc[None], "scales": wsc[None], "zeros": None, "global": wg if aname == "nvfp4" else None}
        _QW[key] = w
    return _QW[key]


@pytest.mark.parametrize("aname", ["nvfp4", "fp8"])
@pytest.mark.parametrize("M", [256, 2048, 8192])
def test_config5_large_m(aname, M):
    # W4A4 NVFP4 x NVFP4 and W8A8 FP8 at N = K = 7168: the TMA-fed kernel
    # with Stream-K over thousands of (tile, stage) iterations
    N = K = 7168
    wname = "nvfp4" if aname == "nvfp4" else "fp8"
    w = _quantised_weights(aname, N, K)
    packed = gpu_pack(wname, w, 1, N, K, aname)
    x = synth.bf16_normal((M, K), synth.generator(600 + M, "cuda"), device="cuda")
    ac, asc, ag = gpu_quant(aname, x)
    glob = None
    if aname == "nvfp4":
        glob = O.nvfp4_global_scale(np_bits(x))
        assert np.float32(ag.item()) == glob
    C = _run_dense(wname, aname, packed, ac, asc, ag if aname == "nvfp4" else None, M, N, K)
    _check_dense(wname, aname, w, x, C, M, N, K, seed=M, glob=glob)


@pytest.mark.parametrize("M", [32, 2048])
def test_fp8_block_scaled_dense(M):
    # block-scaled FP8 W8A8 at N = K = 7168 (128 x 128 weight blocks, per
    # token and 128 k activation scales quantised on the GPU)
    N = K = 7168
    w = make_weights("fp8b", 1, N, K, seed=750 + M, device="cuda")
    packed = gpu_pack("fp8b", w, 1, N, K, "fp8g")
    x = synth.bf16_normal((M, K), synth.generator(751 + M, "cuda"), device="cuda")
    ac, asc, _ = gpu_quant("fp8g", x)
    C = _run_dense("fp8b", "fp8g", packed, ac, asc, None, M, N, K)
    _check_dense("fp8b", "fp8g", w, x, C, M, N, K, seed=M)


@pytest.mark.parametrize("M", [2048, 8192])
def test_mxfp4_mxfp8_dense_large_m(M):
    # MXFP4 weights x MXFP8 activations on the block-scaled MMA at N = K = 7168
    N = K = 7168
    w = make_weights("mxfp4", 1, N, K, seed=700 + M, device="cuda")
    packed = gpu_pack("mxfp4", w, 1, N, K, "mxfp8")
    x = synth.bf16_normal((M, K), synth.generator(701 + M, "cuda"), device="cuda")
    ac, asc, _ = gpu_quant("mxfp8", x)
    C = _run_dense("mxfp4", "mxfp8", packed, ac, asc, None, M, N, K)
    _check_dense("mxfp4", "mxfp8", w, x, C, M, N, K, seed=M)


# ---------------------------------------------------------------------------
# MoE at the configs' shapes: E = 256, top-8, H = 7168, I = 2048
# ---------------------------------------------------------------------------
E_, K_TOP, H_, I_ = 256, 8, 7168, 2048


def _moe_full(wname, aname, T, part, zipf, seed, modes=(0, 1)):
    import quantized_gemm_02_b200 as hq
    N, K, per_slot = (2 * I_, H_, 0) if part == "gate_up" else (H_, I_, 1)
    g = synth.generator(seed, "cuda")
    x = synth.bf16_normal((T * K_TOP if per_slot else T, K), g, device="cuda")
    if zipf:
        ids, wts = synth.routing_zipf(T, E_, K_TOP, 1.2, g, device="cuda")
    else:
        ids, wts = synth.routing_softmax_topk(T, E_, K_TOP, g, device="cuda")
    w = make_weights(wname, E_, N, K, seed=seed + 1, device="cuda")
    packed = gpu_pack(wname, w, E_, N, K, aname)
    rng = _rng(seed)
    ids_np = ids.cpu().numpy()
    flat = ids_np.reshape(-1)
    cols = np.sort(rng.choice(N, 128, replace=False))
    touched = np.unique(flat)
    full_experts = rng.choice(touched, 2, replace=False)
    cols2 = np.sort(rng.choice(N, 512, replace=False))
    # host copies of what the oracle decodes, then the standard-format weights go
    sub = {}
    for key in ("codes", "scales", "zeros"):
        v = w[key]
        if v is None:
            sub[key] = (None, None, None)
            continue
        div = 128 if (wname == "fp8b" and key == "scales") else 1  # block scales: one row per 128
        sub[key] = (np_bits(v[:, torch.as_tensor(cols // div, device="cuda")]),
                    np_bits(v[:, torch.as_tensor(cols2 // div, device="cuda")]),
                    {int(e): np_bits(v[int(e)]) for e in full_experts})
    glob = None if w["global"] is None else np_bits(w["global"])
    del w
    torch.cuda.empty_cache()
    off = torch.empty(E_ + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * K_TOP, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * K_TOP, dtype=torch.int32, device="cuda")
    hq.hq_moe_permute(T, K_TOP, E_, ids, off, perm, inv)
    d = cdesc(wname, aname)
    res = {}
    for mode in modes:
        for combine in (0, 1):
            wsb = hq.hq_moe_workspace_bytes(mode, d, T, K_TOP, E_, N, K, per_slot, combine)
            ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
            out = torch.full(((T if combine else T * K_TOP), N), float("nan"), dtype=torch.bfloat16, device="cuda")
            hq.hq_moe_gemm(mode, d, T, K_TOP, E_, N, K, packed, x, None, None, per_slot, None, wts, off, perm, combine,
                           1.0, out, ws, wsb)
            torch.cuda.synchronize()
            assert hq.hq_device_error() == 0
            res[(mode, combine)] = out
            del ws
    if len(modes) == 2:
        # both modes multiply the same rows in the same tiles and k order
        assert torch.equal(res[(0, 0)], res[(1, 0)]) and torch.equal(res[(0, 1)], res[(1, 1)])
    # oracle side
    xb = np_bits(x)
    gl = O.nvfp4_global_scale(xb) if aname == "nvfp4" else None
    A, rs = _oracle_rows(aname, xb, gl)
    slot_rows = np.arange(T * K_TOP) if per_slot else np.repeat(np.arange(T), K_TOP)
    A_slots = A[slot_rows]
    rs_slots = None if rs is None else rs[slot_rows]
    od = odesc(wname)

    def dec_from(which, e, n):
        # which: 0 = the sampled columns, 1 = the element columns, 2 = whole experts
        c, s, z = (sub["codes"][which], sub["scales"][which], sub["zeros"][which])
        if wname == "fp8b" and which != 2:
            return O.decode_fp8_block_weights(c[e], s[e], 128, row_block=1), None
        return O.decode_weights(od, n, K, c[e], s[e], None if z is None else z[e], None if glob is None else glob[e])

    out_c, bound_c, Y, B = O.moe(A_slots, ids_np, wts.cpu().numpy(), lambda e: dec_from(0, e, len(cols)), 1.0,
                                  row_scale=rs_slots)
    tc = torch.as_tensor(cols)
    for mode in modes:
        assert_close(res[(mode, 0)].cpu()[:, tc], Y, B, what=f"moe {wname}x{aname} T={T} {part} mode {mode} cols")
        assert_close(res[(mode, 1)].cpu()[:, tc], out_c, bound_c, rel=8e-3,
                     what=f"moe {wname}x{aname} T={T} {part} mode {mode} combined cols")
    # every column of the rows routed to two experts
    for e in full_experts:
        slots = np.nonzero(flat == e)[0]
        W, col = dec_from(2, int(e), N)
        ref, bound = O.gemm(A_slots[slots], W, None if rs_slots is None else rs_slots[slots], col)
        for mode in modes:
            assert_close(res[(mode, 0)].cpu()[torch.as_tensor(slots)], ref, bound,
                         what=f"moe {wname}x{aname} T={T} {part} mode {mode} expert {e}")
    # random elements
    ss = rng.integers(0, T * K_TOP, N_ELEMS)
    jj = rng.integers(0, len(cols2), N_ELEMS)
    ref = np.empty(N_ELEMS)
    bound = np.empty(N_ELEMS)
    for e in np.unique(flat[ss]):
        sel = np.nonzero(flat[ss] == e)[0]
        W, col = dec_from(1, int(e), len(cols2))
        a = A_slots[ss[sel]]
        wv = W[jj[sel]]
        r = np.einsum("ik,ik->i", a, wv)
        b = np.einsum("ik,ik->i", np.abs(a), np.abs(wv))
        if rs_slots is not None:
            r, b = r * rs_slots[ss[sel]], b * np.abs(rs_slots[ss[sel]])
        if col is not None:
            r, b = r * col[jj[sel]], b * np.abs(col[jj[sel]])
        ref[sel], bound[sel] = r, b
    for mode in modes:
        got = res[(mode, 0)][torch.as_tensor(ss, device="cuda"), torch.as_tensor(cols2[jj], device="cuda")].cpu()
        assert_close(got, ref, bound, what=f"moe {wname}x{aname} T={T} {part} mode {mode} elements")


@pytest.mark.parametrize("T,part", [(1024, "gate_up"), (4096, "gate_up"), (1024, "down"), (4096, "down")])
def test_config3_moe_w4a16_mxfp4(T, part):
    _moe_full("mxfp4", "bf16", T, part, zipf=False, seed=800 + T)


@pytest.mark.parametrize("T,part", [(512, "gate_up"), (4096, "gate_up"), (4096, "down")])
def test_config4_moe_w4a8_zipf(T, part):
    _moe_full("mxfp4", "mxfp8", T, part, zipf=True, seed=900 + T)


@pytest.mark.parametrize("T,part", [(16, "gate_up"), (4096, "gate_up"), (4096, "down")])
def test_moe_w4a16_mxint4(T, part):
    # MXINT4 weights (INT4 elements, E8M0 per 32) at the config-3 MoE shapes
    _moe_full("mxint4", "bf16", T, part, zipf=False, seed=1100 + T)


def test_moe_fp8_block_scaled():
    # block-scaled FP8 W8A8 MoE (the DeepGEMM-style layout) at the config-3
    # gate-up shape, T = 1024
    _moe_full("fp8b", "fp8g", 1024, "gate_up", zipf=False, seed=1200)


@pytest.mark.parametrize("part", ["gate_up", "down"])
def test_config5_moe_nvfp4(part):
    _moe_full("nvfp4", "nvfp4", 4096, part, zipf=False, seed=1000)
