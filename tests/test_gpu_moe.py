"""GPU parity of the MoE path: routing prepare (bit-exact), grouped and
indexed expert GEMMs, fused weighted top-k sum, on-the-fly activation
quantisation, and the invariants (grouped == indexed, E=1 top-1 == dense)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from hqtest import assert_close, cdesc, gpu_pack, gpu_quant, make_weights, np_bits, oracle_decoder, oracle_quant

pytestmark = pytest.mark.gpu


def gpu_permute(ids_gpu, E):
    import quantized_gemm_02_b200 as hq
    T, k = ids_gpu.shape
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    hq.hq_moe_permute(T, k, E, ids_gpu, off, perm, inv)
    return off, perm, inv


@pytest.mark.parametrize("T,E,k,zipf", [(1, 256, 8, False), (300, 64, 8, True), (2048, 256, 8, False),
                                         (4096, 256, 8, True), (5, 3, 2, False)])
def test_permute_bit_exact(T, E, k, zipf):
    g = synth.generator(T + E)
    ids, _ = synth.routing_zipf(T, E, k, 1.2, g) if zipf else synth.routing_softmax_topk(T, E, k, g)
    off, perm, inv = gpu_permute(ids.cuda(), E)
    torch.cuda.synchronize()
    o_off, o_perm, o_inv = O.moe_permute(ids.numpy(), E)
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(perm.cpu().numpy(), o_perm)
    assert np.array_equal(inv.cpu().numpy(), o_inv)


def test_permute_rejects_bad_ids():
    import quantized_gemm_02_b200 as hq
    ids = torch.tensor([[0, 1], [2, 7]], dtype=torch.int32, device="cuda")
    off, perm, inv = gpu_permute(ids, 4)
    assert hq.hq_device_error() == 6
    assert int(off[4].item()) == -1
    assert hq.hq_device_error() == 0  # cleared


def run_moe(mode, wname, aname, packed, T, k, E, N, K, a, a_per_slot, off, perm, inv, w, rs, combine, ids=None,
            a_scales=None, a_global=None):
    """One hq_moe_gemm call; with ``ids`` and no off / perm the call routes itself."""
    import quantized_gemm_02_b200 as hq
    d = cdesc(wname, aname)
    wsb = hq.hq_moe_workspace_bytes(mode, d, T, k, E, N, K, a_per_slot, combine)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out = torch.empty((T if combine else T * k), N, dtype=torch.bfloat16, device="cuda")
    hq.hq_moe_gemm(mode, d, T, k, E, N, K, packed, a, a_scales, a_global, a_per_slot, ids, w, off, perm, combine, rs,
                   out, ws, wsb)
    return out


def moe_case(wname, aname, T, E, k, N, K, a_per_slot, seed, zipf=False, device_weights=False):
    """Inputs, the GPU results for both modes and both combine settings, and
    the oracle's combined output / per-slot outputs."""
    g = synth.generator(seed)
    x = synth.bf16_normal((T * k if a_per_slot else T, K), g)
    ids, wts = synth.routing_zipf(T, E, k, 1.2, g) if zipf else synth.routing_softmax_topk(T, E, k, g)
    w = make_weights(wname, E, N, K, seed=seed + 1, device="cuda" if device_weights else "cpu")
    packed = gpu_pack(wname, w, E, N, K, aname)
    off, perm, inv = gpu_permute(ids.cuda(), E)
    res = {}
    for mode in (0, 1):
        for combine in (0, 1):
            res[(mode, combine)] = run_moe(mode, wname, aname, packed, T, k, E, N, K, x.cuda(), a_per_slot, off,
                                           perm, inv, wts.cuda(), 1.5, combine)
    torch.cuda.synchronize()
    xb = np_bits(x)
    if aname == "bf16":
        A, row = O.decode_act("bf16", xb.shape[0], K, xb)
    else:
        q, s, og = oracle_quant(aname, xb)
        A, row = O.decode_act(aname, xb.shape[0], K, q, s, og)
    slots_rows = np.arange(T * k) if a_per_slot else np.repeat(np.arange(T), k)
    A_slots = A[slots_rows]
    row_slots = None if row is None else row[slots_rows]
    dec = oracle_decoder(wname, w, N, K)
    out, bound, Y, B = O.moe(A_slots, ids.numpy(), wts.numpy(), dec, routed_scale=1.5, row_scale=row_slots)
    return res, out, bound, Y, B, ids.numpy(), wts.numpy()


@pytest.mark.parametrize("wname,aname", [("mxfp4", "bf16"), ("int4_g128", "bf16"), ("uint4_g64", "bf16"),
                                         ("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("fp8", "fp8"), ("mxint4", "bf16"),
                                         ("fp8b", "fp8g"), ("int3_g128", "bf16"), ("e3m2", "bf16")])
@pytest.mark.parametrize("a_per_slot", [0, 1])
def test_moe_small(wname, aname, a_per_slot):
    T, E, k, N, K = 23, 16, 4, 96, 256
    res, out, bound, Y, B, ids, wts = moe_case(wname, aname, T, E, k, N, K, a_per_slot, seed=31, zipf=True)
    # grouped and indexed agree bit for bit
    assert torch.equal(res[(0, 0)], res[(1, 0)])
    assert torch.equal(res[(0, 1)], res[(1, 1)])
    assert_close(res[(0, 0)].cpu(), Y, B, what="per-slot Y")
    # combine: Y is rounded to bf16 before the fp32 weighted sum, so the bound
    # doubles (two bf16 roundings)
    assert_close(res[(0, 1)].cpu(), out, bound, rel=8e-3, what="combined")


@pytest.mark.parametrize("wname,aname", [("nvfp4", "nvfp4"), ("mxfp4", "mxfp8"), ("fp8", "fp8"), ("fp8b", "fp8g")])
def test_moe_block_scaled_wide_token_tiles(wname, aname):
    # ~150 routed rows per expert: NVFP4 x NVFP4 takes 192-token tiles
    # (activation scale chunks of two 128-row halves), the other pairs
    # 128-token tiles; Zipf routing gives some experts more than one tile
    T, E, k, N, K = 300, 16, 8, 96, 256
    res, out, bound, Y, B, ids, wts = moe_case(wname, aname, T, E, k, N, K, 0, seed=37, zipf=True)
    assert torch.equal(res[(0, 0)], res[(1, 0)])
    assert_close(res[(0, 0)].cpu(), Y, B, what="per-slot Y")
    assert_close(res[(0, 1)].cpu(), out, bound, rel=8e-3, what="combined")


@pytest.mark.parametrize("wname,aname,T", [("mxfp4", "bf16", 100), ("mxfp4", "bf16", 300), ("int4_g128", "fp8", 300),
                                           ("nvfp4", "mxfp8", 100), ("uint4_g64", "nvfp4", 300)])
def test_moe_indexed_multi_stage_tiles(wname, aname, T):
    # 50 and 150 rows per expert on average: 64- and 256-token tiles of the
    # multi-stage kernel; indexed mode gathers the caller's rows (bf16, or
    # the caller's rows decoded once) with 4-row tensor gathers, grouped mode
    # copies the routed rows first; both must agree bit for bit
    E, k, N, K = 16, 8, 96, 256
    res, out, bound, Y, B, ids, wts = moe_case(wname, aname, T, E, k, N, K, 0, seed=41 + T, zipf=True)
    assert torch.equal(res[(0, 0)], res[(1, 0)])
    assert torch.equal(res[(0, 1)], res[(1, 1)])
    assert_close(res[(1, 0)].cpu(), Y, B, what="indexed per-slot Y")
    assert_close(res[(1, 1)].cpu(), out, bound, rel=8e-3, what="indexed combined")


@pytest.mark.parametrize("wname,aname", [("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("int4_g128", "fp8"), ("fp8", "fp8"),
                                         ("mxfp4", "bf16"), ("fp8b", "fp8g")])
@pytest.mark.parametrize("mode", [0, 1])
def test_moe_caller_quantised_and_self_routed(wname, aname, mode):
    # activations quantised by the caller (hq_quant_act) and passed with
    # their scales, routing from topk_ids alone (the call prepares it):
    # bit-identical to on-the-fly quantisation with explicit routing, and
    # within the tolerance of the oracle
    T, E, k, N, K = 37, 16, 4, 96, 256
    g = synth.generator(77)
    x = synth.bf16_normal((T, K), g)
    ids, wts = synth.routing_softmax_topk(T, E, k, g)
    w = make_weights(wname, E, N, K, seed=78)
    packed = gpu_pack(wname, w, E, N, K, aname)
    off, perm, inv = gpu_permute(ids.cuda(), E)
    ref = run_moe(mode, wname, aname, packed, T, k, E, N, K, x.cuda(), 0, off, perm, inv, wts.cuda(), 1.5, 1)
    if aname == "bf16":
        a, a_s, a_g = x.cuda(), None, None
    else:
        a, a_s, a_g = gpu_quant(aname, x.cuda())
        if aname != "nvfp4":
            a_g = None
    got = run_moe(mode, wname, aname, packed, T, k, E, N, K, a, 0, None, None, None, wts.cuda(), 1.5, 1,
                  ids=ids.cuda(), a_scales=a_s, a_global=a_g)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    xb = np_bits(x)
    if aname == "bf16":
        A, row = O.decode_act("bf16", T, K, xb)
    else:
        q, s, og = oracle_quant(aname, xb)
        A, row = O.decode_act(aname, T, K, q, s, og)
    rows = np.repeat(np.arange(T), k)
    o, b, _, _ = O.moe(A[rows], ids.numpy(), wts.numpy(), oracle_decoder(wname, w, N, K), 1.5,
                       None if row is None else row[rows])
    assert_close(got.cpu(), o, b, rel=8e-3, what=f"caller-quantised {wname}x{aname} mode {mode}")


def test_moe_single_expert_top1_equals_dense():
    import quantized_gemm_02_b200 as hq
    T, N, K = 17, 128, 512
    g = synth.generator(3)
    x = synth.bf16_normal((T, K), g).cuda()
    w = make_weights("mxfp4", 1, N, K, seed=4)
    packed = gpu_pack("mxfp4", w, 1, N, K)
    ids = torch.zeros(T, 1, dtype=torch.int32, device="cuda")
    wts = torch.ones(T, 1, dtype=torch.float32, device="cuda")
    off, perm, inv = gpu_permute(ids, 1)
    y = run_moe(0, "mxfp4", "bf16", packed, T, 1, 1, N, K, x, 0, off, perm, inv, wts, 1.0, 0)
    d = cdesc("mxfp4")
    wsb = hq.hq_gemm_workspace_bytes(d, T, N, K)
    ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device="cuda")
    c = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
    hq.hq_gemm(d, T, N, K, packed, x, None, None, c, ws, wsb)
    torch.cuda.synchronize()
    assert torch.equal(y, c)


@pytest.mark.parametrize("T", [1, 16])
def test_config3_shapes_gate_up(T):
    # MoE W4A16 MXFP4 gate-up GEMM at the full expert count: E=256, top-8,
    # N=4096, K=7168; weights drawn on the GPU, oracle on sampled columns of
    # the touched experts.
    E, k, N, K = 256, 8, 4096, 7168
    g = synth.generator(50 + T)
    x = synth.bf16_normal((T, K), g)
    ids, wts = synth.routing_softmax_topk(T, E, k, g)
    w = make_weights("mxfp4", E, N, K, seed=60, device="cuda")
    packed = gpu_pack("mxfp4", w, E, N, K)
    off, perm, inv = gpu_permute(ids.cuda(), E)
    out = {}
    for mode in (0, 1):
        out[mode] = run_moe(mode, "mxfp4", "bf16", packed, T, k, E, N, K, x.cuda(), 0, off, perm, inv, wts.cuda(),
                            1.0, 1)
    torch.cuda.synchronize()
    assert torch.equal(out[0], out[1])
    cols = np.sort(np.random.default_rng(T).choice(N, 128, replace=False))
    A, _ = O.decode_act("bf16", T, K, np_bits(x))
    codes, scales = w["codes"], w["scales"]

    def dec(e):
        c = synth.to_np_bits(codes[e][torch.as_tensor(cols, device="cuda")])
        s = synth.to_np_bits(scales[e][torch.as_tensor(cols, device="cuda")])
        return O.decode_weights(O.Desc("e2m1", 32, "e8m0"), len(cols), K, c, s)

    ref, bound, _, _ = O.moe(np.repeat(A, k, axis=0), ids.numpy(), wts.numpy(), dec, 1.0)
    assert_close(out[0].cpu()[:, torch.as_tensor(cols)], ref, bound, rel=8e-3, what=f"config3 T={T}")


@pytest.mark.parametrize("wname,aname", [("mxfp4", "bf16"), ("int4_g128", "bf16"), ("uint4_g64", "bf16"),
                                         ("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("fp8", "fp8"),
                                         ("nvfp4", "fp8")])
def test_moe_masked(wname, aname):
    # masked layout: E slabs of `slab` rows, expert e uses its first c_e rows;
    # empty and full slabs, NaN in every unused row, the output's unused rows
    # keep their contents.  Quantised activations: the oracle quantises the
    # valid rows alone (NVFP4: their own tensor scale).
    import quantized_gemm_02_b200 as hq
    E, slab, N, K = 8, 48, 96, 256
    counts = np.array([0, 48, 17, 1, 30, 48, 5, 22], dtype=np.int32)
    g = synth.generator(51)
    x = synth.bf16_normal((E * slab, K), g)
    valid = np.concatenate([np.arange(e * slab, e * slab + counts[e]) for e in range(E)])
    mask = np.zeros(E * slab, dtype=bool)
    mask[valid] = True
    x[torch.as_tensor(np.nonzero(~mask)[0])] = float("nan")
    w = make_weights(wname, E, N, K, seed=52)
    packed = gpu_pack(wname, w, E, N, K, aname)
    d = cdesc(wname, aname)
    wsb = hq.hq_moe_masked_workspace_bytes(d, E, slab, N, K, 24)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out = torch.full((E * slab, N), 7.0, dtype=torch.bfloat16, device="cuda")
    hq.hq_moe_gemm_masked(d, E, slab, N, K, packed, x.cuda(), torch.as_tensor(counts).cuda(), 24, out, ws, wsb)
    torch.cuda.synchronize()
    assert hq.hq_device_error() == 0
    xb = np_bits(x[torch.as_tensor(valid)])
    if aname == "bf16":
        A_valid, row_valid = O.decode_act("bf16", len(valid), K, xb)
    else:
        q, s, og = oracle_quant(aname, xb)
        A_valid, row_valid = O.decode_act(aname, len(valid), K, q, s, og)
    A_slab = np.full((E * slab, K), np.nan)
    A_slab[valid] = A_valid
    row_slab = None
    if row_valid is not None:
        row_slab = np.full(E * slab, np.nan)
        row_slab[valid] = row_valid
    Y, B, vmask = O.moe_masked(A_slab, counts, slab, oracle_decoder(wname, w, N, K), row_scale=row_slab)
    assert np.array_equal(vmask, mask)
    got = out.cpu()
    assert_close(got[torch.as_tensor(valid)], Y[valid], B[valid], what=f"masked {wname}x{aname}")
    assert torch.all(got[torch.as_tensor(np.nonzero(~mask)[0])].float() == 7.0)


def test_silu_and_mul():
    # fp32 on the GPU, rounded once to bf16: within half a bf16 step (2^-9
    # relative) of the fp64 oracle plus the fp32 steps' own error; the test
    # allows 2^-8 relative and a tiny absolute term; extreme gates included
    import quantized_gemm_02_b200 as hq
    R, I = 37, 136
    y = synth.bf16_normal((R, 2 * I), synth.generator(61)) * 3
    y[0, :8] = torch.tensor([0.0, 100.0, -100.0, 1e-3, -1e-3, 88.0, -90.0, 7.0], dtype=torch.bfloat16)
    out = torch.empty(R, I, dtype=torch.bfloat16, device="cuda")
    hq.hq_silu_and_mul(R, I, y.cuda(), out)
    torch.cuda.synchronize()
    ref = O.silu_and_mul(y.float().numpy().astype(np.float64))
    got = out.cpu().float().numpy().astype(np.float64)
    tol = np.abs(ref) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) / tol))


def _gated_pack(wname, aname, w, E, N2, K):
    import quantized_gemm_02_b200 as hq
    d = cdesc(wname, aname)
    packed = torch.empty(hq.hq_packed_weights_bytes(d, E, N2, K), dtype=torch.uint8, device="cuda")
    cu = {kk: (None if v is None else v.cuda()) for kk, v in w.items()}
    hq.hq_pack_weights_gated(d, E, N2, K, cu["codes"], cu["scales"], cu["zeros"], cu["global"], packed)
    return packed


@pytest.mark.parametrize("wname,aname", [("uint4_g64", "bf16"), ("mxfp4", "bf16"), ("fp8", "bf16"),
                                         ("mxfp4", "mxfp8"), ("nvfp4", "nvfp4"), ("fp8", "fp8")])
def test_pack_unpack_gated_identity(wname, aname):
    # the gated row order (gate and up rows side by side) round-trips
    import quantized_gemm_02_b200 as hq
    E, N2, K = 2, 256, 256
    w = make_weights(wname, E, N2, K, seed=90)
    packed = _gated_pack(wname, aname, w, E, N2, K)
    plain = gpu_pack(wname, w, E, N2, K, aname)
    assert not torch.equal(packed, plain)  # the row order differs
    out = {kk: (None if v is None else torch.zeros_like(v, device="cuda")) for kk, v in w.items()}
    hq.hq_unpack_weights_gated(cdesc(wname, aname), E, N2, K, packed, out["codes"], out["scales"], out["zeros"],
                               out["global"])
    torch.cuda.synchronize()
    for kk, v in w.items():
        if v is not None:
            assert np.array_equal(np_bits(out[kk]), np_bits(v)), kk


@pytest.mark.parametrize("wname,aname,T", [("mxfp4", "bf16", 5), ("mxfp4", "bf16", 300), ("int4_g128", "bf16", 40),
                                           ("uint4_g64", "fp8", 300), ("mxfp4", "mxfp8", 37), ("mxfp4", "mxfp8", 300),
                                           ("nvfp4", "nvfp4", 300), ("fp8", "fp8", 37), ("mxint4", "bf16", 23)])
@pytest.mark.parametrize("mode", [0, 1])
def test_moe_gate_up_with_fused_silu(wname, aname, T, mode):
    # SiLU-and-mul in the gate-up epilogue against the oracle's
    # silu_and_mul of its expert outputs.  Tolerance: the GEMM bound carried
    # through silu(g) * u (|silu'| <= 1.1), plus one bf16 rounding (2^-8
    # relative allows the fp32 steps too).  Decode, multi-stage (split and
    # whole tiles) and block-scaled kernels, both modes.
    import quantized_gemm_02_b200 as hq
    E, k, I, K = 16, 4, 128, 256
    N2 = 2 * I
    g = synth.generator(95 + T)
    x = synth.bf16_normal((T, K), g)
    ids, wts = synth.routing_zipf(T, E, k, 1.2, g)
    w = make_weights(wname, E, N2, K, seed=96)
    packed = _gated_pack(wname, aname, w, E, N2, K)
    d = cdesc(wname, aname)
    wsb = hq.hq_moe_gated_workspace_bytes(mode, d, T, k, E, I, K)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out = torch.full((T * k, I), float("nan"), dtype=torch.bfloat16, device="cuda")
    hq.hq_moe_gemm_gated(mode, d, T, k, E, I, K, packed, x.cuda(), None, None, ids.cuda(), None, None, out, ws, wsb)
    torch.cuda.synchronize()
    assert hq.hq_device_error() == 0
    xb = np_bits(x)
    if aname == "bf16":
        A, row = O.decode_act("bf16", T, K, xb)
    else:
        q, s, og = oracle_quant(aname, xb)
        A, row = O.decode_act(aname, T, K, q, s, og)
    rows = np.repeat(np.arange(T), k)
    Y, B = O.moe_expert_outputs(A[rows], ids.numpy(), oracle_decoder(wname, w, N2, K),
                                None if row is None else row[rows])
    ref = O.silu_and_mul(Y)
    gg, uu = Y[:, :I], Y[:, I:]
    sig = 1.0 / (1.0 + np.exp(-gg))
    dsilu = np.abs(sig * (1.0 + gg * (1.0 - sig)))
    tol = 4e-3 * (dsilu * B[:, :I] * np.abs(uu) + np.abs(gg * sig) * B[:, I:]) + 2.0 ** -8 * np.abs(ref) + 1e-5
    got = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= tol), float(np.max(err / tol))
