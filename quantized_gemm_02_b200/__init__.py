"""Python binding of libhq, the sm_100a quantised-weight GEMM library.

Argument marshalling only: every function below forwards to the C entry point
of the same name declared in ``include/hq.h`` (torch tensors become device
pointers, the stream defaults to torch's current stream) and raises
:class:`HQError` on a non-OK status.  No step of the computation runs here;
if ``libhq.so`` is missing the import of any entry point fails loudly.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "HQError", "QuantDesc", "ComputeConfig", "PlanInfo", "lib", "library_path", "EXPORTS",
    "HQ_BF16", "HQ_FP32", "HQ_INT4", "HQ_UINT4", "HQ_E2M1", "HQ_E4M3", "HQ_E8M0", "HQ_UE4M3", "HQ_MXFP8",
    "HQ_NVFP4", "HQ_INT2", "HQ_UINT2", "HQ_INT3", "HQ_UINT3", "HQ_E2M3", "HQ_E3M2", "HQ_E0M3", "HQ_INT1", "HQ_UINT1",
    "HQ_MOE_GROUPED", "HQ_MOE_INDEXED",
    "hq_status_string", "hq_device_error", "hq_packed_weights_bytes", "hq_pack_weights", "hq_unpack_weights",
    "hq_quant_act", "hq_gemm_workspace_bytes", "hq_gemm", "hq_gemm_config_workspace_bytes",
    "hq_gemm_config", "hq_gemm_plan", "hq_moe_plan", "hq_moe_permute", "hq_moe_workspace_bytes",
    "hq_moe_gemm", "hq_moe_masked_workspace_bytes", "hq_moe_gemm_masked", "hq_silu_and_mul", "hq_moe_unpermute_sum",
    "hq_gemm_noalloc", "hq_selftest_wait_timeout", "hq_pack_weights_gated", "hq_unpack_weights_gated",
    "hq_moe_gated_workspace_bytes", "hq_moe_gemm_gated",
]

HQ_BF16, HQ_FP32, HQ_INT4, HQ_UINT4, HQ_E2M1, HQ_E4M3, HQ_E8M0, HQ_UE4M3, HQ_MXFP8, HQ_NVFP4 = range(10)
HQ_INT2, HQ_UINT2, HQ_INT3, HQ_UINT3, HQ_E2M3, HQ_E3M2, HQ_E0M3, HQ_INT1, HQ_UINT1 = range(10, 19)
HQ_MOE_GROUPED, HQ_MOE_INDEXED = 0, 1

STATUS = {
    0: "HQ_OK", 1: "HQ_ERR_INVALID_ARG", 2: "HQ_ERR_UNSUPPORTED", 3: "HQ_ERR_WORKSPACE", 4: "HQ_ERR_CUDA",
    5: "HQ_ERR_TIMEOUT", 6: "HQ_ERR_DEVICE_INDEX", 7: "HQ_ERR_ARCH",
}

# Every symbol include/hq.h declares.
EXPORTS = (
    "hq_status_string", "hq_device_error", "hq_packed_weights_bytes", "hq_pack_weights", "hq_unpack_weights",
    "hq_quant_act", "hq_gemm_workspace_bytes", "hq_gemm", "hq_gemm_config_workspace_bytes",
    "hq_gemm_config", "hq_gemm_plan", "hq_moe_plan", "hq_moe_permute", "hq_moe_workspace_bytes",
    "hq_moe_gemm", "hq_moe_masked_workspace_bytes", "hq_moe_gemm_masked", "hq_silu_and_mul", "hq_moe_unpermute_sum",
    "hq_gemm_noalloc", "hq_selftest_wait_timeout", "hq_pack_weights_gated", "hq_unpack_weights_gated",
    "hq_moe_gated_workspace_bytes", "hq_moe_gemm_gated",
)


class HQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({_lib().hq_status_string(status).decode()})")


class QuantDesc(ctypes.Structure):
    """hq_quant_desc: the unified quantisation description."""
    _fields_ = [
        ("w_dtype", ctypes.c_int32), ("w_group", ctypes.c_int32), ("w_scale_dtype", ctypes.c_int32),
        ("w_has_zero", ctypes.c_int32), ("w_has_global", ctypes.c_int32), ("a_dtype", ctypes.c_int32),
        ("a_group", ctypes.c_int32),
    ]

    def __repr__(self):
        return ("QuantDesc(w_dtype=%d, w_group=%d, w_scale_dtype=%d, w_has_zero=%d, w_has_global=%d, a_dtype=%d, "
                "a_group=%d)" % (self.w_dtype, self.w_group, self.w_scale_dtype, self.w_has_zero, self.w_has_global,
                                 self.a_dtype, self.a_group))


class ComputeConfig(ctypes.Structure):
    """hq_compute_config: compute options (zero = the defaults)."""
    _fields_ = [("batch_invariant", ctypes.c_int32), ("reserved", ctypes.c_int32 * 7)]


class PlanInfo(ctypes.Structure):
    """hq_plan_info: the kernel and tiling a call would use."""
    _fields_ = [("kernel", ctypes.c_int32), ("layout", ctypes.c_int32), ("token_tile", ctypes.c_int32),
                ("weight_tiles", ctypes.c_int32), ("token_tiles", ctypes.c_int32), ("ctas", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]

    def as_dict(self):
        return {k: getattr(self, k) for k in ("kernel", "layout", "token_tile", "weight_tiles", "token_tiles",
                                                "ctas")}


HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(HERE, "libhq.so")


_LIB = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m quantized_gemm_02_b200.build`")
        L = ctypes.CDLL(path)
        P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        D = ctypes.POINTER(QuantDesc)
        C = ctypes.POINTER(ComputeConfig)
        sig = {
            "hq_status_string": (ctypes.c_char_p, [I]),
            "hq_device_error": (I, [P]),
            "hq_packed_weights_bytes": (Z, [D, I, I, I]),
            "hq_pack_weights": (I, [D, I, I, I, P, P, P, P, P, P]),
            "hq_unpack_weights": (I, [D, I, I, I, P, P, P, P, P, P]),
            "hq_quant_act": (I, [D, I, I, P, P, P, P, P, P, Z, P]),
            "hq_gemm_workspace_bytes": (Z, [D, I, I, I]),
            "hq_gemm": (I, [D, I, I, I, P, P, P, P, P, P, Z, P]),
            "hq_moe_permute": (I, [I, I, I, P, P, P, P, P]),
            "hq_moe_workspace_bytes": (Z, [I, D, I, I, I, I, I, I, I]),
            "hq_moe_gemm": (I, [I, D, I, I, I, I, I, P, P, P, P, I, P, P, P, P, I, F, P, P, Z, P]),
            "hq_moe_masked_workspace_bytes": (Z, [D, I, I, I, I, I]),
            "hq_moe_gemm_masked": (I, [D, I, I, I, I, P, P, P, I, P, P, Z, P]),
            "hq_silu_and_mul": (I, [I, I, P, P, P]),
            "hq_gemm_config_workspace_bytes": (Z, [D, C, I, I, I]),
            "hq_gemm_config": (I, [D, C, I, I, I, P, P, P, P, P, P, Z, P]),
            "hq_gemm_plan": (I, [D, C, I, I, I, ctypes.POINTER(PlanInfo)]),
            "hq_moe_plan": (I, [D, I, I, I, I, I, I, ctypes.POINTER(PlanInfo)]),
            "hq_moe_unpermute_sum": (I, [I, I, I, P, P, P, F, P, P]),
            "hq_gemm_noalloc": (I, [D, I, I, I, P, P, P, P, P, P]),
            "hq_selftest_wait_timeout": (I, [ctypes.c_ulonglong, P]),
            "hq_pack_weights_gated": (I, [D, I, I, I, P, P, P, P, P, P]),
            "hq_unpack_weights_gated": (I, [D, I, I, I, P, P, P, P, P, P]),
            "hq_moe_gated_workspace_bytes": (Z, [I, D, I, I, I, I, I]),
            "hq_moe_gemm_gated": (I, [I, D, I, I, I, I, I, P, P, P, P, P, P, P, P, P, Z, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


lib = _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, status):
    if status != 0:
        raise HQError(fn, status)


def hq_status_string(status: int) -> str:
    return _lib().hq_status_string(status).decode()


def hq_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word."""
    return _lib().hq_device_error(_stream(stream))


def hq_packed_weights_bytes(desc: QuantDesc, E: int, N: int, K: int) -> int:
    return _lib().hq_packed_weights_bytes(ctypes.byref(desc), E, N, K)


def hq_pack_weights(desc, E, N, K, codes, scales, zeros, global_scale, packed, stream=None):
    _check("hq_pack_weights", _lib().hq_pack_weights(
        ctypes.byref(desc), E, N, K, _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(global_scale), _ptr(packed),
        _stream(stream)))


def hq_unpack_weights(desc, E, N, K, packed, codes, scales, zeros, global_scale, stream=None):
    _check("hq_unpack_weights", _lib().hq_unpack_weights(
        ctypes.byref(desc), E, N, K, _ptr(packed), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(global_scale),
        _stream(stream)))


def hq_quant_act(desc, M, K, x, codes, scales, global_out=None, static_global=None, workspace=None,
                 ws_bytes=0, stream=None):
    _check("hq_quant_act", _lib().hq_quant_act(
        ctypes.byref(desc), M, K, _ptr(x), _ptr(codes), _ptr(scales), _ptr(global_out), _ptr(static_global),
        _ptr(workspace), ws_bytes, _stream(stream)))


def hq_gemm_workspace_bytes(desc, M, N, K) -> int:
    return _lib().hq_gemm_workspace_bytes(ctypes.byref(desc), M, N, K)


def hq_gemm(desc, M, N, K, packed_w, a, a_scales, a_global, c, workspace, ws_bytes, stream=None):
    _check("hq_gemm", _lib().hq_gemm(
        ctypes.byref(desc), M, N, K, _ptr(packed_w), _ptr(a), _ptr(a_scales), _ptr(a_global), _ptr(c),
        _ptr(workspace), ws_bytes, _stream(stream)))


def _cfg(cfg):
    return None if cfg is None else ctypes.byref(cfg)


def hq_gemm_config_workspace_bytes(desc, cfg, M, N, K) -> int:
    return _lib().hq_gemm_config_workspace_bytes(ctypes.byref(desc), _cfg(cfg), M, N, K)


def hq_gemm_config(desc, cfg, M, N, K, packed_w, a, a_scales, a_global, c, workspace, ws_bytes, stream=None):
    _check("hq_gemm_config", _lib().hq_gemm_config(
        ctypes.byref(desc), _cfg(cfg), M, N, K, _ptr(packed_w), _ptr(a), _ptr(a_scales), _ptr(a_global), _ptr(c),
        _ptr(workspace), ws_bytes, _stream(stream)))


def hq_gemm_plan(desc, cfg, M, N, K) -> dict:
    info = PlanInfo()
    _check("hq_gemm_plan", _lib().hq_gemm_plan(ctypes.byref(desc), _cfg(cfg), M, N, K, ctypes.byref(info)))
    return info.as_dict()


def hq_moe_plan(desc, T, topk, E, N, K, a_per_slot) -> dict:
    info = PlanInfo()
    _check("hq_moe_plan", _lib().hq_moe_plan(ctypes.byref(desc), T, topk, E, N, K, a_per_slot, ctypes.byref(info)))
    return info.as_dict()


def hq_moe_permute(T, topk, E, topk_ids, expert_offsets, perm, inv_perm, stream=None):
    _check("hq_moe_permute", _lib().hq_moe_permute(
        T, topk, E, _ptr(topk_ids), _ptr(expert_offsets), _ptr(perm), _ptr(inv_perm), _stream(stream)))


def hq_moe_workspace_bytes(mode, desc, T, topk, E, N, K, a_per_slot, combine) -> int:
    return _lib().hq_moe_workspace_bytes(mode, ctypes.byref(desc), T, topk, E, N, K, a_per_slot, combine)


def hq_moe_masked_workspace_bytes(desc, E, slab, N, K, expected_m) -> int:
    return _lib().hq_moe_masked_workspace_bytes(ctypes.byref(desc), E, slab, N, K, expected_m)


def hq_moe_gemm_masked(desc, E, slab, N, K, packed_w, a, expert_num_tokens, expected_m, out, workspace, ws_bytes,
                       stream=None):
    _check("hq_moe_gemm_masked", _lib().hq_moe_gemm_masked(
        ctypes.byref(desc), E, slab, N, K, _ptr(packed_w), _ptr(a), _ptr(expert_num_tokens), expected_m, _ptr(out),
        _ptr(workspace), ws_bytes, _stream(stream)))


def hq_silu_and_mul(R, I, y, out, stream=None):
    _check("hq_silu_and_mul", _lib().hq_silu_and_mul(R, I, _ptr(y), _ptr(out), _stream(stream)))


def hq_moe_gemm(mode, desc, T, topk, E, N, K, packed_w, a, a_scales, a_global, a_per_slot, topk_ids, topk_weights,
                expert_offsets, perm, combine, routed_scale, out, workspace, ws_bytes, stream=None):
    _check("hq_moe_gemm", _lib().hq_moe_gemm(
        mode, ctypes.byref(desc), T, topk, E, N, K, _ptr(packed_w), _ptr(a), _ptr(a_scales), _ptr(a_global),
        a_per_slot, _ptr(topk_ids), _ptr(topk_weights), _ptr(expert_offsets), _ptr(perm), combine,
        float(routed_scale), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


def hq_moe_unpermute_sum(T, topk, N, y, inv_perm, topk_weights, routed_scale, out, stream=None):
    _check("hq_moe_unpermute_sum", _lib().hq_moe_unpermute_sum(
        T, topk, N, _ptr(y), _ptr(inv_perm), _ptr(topk_weights), float(routed_scale), _ptr(out),
        _stream(stream)))


def hq_gemm_noalloc(desc, M, N, K, packed_w, a, a_scales, a_global, c, stream=None):
    """hq_gemm without a caller workspace: the library's fixed 64 MiB device
    scratch array is used instead (for callers that cannot allocate)."""
    _check("hq_gemm_noalloc", _lib().hq_gemm_noalloc(
        ctypes.byref(desc), M, N, K, _ptr(packed_w), _ptr(a), _ptr(a_scales), _ptr(a_global), _ptr(c),
        _stream(stream)))


def hq_selftest_wait_timeout(limit_ns: int, stream=None):
    """Runs the bounded-wait self-test (a wait nothing satisfies, limited to
    limit_ns); afterwards hq_device_error() reports HQ_ERR_TIMEOUT."""
    _check("hq_selftest_wait_timeout", _lib().hq_selftest_wait_timeout(int(limit_ns), _stream(stream)))



def hq_pack_weights_gated(desc, E, N2, K, codes, scales, zeros, global_scale, packed, stream=None):
    """hq_pack_weights for gate-up weights read by hq_moe_gemm_gated."""
    _check("hq_pack_weights_gated", _lib().hq_pack_weights_gated(
        ctypes.byref(desc), E, N2, K, _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(global_scale), _ptr(packed),
        _stream(stream)))


def hq_unpack_weights_gated(desc, E, N2, K, packed, codes, scales, zeros, global_scale, stream=None):
    _check("hq_unpack_weights_gated", _lib().hq_unpack_weights_gated(
        ctypes.byref(desc), E, N2, K, _ptr(packed), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(global_scale),
        _stream(stream)))


def hq_moe_gated_workspace_bytes(mode, desc, T, topk, E, I, K) -> int:
    return _lib().hq_moe_gated_workspace_bytes(mode, ctypes.byref(desc), T, topk, E, I, K)


def hq_moe_gemm_gated(mode, desc, T, topk, E, I, K, packed_w, a, a_scales, a_global, topk_ids, expert_offsets, perm,
                      out, workspace, ws_bytes, stream=None):
    """Gate-up MoE GEMM with SiLU-and-mul in its epilogue: out [T * topk, I]."""
    _check("hq_moe_gemm_gated", _lib().hq_moe_gemm_gated(
        mode, ctypes.byref(desc), T, topk, E, I, K, _ptr(packed_w), _ptr(a), _ptr(a_scales), _ptr(a_global),
        _ptr(topk_ids), _ptr(expert_offsets), _ptr(perm), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))
