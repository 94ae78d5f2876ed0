"""Device-side failure detection without a GPU fault: a wait that nothing
satisfies gives up after its bound, records HQ_ERR_TIMEOUT in the device
error word, and the context stays usable for the next call."""
import numpy as np
import pytest
import torch

import synth
from hqtest import assert_close, cdesc, gpu_pack, make_weights, oracle_decoder
import oracle as O

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    import quantized_gemm_02_b200 as hq
    assert hq.hq_device_error() == 0
    hq.hq_selftest_wait_timeout(2_000_000)  # 2 ms
    assert hq.hq_device_error() == 5  # HQ_ERR_TIMEOUT
    assert hq.hq_device_error() == 0  # read clears it


def test_selftest_rejects_unbounded_limits():
    import quantized_gemm_02_b200 as hq
    for bad in (0, 2_000_000_000):
        with pytest.raises(hq.HQError) as e:
            hq.hq_selftest_wait_timeout(bad)
        assert e.value.status == 1  # HQ_ERR_INVALID_ARG


def test_context_usable_after_timeout():
    import quantized_gemm_02_b200 as hq
    hq.hq_selftest_wait_timeout(1_000_000)
    assert hq.hq_device_error() == 5
    M, N, K = 4, 136, 256
    w = make_weights("int4_g128", 1, N, K, seed=11)
    packed = gpu_pack("int4_g128", w, 1, N, K)
    x = synth.bf16_normal((M, K), synth.generator(12))
    d = cdesc("int4_g128")
    wsb = hq.hq_gemm_workspace_bytes(d, M, N, K)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    hq.hq_gemm(d, M, N, K, packed, x.cuda(), None, None, c, ws, wsb)
    assert hq.hq_device_error() == 0
    A, _ = O.decode_act("bf16", M, K, synth.to_np_bits(x))
    W, col = oracle_decoder("int4_g128", w, N, K)(0)
    ref, bound = O.gemm(A, W, None, col)
    assert_close(c.cpu(), ref, bound, what="GEMM after a timed-out wait")
