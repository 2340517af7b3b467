"""Failure detection on the GPU without a fault: a bounded wait that nothing
releases gives up after its limit, reports MOE_DEV_TIMEOUT through the
context's device status word, and leaves the context usable."""

import time

import pytest
import torch

import oracle
from helpers import LayerCase, assert_close_out

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_stays_usable():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    case = LayerCase(16, 256, 8, 2, 512, seed=31)
    ctx = case.layer.ctx
    assert case.layer.status() == 0
    flag = torch.zeros(1, dtype=torch.int32, device=case.dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    M.moe_debug_wait_flag(ctx, flag, 50_000_000)  # 50 ms; nothing sets the flag
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert 0.04 <= waited < 10.0, waited
    assert case.layer.status() == M.binding.MOE_DEV_TIMEOUT  # read, then cleared
    assert case.layer.status() == 0
    flag.fill_(1)  # a set flag releases the wait at once, with no error
    M.moe_debug_wait_flag(ctx, flag, 50_000_000)
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    out = case.forward()  # the context still runs the layer
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    assert_close_out(oracle.as_u16(out), case.oracle_forward()["out"], 2e-2)
    with pytest.raises(M.MoeError):
        M.moe_debug_wait_flag(ctx, flag, 3_000_000_000)  # above the 2 s bound: refused on the host
    case.close()
