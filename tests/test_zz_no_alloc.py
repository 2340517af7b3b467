"""moe_route_noalloc (static scratch, no context, no workspace) against moe_route.

This file is collected last so that, in a run that stops at the first failure,
every other test has already run. It must pass both alone in a fresh process
and after the rest of the suite.

The no-allocation router exists for callers that cannot allocate device memory
(engines that own all of HBM through their own pool, latency-critical paths
that cannot take cudaMalloc's device-wide synchronisation, plug-ins inside a
process whose allocator owns the device). Here it is called through the C ABI
several times in a row on different inputs (3 tokens, which takes the 4-token
logit kernel; 64 and 37 tokens; 170 tokens, next to the 65,536-logit limit at
384 experts); each call must give the workspace router's bits: the same top-k
indices and the same routing weights (both routers compute the same logits
in the same order and the weights with the same expf, sum and divide).
"""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_route_noalloc_matches_route_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    M.lib()
    dev = torch.device("cuda")
    H, E, K = 4096, 384, 8
    wr = synth.router_weight(E, H, seed=21, device=dev)
    bias = synth.zipf_logit_bias(E, 1.1, seed=21).to(dev)
    layer = M.MoeLayer(H, E, K, 2048, device=dev)
    for call, (T, first) in enumerate(((3, 9000), (64, 0), (37, 5000), (170, 12000))):
        x = synth.tokens(T, H, seed=21, device=dev, first_token=first)
        ref_idx, ref_w = layer.route(x, wr, bias)
        idx = torch.full((T, K), -7, dtype=torch.int32, device=dev)
        w = torch.full((T, K), -7.0, dtype=torch.float32, device=dev)
        M.moe_route_noalloc(x, wr, bias, T, H, E, K, idx, w)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy()), f"call {call}"
        assert np.array_equal(w.cpu().numpy().view(np.uint32), ref_w.cpu().numpy().view(np.uint32)), f"call {call}"
    # sizes beyond the static scratch are refused with a clear error
    too_many = M.binding.lib().moe_route_noalloc(None, None, None, 171, H, E, K, None, None, None)
    assert too_many == 2
    assert b"static scratch" in M.binding.lib().moe_last_error()
    layer.close()
