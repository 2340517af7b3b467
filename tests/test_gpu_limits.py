"""The header's size limits, exercised on the GPU against the oracle.

- T = 65536 tokens, K = 32, E = 1024 (2,097,152 pairs, the most the limits
  allow), small H and I: routing and the permutation bit-exact for every
  token, outputs on sampled tokens within 2e-2.
- H = I = 8192 (the largest hidden and intermediate sizes) with T = 16384 and
  K = 32: T * K * H = 2^32 elements, so every row offset into x_perm, h and
  y_pair needs 64-bit arithmetic; sampled outputs within 2e-2 (the last token
  among them).
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_out, oracle_layer_out

pytestmark = pytest.mark.gpu


def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _layer(H, E, K, I, seed):
    import mixture_experts_layer_24_b200 as M
    dev = torch.device("cuda")
    layer = M.MoeLayer(H, E, K, I, device=dev)
    keep = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=seed, device=dev)
        layer.register(e, g, d)
        keep.append((g, d))
    wr = synth.router_weight(E, H, seed=seed, device=dev)
    torch.cuda.synchronize()
    return layer, keep, wr


def test_most_pairs_most_experts_widest_top_k():
    _need_cuda()
    H, E, K, I, T, seed = 128, 1024, 32, 128, 65536, 71
    layer, keep, wr = _layer(H, E, K, I, seed)
    x = synth.tokens(T, H, seed=seed, device="cuda")
    idx, w = layer.route(x, wr)
    counts, offsets, ps, pk, inv = layer.permute(idx)
    out = layer.forward(x, wr)
    torch.cuda.synchronize()
    assert layer.status() == 0
    xu = oracle.as_u16(x)
    _, io, wo = oracle.route(xu, wr.cpu().numpy(), None, K)
    assert np.array_equal(idx.cpu().numpy(), io)
    assert np.max(np.abs(w.cpu().numpy() - wo)) < 1e-6
    for g, r in zip((counts, offsets, ps, pk, inv), oracle.permute(io, E)):
        assert np.array_equal(g.cpu().numpy().reshape(-1), np.asarray(r).reshape(-1))
    tok = np.array([0, 1, 4095, 40000, T - 2, T - 1])
    ref = oracle_layer_out(xu[tok], wr.cpu().numpy(), None, K, E, H, I, seed)
    assert_close_out(oracle.as_u16(out)[tok], ref, 2e-2)
    layer.close()


def test_widest_hidden_and_intermediate_past_2_pow_31_elements():
    _need_cuda()
    H, E, K, I, T, seed = 8192, 32, 32, 8192, 16384, 72
    layer, keep, wr = _layer(H, E, K, I, seed)
    x = synth.tokens(T, H, seed=seed, device="cuda")
    out = layer.forward(x, wr)
    torch.cuda.synchronize()
    assert layer.status() == 0
    tok = np.array([0, 9000, T - 1])
    ref = oracle_layer_out(oracle.as_u16(x)[tok], wr.cpu().numpy(), None, K, E, H, I, seed)
    assert_close_out(oracle.as_u16(out)[tok], ref, 2e-2)
    # the same last token alone: the same bits
    alone = layer.forward(x[T - 1:].contiguous(), wr)
    torch.cuda.synchronize()
    assert np.array_equal(oracle.as_u16(alone)[0], oracle.as_u16(out)[T - 1])
    layer.close()


@pytest.mark.parametrize("T", [8, 256])
def test_fp8_widest_hidden_and_intermediate(T):
    """FP8 at H = I = 8192: 64 scale blocks along each reduction, the most the
    FP8 kernels hold. At 256 tokens that is the separate GEMMs with the largest
    per-tile scale table (four stages); at 8 tokens the fused decode launch.
    Sampled tokens against the oracle (its own quantisation of the same bf16
    draws), first and last included."""
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    from helpers import LayerCase
    H, E, K, I, seed = 8192, 8, 2, 8192, 73
    case = LayerCase(T, H, E, K, I, seed=seed, wdtype=M.MOE_FP8_E4M3_B128)
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    tok = np.array(sorted({0, T // 2, T - 1}))
    ref = case.oracle_forward(tokens=tok)["out"]
    assert_close_out(oracle.as_u16(out)[tok], ref, 4e-2)
    case.close()
