"""Spare slots as an LRU cache of host-resident experts (moe_slots_set_policy).

Every expert lives in pinned host memory and goes through a cache of spare
HBM slots smaller than the routed working set. Over a sequence of forwards
(different batches, new and repeated tokens) the outputs are bit-identical
to an all-resident layer over the same weights: the same kernels read the
same bytes (vLLM-Moet, topairepos.com page, hybrid results table, row
"identity"). A repeated batch finds every one of its experts in the cache and
copies nothing; a batch that routes more host experts than there are slots
takes the per-call staging path and still matches. Every call's output is
also checked against the CPU oracle (max|err| <= 2e-2 * max|ref| for bf16,
4e-2 for FP8), with the weights drawn and quantised on the host.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_out, oracle_layer_out

TOL = {0: 2e-2, 1: 4e-2}

pytestmark = pytest.mark.gpu

H, E, K, I = 512, 64, 4, 256
N_SLOTS = 12


def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _layers(wdtype, policy):
    import mixture_experts_layer_24_b200 as M
    dev = torch.device("cuda")
    ref = M.MoeLayer(H, E, K, I, wdtype=wdtype, device=dev)
    cache = M.MoeLayer(H, E, K, I, wdtype=wdtype, n_spare_slots=N_SLOTS, device=dev)
    M.moe_slots_set_policy(cache.slots, policy)
    keep = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=5, device=dev)
        if wdtype == M.MOE_FP8_E4M3_B128:
            qg = torch.empty((2 * I, H), dtype=torch.uint8, device=dev)
            sg = torch.empty((2 * I // 128, H // 128), dtype=torch.float32, device=dev)
            qd = torch.empty((H, I), dtype=torch.uint8, device=dev)
            sd = torch.empty((H // 128, I // 128), dtype=torch.float32, device=dev)
            M.moe_quantize_e4m3(g, 2 * I, H, 128, qg, sg)
            M.moe_quantize_e4m3(d, H, I, 128, qd, sd)
            torch.cuda.synchronize()
            w = (qg, qd, sg, sd)
        else:
            w = (g, d, None, None)
        ref.register(e, *w, M.MOE_LOC_HBM)
        hw = tuple(None if t is None else t.cpu().pin_memory() for t in w)
        cache.register(e, *hw, M.MOE_LOC_HOST_PINNED)
        keep.append((w, hw))
    wr = synth.router_weight(E, H, seed=5, device=dev)
    # no logit prior: at this width the Zipf prior would send every token to the same few experts, and the
    # sequence must outgrow the cache (evictions, and one call with more routed experts than slots)
    bias = None
    return ref, cache, wr, bias, keep


# batch sizes and first tokens of the sequence: call 2 repeats call 1 (its experts are the most recently used,
# so all of them are cached), call 5 routes more host experts than there are slots (per-call staging)
SEQUENCE = [(1, 100), (2, 200), (2, 200), (3, 400), (1, 100), (16, 500), (2, 600), (1, 700)]
REPEAT = 2


@pytest.mark.parametrize("wdtype", [0, 1])
def test_lru_cache_bit_identical_and_hits(wdtype):
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    ref, cache, wr, bias, keep = _layers(wdtype, M.MOE_SLOTS_LRU)
    dev = torch.device("cuda")
    total_hits = 0
    for i, (T, first) in enumerate(SEQUENCE):
        x = synth.tokens(T, H, seed=5, device=dev, first_token=first)
        a = ref.forward(x, wr, bias)
        b = cache.forward(x, wr, bias)
        torch.cuda.synchronize()
        assert cache.status() == 0 and ref.status() == 0
        assert np.array_equal(oracle.as_u16(a), oracle.as_u16(b)), f"call {i} (T={T}) differs"
        ref_o = oracle_layer_out(oracle.as_u16(x), wr.cpu().numpy(), None, K, E, H, I, seed=5, fp8=wdtype == 1)
        assert_close_out(oracle.as_u16(b), ref_o, TOL[wdtype])
        st = cache.stats()
        assert st["last_routed_cold"] == st["last_touched"]  # every expert lives on the host
        if st["last_routed_cold"] <= N_SLOTS:
            assert st["last_hits"] + st["last_cold"] == st["last_routed_cold"]
        total_hits += st["last_hits"]
        if i == REPEAT:
            assert st["last_cold"] == 0 and st["last_hits"] == st["last_routed_cold"], st
    st = cache.stats()
    assert st["cache_hits"] == total_hits > 0
    assert st["cold_staged"] > N_SLOTS  # the working set outgrew the cache: slots were evicted and refilled
    ref.close()
    cache.close()


def test_per_call_policy_matches_and_never_hits():
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    ref, cache, wr, bias, keep = _layers(0, M.MOE_SLOTS_PER_CALL)
    dev = torch.device("cuda")
    for T, first in SEQUENCE[:4]:
        x = synth.tokens(T, H, seed=5, device=dev, first_token=first)
        a = ref.forward(x, wr, bias)
        b = cache.forward(x, wr, bias)
        torch.cuda.synchronize()
        assert np.array_equal(oracle.as_u16(a), oracle.as_u16(b))
        st = cache.stats()
        assert st["last_hits"] == 0 and st["last_cold"] == st["last_routed_cold"]
    ref.close()
    cache.close()


def test_reregistering_an_expert_drops_its_cached_copy():
    """A cached expert re-registered with other weights must not be served from the stale slot."""
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    ref, cache, wr, bias, keep = _layers(0, M.MOE_SLOTS_LRU)
    dev = torch.device("cuda")
    x = synth.tokens(1, H, seed=5, device=dev, first_token=100)
    cache.forward(x, wr, bias)
    idx, _ = ref.route(x, wr, bias)
    e = int(idx[0, 0].item())
    # swap expert e's weights for another expert's in both layers
    (w_other, hw_other) = keep[(e + 1) % E]
    ref.register(e, *w_other, M.MOE_LOC_HBM)
    cache.register(e, *hw_other, M.MOE_LOC_HOST_PINNED)
    a = ref.forward(x, wr, bias)
    b = cache.forward(x, wr, bias)
    torch.cuda.synchronize()
    assert np.array_equal(oracle.as_u16(a), oracle.as_u16(b))
    assert cache.stats()["last_cold"] >= 1  # e was copied again
    ref.close()
    cache.close()


@pytest.mark.parametrize("wdtype", [0, 1])
def test_device_side_cache_in_a_cuda_graph(wdtype):
    """Decode batches whose pairs fit in the spare slots keep the whole cache
    bookkeeping on the device (plan, copies of the missed experts, FFN), so the
    forward can be captured once and replayed: over replays with new tokens the
    cache fills, hits and evicts inside the graph, and every output equals the
    all-resident layer's bits and the oracle within 2e-2 (bf16) or 4e-2 (FP8:
    the cached records include the weight block scales)."""
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    ref, cache, wr, bias, keep = _layers(wdtype, M.MOE_SLOTS_LRU)
    dev = torch.device("cuda")
    T = 2  # 8 pairs <= 12 slots: the device-side path
    x = synth.tokens(T, H, seed=5, device=dev, first_token=9000)
    g, out = cache.capture(x, wr, bias)
    seen_hits = 0
    for i, first in enumerate([9000, 9100, 9000, 9200, 9300, 9100, 9400, 9000]):
        x.copy_(synth.tokens(T, H, seed=5, device=dev, first_token=first))
        g.replay()
        a = ref.forward(x, wr, bias)
        torch.cuda.synchronize()
        assert cache.status() == 0 and ref.status() == 0
        got = oracle.as_u16(out)
        assert np.array_equal(got, oracle.as_u16(a)), f"replay {i} differs"
        assert_close_out(got, oracle_layer_out(oracle.as_u16(x), wr.cpu().numpy(), None, K, E, H, I, seed=5,
                                               fp8=wdtype == 1), TOL[wdtype])
        st = cache.stats()
        assert st["last_hits"] + st["last_cold"] == st["last_routed_cold"]
        seen_hits += st["last_hits"]
    assert seen_hits > 0
    assert cache.stats()["cold_staged"] > N_SLOTS  # the graph's own copies refilled evicted slots
    ref.close()
    cache.close()
