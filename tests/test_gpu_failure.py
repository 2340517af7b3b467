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


# --------------------------------------------------- unregistered expert --

import numpy as np  # noqa: E402


def _oracle_without(case, missing):
    """Oracle output with every pair routed to `missing` dropped: each token's sum
    runs over its other pairs, k ascending (the missing expert is every token's
    top-1 here, so each token keeps K - 1 pairs)."""
    xu, wr, bias = case.oracle_inputs()
    _, idx, w = oracle.route(xu, wr, bias, case.K)
    keep = idx != missing
    assert np.all(keep.sum(axis=1) == case.K - 1)
    pt = np.nonzero(keep)[0].astype(np.int32)  # row-major: token, then k ascending
    pe = idx[keep]
    pw = w[keep].astype(np.float32)
    gu, dn, sgu, sdn = case.expert_arrays(np.unique(pe))
    if case.q is None:
        y = oracle.ffn_bf16(xu, pt, pe, pw, gu, dn, case.E)
    else:
        y = oracle.ffn_fp8(xu, pt, pe, pw, gu, sgu, dn, sdn, case.E)
    return oracle.combine(y, np.arange(case.T * (case.K - 1), dtype=np.int32).reshape(case.T, case.K - 1))


@pytest.mark.parametrize("T,wdtype,host", [(4, 0, False),     # decode: FFN planned inside the kernel
                                           (100, 0, False),   # one-launch permutation + plan
                                           (400, 0, False),   # rank/scan/scatter, then the plan kernel
                                           (8, 1, False),     # FP8, one-launch FFN
                                           (8, 0, True)])     # host-resident experts: host-side staging
def test_unregistered_expert_is_flagged_and_dropped(T, wdtype, host):
    """Routing to an expert that has no registered weights sets MOE_DEV_NO_SLOT
    and drops those pairs: each token's output is the oracle's sum over its
    other pairs. Registering the expert afterwards restores the full layer."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    H, E, K, I = 512, 16, 4, 256
    missing = 5
    hot = set(range(0, E, 2)) if host else None  # odd experts in pinned host memory
    case = LayerCase(T, H, E, K, I, seed=40 + T, wdtype=wdtype, unregistered=(missing,), hot=hot,
                     n_spare=8 if host else 0)
    bias = torch.zeros(E, dtype=torch.float32)
    bias[missing] = 64.0  # far above the logits' spread: every token's top-1
    case.bias = bias.to(case.dev)
    tol = 4e-2 if wdtype else 2e-2
    out = case.forward()
    torch.cuda.synchronize()
    st = case.layer.status()
    assert st & M.binding.MOE_DEV_NO_SLOT, st
    assert not st & M.binding.MOE_DEV_TIMEOUT
    assert_close_out(oracle.as_u16(out), _oracle_without(case, missing), tol)
    # register it: the same context now runs the whole layer
    g, d = case.w_gu[missing], case.w_dn[missing]
    if case.q is None:
        case.layer.register(missing, g, d)
    else:
        qg, sg, qd, sd = case.q[missing]
        case.layer.register(missing, qg, qd, sg, sd)
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    assert_close_out(oracle.as_u16(out), case.oracle_forward()["out"], tol)
    case.close()


def test_unregistered_expert_rows_are_zero_in_expert_ffn():
    """moe_expert_ffn on its own: the y_pair rows of pairs routed to an
    unregistered expert are written as zeros (the others match the oracle)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    H, E, K, I, T, missing = 512, 16, 4, 256, 300, 9
    case = LayerCase(T, H, E, K, I, seed=77, unregistered=(missing,))
    bias = torch.zeros(E, dtype=torch.float32)
    bias[missing] = 64.0
    case.bias = bias.to(case.dev)
    idx, w = case.layer.route(case.x, case.wr, case.bias)
    counts, offsets, ps, pk, inv = case.layer.permute(idx)
    y = case.layer.expert_ffn(case.x, ps, pk, offsets, w)
    torch.cuda.synchronize()
    assert case.layer.status() & M.binding.MOE_DEV_NO_SLOT
    off = offsets.cpu().numpy()
    yn = y.cpu().numpy()
    assert off[missing + 1] - off[missing] == T
    assert not np.any(yn[off[missing]:off[missing + 1]])
    # the other rows: the oracle's y for the same sorted pairs
    ps_n, pk_n, idx_n, w_n = ps.cpu().numpy(), pk.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()
    rows = np.r_[0:off[missing], off[missing + 1]:off[E]]
    pe = idx_n[ps_n[rows], pk_n[rows]]
    gu, dn, _, _ = case.expert_arrays(np.unique(pe))
    ref = oracle.ffn_bf16(oracle.as_u16(case.x), ps_n[rows], pe, w_n[ps_n[rows], pk_n[rows]], gu, dn, E)
    assert np.max(np.abs(yn[rows] - ref)) <= 2e-2 * np.max(np.abs(ref))
    case.close()


# ------------------------------------------------- failed allocations --

MOE_ERR_OOM = 6


def test_failed_allocations_return_oom_and_the_next_call_works():
    """Host-side fault injection (no GPU fault): each of the library's own
    allocations is made to fail in turn -- the context's device words, the slot
    table's device arrays, its spare slots and device LRU state, and its two
    pinned staging buffers. Each failing call returns MOE_ERR_OOM with what it
    had allocated released (a half-built MoeLayer releases its context too);
    with the hook disarmed the same calls succeed, and a layer with host-resident
    experts behind those spare slots then matches the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    H, E, K, I = 256, 8, 2, 512
    try:
        for skip in (0, 1):  # d_status, then d_counters
            M.moe_debug_fail_allocs(M.MOE_ALLOC_DEVICE, skip, 1)
            with pytest.raises(M.MoeError) as ei:
                M.moe_ctx_create(H, E, K, I)
            assert ei.value.status == MOE_ERR_OOM
        M.moe_debug_fail_allocs(M.MOE_ALLOC_ANY, 0, 0)
        ctx = M.moe_ctx_create(H, E, K, I)
        # slot table with 4 spare slots: device maps, slot index, spare slots, LRU state; pinned staging words
        # and LRU staging
        for kind, skip in ((M.MOE_ALLOC_DEVICE, 0), (M.MOE_ALLOC_DEVICE, 1), (M.MOE_ALLOC_DEVICE, 2),
                           (M.MOE_ALLOC_DEVICE, 3), (M.MOE_ALLOC_PINNED, 0), (M.MOE_ALLOC_PINNED, 1)):
            M.moe_debug_fail_allocs(kind, skip, 1)
            with pytest.raises(M.MoeError) as ei:
                M.moe_slots_create(ctx, 4)
            assert ei.value.status == MOE_ERR_OOM, (kind, skip)
            M.moe_debug_fail_allocs(M.MOE_ALLOC_ANY, 0, 0)
        slots = M.moe_slots_create(ctx, 4)
        M.moe_slots_destroy(slots)
        M.moe_ctx_destroy(ctx)
        # a layer whose slot table cannot get its pinned words: the constructor raises and keeps nothing
        M.moe_debug_fail_allocs(M.MOE_ALLOC_PINNED, 0, 1)
        with pytest.raises(M.MoeError) as ei:
            M.MoeLayer(H, E, K, I, n_spare_slots=4)
        assert ei.value.status == MOE_ERR_OOM
    finally:
        M.moe_debug_fail_allocs(M.MOE_ALLOC_ANY, 0, 0)
    case = LayerCase(16, H, E, K, I, seed=37, n_spare=4, hot={0, 1, 2, 3})
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    assert_close_out(oracle.as_u16(out), case.oracle_forward()["out"], 2e-2)
    case.close()


def test_failed_mxfp4_scale_allocation_then_registration_works():
    """MXFP4 registration allocates the experts' blocked scales; when that
    allocation fails the call returns MOE_ERR_OOM, and registering again
    succeeds with results identical to a layer that never saw the failure."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    import synth
    H, E, K, I, T = 256, 4, 2, 256, 8
    dev = torch.device("cuda")
    ws = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=41, device=dev)
        qg = torch.empty((2 * I, H // 2), dtype=torch.uint8, device=dev)
        sg = torch.empty((2 * I, H // 32), dtype=torch.uint8, device=dev)
        qd = torch.empty((H, I // 2), dtype=torch.uint8, device=dev)
        sd = torch.empty((H, I // 32), dtype=torch.uint8, device=dev)
        M.moe_quantize_mx(g, 2 * I, H, 0, qg, sg)
        M.moe_quantize_mx(d, H, I, 0, qd, sd)
        ws.append((qg, qd, sg, sd))
    x = synth.tokens(T, H, seed=41, device=dev)
    wr = synth.router_weight(E, H, seed=41, device=dev)
    outs = []
    for inject in (False, True):
        layer = M.MoeLayer(H, E, K, I, wdtype=M.MOE_MXFP4, device=dev)
        for e in range(E):
            if inject and e == 1:
                M.moe_debug_fail_allocs(M.MOE_ALLOC_DEVICE, 0, 1)
                try:
                    with pytest.raises(M.MoeError) as ei:
                        layer.register(e, *ws[e])
                    assert ei.value.status == MOE_ERR_OOM
                finally:
                    M.moe_debug_fail_allocs(M.MOE_ALLOC_ANY, 0, 0)
            layer.register(e, *ws[e])
        outs.append(oracle.as_u16(layer.forward(x, wr)))
        torch.cuda.synchronize()
        assert layer.status() == 0
        layer.close()
    assert np.array_equal(outs[0], outs[1])
