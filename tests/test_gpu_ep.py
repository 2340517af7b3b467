"""Expert parallelism on one GPU: G ranks as threads of one process, each with
its own libmoe contexts (all E experts for routing and combine, its E/G
experts for the FFN), exchanging rows through the host (``ep.LocalComm``:
nothing on the device waits for another rank). Each rank's output must equal
the single-GPU forward of the same tokens bit for bit, and the oracle within
tolerance; the NCCL exchange of a multi-GPU run moves the same rows."""

import threading

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


def _run_ranks(world, make_steps, xs, wr, bias):
    from mixture_experts_layer_24_b200 import ep
    comms = ep.LocalComm.group(world)
    outs, errs = {}, []
    steps = [make_steps(r) for r in range(world)]

    def run(r):
        try:
            torch.cuda.set_device(0)
            outs[r] = ep.ep_forward(steps[r], comms[r], xs[r], wr, bias)
            torch.cuda.synchronize()
        except Exception as exc:  # surfaced below
            errs.append(exc)
            comms[r].shared.barrier.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=600)
    assert not errs, errs
    status = [s.status() for s in steps]
    for s in steps:
        s.close()
    return outs, status


@pytest.mark.parametrize("world,wdtype", [(2, 0), (4, 0), (3, 0), (4, 1), (2, 2)])
def test_ep_ranks_match_single_gpu_small(world, wdtype):
    """bf16 (0), FP8 (1) and MXFP4 (2) experts split over `world` ranks. MXFP4
    is checked bit for bit against the single-GPU MXFP4 forward, which
    tests/test_gpu_mxfp4.py checks against the oracle."""
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    from mixture_experts_layer_24_b200 import ep
    H, E, K, I = 512, 48, 4, 256
    dev = torch.device("cuda", 0)
    wr = synth.router_weight(E, H, seed=61, device=dev)
    bias = synth.zipf_logit_bias(E, 1.1, seed=61).to(dev)
    ws = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=61, device=dev)
        if wdtype == 2:
            qg = torch.empty((2 * I, H // 2), dtype=torch.uint8, device=dev)
            sg = torch.empty((2 * I, H // 32), dtype=torch.uint8, device=dev)
            qd = torch.empty((H, I // 2), dtype=torch.uint8, device=dev)
            sd = torch.empty((H, I // 32), dtype=torch.uint8, device=dev)
            M.moe_quantize_mx(g, 2 * I, H, 0, qg, sg)
            M.moe_quantize_mx(d, H, I, 0, qd, sd)
            ws.append((qg, qd, sg, sd))
        elif wdtype == 1:
            qg = torch.empty((2 * I, H), dtype=torch.uint8, device=dev)
            sg = torch.empty((2 * I // 128, H // 128), dtype=torch.float32, device=dev)
            qd = torch.empty((H, I), dtype=torch.uint8, device=dev)
            sd = torch.empty((H // 128, I // 128), dtype=torch.float32, device=dev)
            M.moe_quantize_e4m3(g, 2 * I, H, 128, qg, sg)
            M.moe_quantize_e4m3(d, H, I, 128, qd, sd)
            ws.append((qg, qd, sg, sd))
        else:
            ws.append((g, d, None, None))
    torch.cuda.synchronize()
    single = M.MoeLayer(H, E, K, I, wdtype=wdtype, device=dev)
    for e in range(E):
        single.register(e, *ws[e])
    T_of = [1, 9, 70, 300][:world] if world <= 4 else None
    xs = [synth.tokens(T_of[r], H, seed=61, device=dev, first_token=5000 * r) for r in range(world)]

    def make_steps(r):
        st = ep.LibmoeSteps(H, E, K, I, r, world, wdtype=wdtype, device=dev)
        for e in range(st.e0, st.e0 + st.E_loc):
            st.register(e, *ws[e])
        return st

    outs, status = _run_ranks(world, make_steps, xs, wr, bias)
    assert all(s == 0 for s in status), status
    for r in range(world):
        ref = single.forward(xs[r], wr, bias)
        torch.cuda.synchronize()
        got = oracle.as_u16(outs[r])
        assert np.array_equal(got, oracle.as_u16(ref)), f"rank {r} of {world}"
        if wdtype == 2:
            continue
        tok = np.unique([0, T_of[r] // 2, T_of[r] - 1])
        ref_o = oracle_layer_out(oracle.as_u16(xs[r])[tok], wr.cpu().numpy(), bias.cpu().numpy(), K, E, H, I,
                                 seed=61, fp8=wdtype == 1)
        assert_close_out(got[tok], ref_o, 4e-2 if wdtype else 2e-2)
    single.close()


def test_ep_full_size_four_ranks():
    """The 384-expert layer over 4 ranks (96 experts each, weights shared on the
    one GPU): decode batches 1 and 8 and a 512-token chunk per rank, bit for
    bit against the single-GPU forward of the same tokens."""
    _need_cuda()
    import mixture_experts_layer_24_b200 as M
    from mixture_experts_layer_24_b200 import ep
    H, E, K, I, world = 4096, 384, 8, 2048, 4
    dev = torch.device("cuda", 0)
    wr = synth.router_weight(E, H, seed=0, device=dev)
    bias = synth.zipf_logit_bias(E, 1.1, seed=0).to(dev)
    single = M.MoeLayer(H, E, K, I, device=dev)
    ws = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=0, device=dev)
        single.register(e, g, d)
        ws.append((g, d))
    torch.cuda.synchronize()
    T_of = [1, 8, 512, 64]
    xs = [synth.tokens(T_of[r], H, seed=0, device=dev, first_token=70000 + 5000 * r) for r in range(world)]

    def make_steps(r):
        st = ep.LibmoeSteps(H, E, K, I, r, world, device=dev)
        for e in range(st.e0, st.e0 + st.E_loc):
            st.register(e, *ws[e])
        return st

    outs, status = _run_ranks(world, make_steps, xs, wr, bias)
    assert all(s == 0 for s in status), status
    for r in range(world):
        ref = single.forward(xs[r], wr, bias)
        torch.cuda.synchronize()
        assert np.array_equal(oracle.as_u16(outs[r]), oracle.as_u16(ref)), f"rank {r}"
    single.close()
