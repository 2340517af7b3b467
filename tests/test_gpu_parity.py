"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Integer outputs (top-k indices, counts, offsets, the permutation, FP8 codes
and scales, the combine's bf16 bits on shared inputs) must match bit for bit.
Floating-point layer outputs must satisfy max|err| <= 2e-2 * max|ref| (bf16
weights) or 4e-2 (FP8 weights); routing weights within 1e-6.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import LayerCase, assert_close_out, f32_of_bf16_bits

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")
TOL_BF16 = 2e-2
TOL_FP8 = 4e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    M.lib()  # fail loudly if libmoe.so is missing
    yield


def M():
    import mixture_experts_layer_24_b200 as m
    return m


# ------------------------------------------------------------------ route --

@pytest.mark.parametrize("T,H,E,K,zipf", [(16, 256, 8, 2, None), (1, 4096, 384, 8, 1.1), (3, 4096, 384, 8, 1.1),
                                          (64, 4096, 384, 8, 1.1), (300, 1024, 64, 6, None),
                                          (1000, 512, 100, 4, 1.1), (333, 1024, 40, 8, None),
                                          (2049, 4096, 384, 8, 1.1)])
def test_route_matches_oracle(T, H, E, K, zipf):
    dev = torch.device("cuda")
    x = synth.tokens(T, H, seed=1, device=dev)
    wr = synth.router_weight(E, H, seed=1, device=dev)
    bias = None if zipf is None else synth.zipf_logit_bias(E, zipf, seed=1).to(dev)
    layer = M().MoeLayer(H, E, K, 256)
    idx, w = layer.route(x, wr, bias)
    torch.cuda.synchronize()
    lo, io, wo = oracle.route(oracle.as_u16(x), wr.cpu().numpy(), None if bias is None else bias.cpu().numpy(), K)
    assert np.array_equal(idx.cpu().numpy(), io)
    assert np.max(np.abs(w.cpu().numpy().astype(np.float64) - wo)) < 1e-6
    assert layer.status() == 0
    layer.close()


def test_route_reduction_order_decides_topk():
    """Golden logit cases: under the specified order expert 0's logit is the
    case's expected value; expert 1 sits between the specified and the naive
    sequential result, so top-1 tells which order the kernel used."""
    cases = json.load(open(os.path.join(GOLD, "order_cases.json")))["logit_cases"]
    dev = torch.device("cuda")
    for c in cases:
        H = c["H"]
        x = torch.zeros((1, H), dtype=torch.float32)
        wr = torch.zeros((3, H), dtype=torch.float32)
        for h, xv, wv in c["terms"]:
            x[0, h] = xv
            wr[0, h] = wv
        seq = np.float32(0)
        for h, xv, wv in c["terms"]:
            seq = np.float32(np.float64(seq) + np.float64(np.float32(xv)) * np.float64(np.float32(wv)))
        exp = np.float32(c["expected"])
        x[0, 200 % H] += 0.0
        mid = (float(exp) + float(seq)) / 2 if float(seq) != float(exp) else float(exp) - 1e-3
        wr[1, H - 1] = mid
        x[0, H - 1] = 1.0
        layer = M().MoeLayer(H, 3, 1, 128)
        idx, w = layer.route(x.to(torch.bfloat16).to(dev), wr.to(dev))
        io = oracle.route(oracle.as_u16(x.to(torch.bfloat16)), wr.numpy(), None, 1)[1]
        assert idx.cpu().numpy()[0, 0] == io[0, 0], c["why"]
        layer.close()


@pytest.mark.parametrize("T", [1, 5, 13, 40, 64, 65, 200, 333])
def test_route_reduction_order_every_router_kernel(T):
    """The golden order cases again, side by side in one batch, so that every
    router kernel (one-launch small batches, the register-tiled decode tiles,
    the token-pair prefill tile) meets them, with the cases of neighbouring
    tokens different and ragged token and expert tiles. Case c lives in h block
    [256c, 256c + 256) (a multiple of 32, so its lanes and in-lane order are
    unchanged); expert 2c holds its weights, expert 2c+1 the midpoint between
    the specified and the sequential sum, read through x[256c + 255] = 1."""
    cases = json.load(open(os.path.join(GOLD, "order_cases.json")))["logit_cases"]
    n = len(cases)
    H, E = 256 * n, 2 * n + 4  # four all-zero experts make the expert tiles ragged
    x = torch.zeros((T, H), dtype=torch.float32)
    wr = torch.zeros((E, H), dtype=torch.float32)
    for c, case in enumerate(cases):
        base = 256 * c
        seq = np.float32(0)
        for h, xv, wv in case["terms"]:
            assert h < 255
            wr[2 * c, base + h] = wv
            seq = np.float32(np.float64(seq) + np.float64(np.float32(xv)) * np.float64(np.float32(wv)))
        exp = np.float32(case["expected"])
        wr[2 * c + 1, base + 255] = (float(exp) + float(seq)) / 2 if float(seq) != float(exp) else float(exp) - 1e-3
    for t in range(T):
        c = (3 * t + 1) % n
        for h, xv, wv in cases[c]["terms"]:
            x[t, 256 * c + h] = xv
        x[t, 256 * c + 255] = 1.0
    xb = x.to(torch.bfloat16)
    layer = M().MoeLayer(H, E, 1, 128)
    idx, w = layer.route(xb.to(torch.device("cuda")), wr.to(torch.device("cuda")))
    torch.cuda.synchronize()
    io = oracle.route(oracle.as_u16(xb), wr.numpy(), None, 1)[1]
    assert np.array_equal(idx.cpu().numpy(), io)
    assert layer.status() == 0
    layer.close()


def test_route_ties_go_to_lower_index():
    dev = torch.device("cuda")
    H, E, K = 256, 40, 8
    x = torch.zeros((4, H), dtype=torch.bfloat16, device=dev)
    x[:, 0] = 1.0
    wr = torch.zeros((E, H), dtype=torch.float32, device=dev)
    wr[:, 0] = torch.tensor([(e % 5) * 0.5 for e in range(E)], dtype=torch.float32)
    wr[3, 0] = -0.0
    layer = M().MoeLayer(H, E, K, 128)
    idx, w = layer.route(x, wr)
    io = oracle.route(oracle.as_u16(x), wr.cpu().numpy(), None, K)[1]
    assert np.array_equal(idx.cpu().numpy(), io)
    layer.close()


@pytest.mark.parametrize("T", [1, 3, 8, 16, 40])
def test_ties_through_the_decode_forward(T):
    """Tied logits through the decode forward (the router's fused last-CTA
    top-k up to 4 tokens, the warp top-k kernel above): router rows repeat
    with period 13, so experts e, e+13, e+26 (and 39) tie, and the top-8
    boundary cuts through a tied group. The lower index wins and goes first,
    as in the oracle; a wrong pick brings another expert's FFN into the
    output, a wrong order changes the bits of the k-ordered sum."""
    H, E, K, I = 256, 40, 8, 128
    case = LayerCase(T, H, E, K, I, seed=7 + T)
    case.wr = case.wr[torch.arange(E, device=case.dev) % 13].contiguous()
    out = oracle.as_u16(case.forward())
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    ref = case.oracle_forward()
    lo = np.sort(oracle.route(*case.oracle_inputs(), K)[0], axis=1)[:, ::-1]
    assert np.all(lo[:, K - 1] == lo[:, K]), "the top-8 boundary cuts through a tied group"
    idx, _ = case.layer.route(case.x, case.wr, case.bias)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    assert_close_out(out, ref["out"], TOL_BF16)
    # the same tokens inside a 200-token batch (router GEMM + top-k kernel): the same bits
    xb = torch.cat([case.x, synth.tokens(200 - T, H, seed=99, device=case.dev)]).contiguous()
    assert np.array_equal(oracle.as_u16(case.layer.forward(xb, case.wr, case.bias))[:T], out)
    case.close()


# ---------------------------------------------------------------- permute --

@pytest.mark.parametrize("T,E,K,mode", [(1, 384, 8, "rand"), (17, 8, 2, "rand"), (4096, 384, 8, "zipf"),
                                        (5000, 384, 8, "hot"), (333, 7, 7, "rand"), (64, 1024, 32, "rand"),
                                        (2048, 16, 3, "rand")])
def test_permute_bit_exact(T, E, K, mode):
    rng = np.random.default_rng(T + E + K)
    if mode == "hot":  # every token on the same K experts
        idx = np.tile(np.arange(K, dtype=np.int32), (T, 1))
    elif mode == "zipf":
        p = np.arange(1, E + 1, dtype=np.float64) ** -1.1
        p /= p.sum()
        idx = np.stack([rng.choice(E, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    else:
        idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    layer = M().MoeLayer(256, E, K, 128)
    got = layer.permute(torch.from_numpy(idx).cuda())
    ref = oracle.permute(idx, E)
    for g, r in zip(got, ref):
        assert np.array_equal(g.cpu().numpy().reshape(-1), np.asarray(r).reshape(-1))
    assert layer.status() == 0
    layer.close()


def test_permute_flags_bad_expert():
    idx = np.array([[0, 1], [2, 99], [1, 0]], dtype=np.int32)
    layer = M().MoeLayer(256, 4, 2, 128)
    counts, offsets, ps, pk, inv = layer.permute(torch.from_numpy(idx).cuda())
    assert layer.status() & M().binding.MOE_DEV_BAD_EXPERT
    assert inv.cpu().numpy()[1, 1] == -1
    assert int(offsets[-1]) == 5
    layer.close()


# ---------------------------------------------------------- combine/quant --

@pytest.mark.parametrize("T,K,H", [(1, 1, 128), (7, 8, 4096), (300, 2, 256), (64, 32, 512)])
def test_combine_bit_exact(T, K, H):
    y = synth.normal_f32((T * K, H), 3, synth.TID_YPAIR)
    inv = torch.from_numpy(np.random.default_rng(T).permutation(T * K).astype(np.int32).reshape(T, K))
    layer = M().MoeLayer(H, max(K, 2), K, 128)
    out = layer.combine(y.cuda(), inv.cuda())
    ref = oracle.combine(y.numpy(), inv.numpy())
    assert np.array_equal(oracle.as_u16(out), ref)
    layer.close()


@pytest.mark.parametrize("rows,cols,br", [(1, 128, 1), (33, 4096, 1), (256, 384, 128), (300, 512, 128),
                                          (4096, 2048, 128)])
def test_quantizer_bit_exact(rows, cols, br):
    src = synth.normal((rows, cols), 4, 77, 0.02, torch.bfloat16, "cuda")
    src[0, :128] = 0
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty(((rows + br - 1) // br, cols // 128), dtype=torch.float32, device="cuda")
    M().moe_quantize_e4m3(src, rows, cols, br, q, s)
    qo, so = oracle.quant_e4m3(oracle.as_u16(src), br)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy(), so)


# ------------------------------------------------------------- expert FFN --

@pytest.mark.parametrize("T,H,E,K,I", [(16, 256, 8, 2, 512), (5, 512, 4, 2, 256), (200, 256, 6, 3, 384),
                                       (700, 384, 12, 4, 256), (40, 1024, 16, 8, 512)])
def test_forward_small_bf16(T, H, E, K, I):
    case = LayerCase(T, H, E, K, I, seed=T)
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    ref = case.oracle_forward()
    assert_close_out(oracle.as_u16(out), ref["out"], TOL_BF16)
    case.close()


@pytest.mark.parametrize("wdtype", [0, 1])
@pytest.mark.parametrize("T,H,E,K,I,mode", [(33, 256, 4, 4, 256, "k_eq_e"),    # every token on every expert
                                            (300, 256, 8, 2, 256, "one_pair"),  # all tokens on experts 5 and 2
                                            (7, 512, 1, 1, 384, "single"),      # one expert, top-1
                                            (129, 384, 6, 1, 256, "one_pair")])
def test_forward_routing_edge_cases(T, H, E, K, I, mode, wdtype):
    """Routing extremes through the whole forward: K = E; every token on the
    same experts (the others get no rows; 300 rows is not a multiple of any
    tile width); a single expert with top-1 (the layer is one dense SwiGLU FFN
    scaled by weight 1)."""
    case = LayerCase(T, H, E, K, I, seed=T + E, wdtype=wdtype)
    if mode == "one_pair":  # a logit prior far above the logits' spread
        bias = torch.zeros(E, dtype=torch.float32)
        bias[5 % E] = 64.0
        bias[2 % E] = 32.0
        case.bias = bias.to(case.dev)
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    ref = case.oracle_forward()
    if mode == "one_pair":
        assert set(np.unique(ref["idx"]).tolist()) <= {5 % E, 2 % E}
    assert_close_out(oracle.as_u16(out), ref["out"], TOL_FP8 if wdtype else TOL_BF16)
    idx, _ = case.layer.route(case.x, case.wr, case.bias)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    case.close()


def test_expert_ffn_y_pair_bf16():
    T, H, E, K, I = 48, 512, 8, 2, 256
    case = LayerCase(T, H, E, K, I, seed=5)
    idx, w = case.layer.route(case.x, case.wr)
    counts, offsets, ps, pk, inv = case.layer.permute(idx)
    y = case.layer.expert_ffn(case.x, ps, pk, offsets, w)
    torch.cuda.synchronize()
    ps_n, pk_n = ps.cpu().numpy(), pk.cpu().numpy()
    idx_n, w_n = idx.cpu().numpy(), w.cpu().numpy()
    pe = idx_n[ps_n, pk_n]
    pw = w_n[ps_n, pk_n]
    gu, dn, _, _ = case.expert_arrays(range(E))
    ref = oracle.ffn_bf16(oracle.as_u16(case.x), ps_n, pe, pw, gu, dn, E)
    got = y.cpu().numpy()
    assert np.max(np.abs(got - ref)) <= TOL_BF16 * np.max(np.abs(ref))
    assert np.sqrt(np.mean((got - ref) ** 2)) <= 2e-3 * np.sqrt(np.mean(ref ** 2))
    case.close()


@pytest.mark.parametrize("T,H,E,K,I", [(16, 256, 8, 2, 512), (100, 512, 8, 4, 384), (600, 256, 10, 2, 256)])
def test_forward_small_fp8(T, H, E, K, I):
    case = LayerCase(T, H, E, K, I, seed=T + 1, wdtype=1)
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    ref = case.oracle_forward()
    assert_close_out(oracle.as_u16(out), ref["out"], TOL_FP8)
    case.close()


# --------------------------------------------------------- invariance ----

def test_batch_invariance_small():
    H, E, K, I = 512, 16, 4, 256
    big = LayerCase(300, H, E, K, I, seed=9)
    full = oracle.as_u16(big.forward())
    for T in (1, 2, 4, 8, 16, 17, 64, 129):
        x = big.x[:T].contiguous()
        out = oracle.as_u16(big.layer.forward(x, big.wr, big.bias))
        assert np.array_equal(out, full[:T]), T
    big.close()


def test_empty_batch_is_a_no_op():
    case = LayerCase(4, 256, 8, 2, 256, seed=2)
    out = torch.full((0, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    case.layer.forward(case.x[:0], case.wr, None, out=out)
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    case.close()


@pytest.mark.parametrize("T,wdtype", [(1, 0), (8, 0), (64, 0), (100, 0), (8, 1), (64, 1)])
def test_graph_replay_matches_eager(T, wdtype):
    """A forward captured in a CUDA graph (kernels chained by programmatic
    dependent launch) gives the eager bits, replay after replay, and the
    oracle's output within tolerance. T = 1 .. 64 (bf16) are the decode
    batches that run planned from the router's top-k in one FFN launch (the
    launches bench.py replays); 100 tokens take the permutation and separate
    GEMMs; FP8 8 tokens take the one-launch FP8 FFN, 64 the separate ones."""
    case = LayerCase(T, 512, 16, 4, 256, seed=12, wdtype=wdtype)
    tol = TOL_FP8 if wdtype else TOL_BF16
    ref = oracle.as_u16(case.forward())
    assert_close_out(ref, case.oracle_forward()["out"], tol)
    g, out = case.layer.capture(case.x, case.wr, case.bias)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(oracle.as_u16(out), ref)
    # new input contents, same buffer
    case.x.copy_(synth.tokens(T, 512, seed=13, device="cuda"))
    g.replay()
    torch.cuda.synchronize()
    got = oracle.as_u16(out)
    assert np.array_equal(got, oracle.as_u16(case.forward()))
    assert_close_out(got, case.oracle_forward()["out"], tol)
    assert case.layer.status() == 0
    case.close()


@pytest.mark.parametrize("T", [1, 5, 64, 65, 129])
def test_small_and_large_paths_agree(T):
    """Batches around the decode/prefill switch of the router (64 tokens) and of
    the single-launch permutation (1024 pairs) give the oracle's routing and
    the same bits as the same tokens inside a bigger batch."""
    H, E, K, I = 1024, 64, 8, 256
    big = LayerCase(160, H, E, K, I, seed=31, zipf=1.1)
    ref = oracle.as_u16(big.forward())
    x = big.x[:T].contiguous()
    idx, w = big.layer.route(x, big.wr, big.bias)
    _, io, wo = oracle.route(oracle.as_u16(x), big.wr.cpu().numpy(), big.bias.cpu().numpy(), K)
    assert np.array_equal(idx.cpu().numpy(), io)
    assert np.max(np.abs(w.cpu().numpy() - wo)) < 1e-6
    got = big.layer.permute(idx)
    for g, r in zip(got, oracle.permute(io, E)):
        assert np.array_equal(g.cpu().numpy().reshape(-1), np.asarray(r).reshape(-1))
    out = oracle.as_u16(big.layer.forward(x, big.wr, big.bias))
    assert np.array_equal(out, ref[:T])
    big.close()
