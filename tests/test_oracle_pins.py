"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks one part of the oracle against a hand-derived value, a
closed form, an invariant, an independent library routine (numpy float64
matmul, numpy stable sort, torch's float8 cast), or brute force on tiny inputs,
so that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
U = 2.0 ** -24  # fp32 unit roundoff


def bf16_round_np(a: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bf16 -> float64 through torch (independent of the oracle)."""
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def f32(u16):
    return oracle.bf16_bits_to_f32(u16).astype(np.float64)


def silu64(g):
    return g / (1.0 + np.exp(-g))


# ------------------------------------------------------------------ logits --

def test_logits_within_fp32_error_bound_of_float64_matmul():
    T, H, E = 5, 1024, 24
    x = synth.tokens(T, H, seed=3)
    wr = synth.router_weight(E, H, seed=3).numpy()
    bias = synth.zipf_logit_bias(E, seed=3).numpy()
    xu = oracle.as_u16(x)
    xf = x.to(torch.float64).numpy()
    for b in (None, bias):
        l32 = oracle.router_logits(xu, wr, b).astype(np.float64)
        l64 = xf @ wr.astype(np.float64).T
        absdot = np.abs(xf) @ np.abs(wr.astype(np.float64)).T
        n = H // 32 + 5 + 1  # per-lane fma chain + 5 tree levels (+1 slack)
        gamma = n * U / (1 - n * U)
        bound = gamma * absdot
        if b is not None:
            l64 = l64 + b.astype(np.float64)[None, :]
            bound = bound + U * np.abs(l64) * 2
        err = np.abs(l32 - l64)
        assert np.all(err <= bound + 1e-30), float((err - bound).max())
        # and far from trivially loose: a transposed / shifted operand is way off
        assert np.max(np.abs(l64)) > 100 * np.max(bound)


def test_logit_reduction_order_golden_cases():
    cases = json.load(open(os.path.join(GOLD, "order_cases.json")))["logit_cases"]
    for c in cases:
        H = c["H"]
        x = np.zeros((1, H), np.float32)
        w = np.zeros((1, H), np.float32)
        for h, xv, wv in c["terms"]:
            x[0, h] = xv
            w[0, h] = wv
        xu = oracle.as_u16(torch.from_numpy(x).to(torch.bfloat16))
        assert np.array_equal(f32(xu), x.astype(np.float64)), "case inputs must be exact in bf16"
        got = oracle.router_logits(xu, w)[0, 0]
        assert np.float32(got) == np.float32(c["expected"]), (c["why"], got)


def test_logit_bias_is_one_fp32_add():
    H, E = 256, 4
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    w = np.zeros((E, H), np.float32)
    w[:, 0] = [1.0, 2.0, 16777216.0, -3.0]
    bias = np.array([0.5, -2.0, 1.0, 3.0], np.float32)
    xu = oracle.as_u16(torch.from_numpy(x).to(torch.bfloat16))
    got = oracle.router_logits(xu, w, bias)[0]
    # hand: 1.5, 0, 2^24+1 -> 2^24 (tie to even), 0
    assert got.tolist() == [1.5, 0.0, 16777216.0, 0.0]


# ------------------------------------------------------------------- top-k --

def test_topk_equals_full_stable_sort_with_ties():
    rng = np.random.default_rng(0)
    T, E = 64, 40
    logits = rng.integers(-3, 4, size=(T, E)).astype(np.float32) * 0.25  # many exact ties
    for K in (1, 2, 5, 8, E):
        idx, w = oracle.topk(logits, K)
        for t in range(T):
            order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))  # logit desc, e asc
            assert idx[t].tolist() == order[:K].tolist()


def test_topk_signed_zero_is_a_tie():
    logits = np.array([[-0.0, 0.0, -1.0, 0.0]], np.float32)
    idx, _ = oracle.topk(logits, 3)
    assert idx[0].tolist() == [0, 1, 3]


def test_topk_all_equal_gives_lowest_indices_and_uniform_weights():
    logits = np.full((2, 12), 0.75, np.float32)
    idx, w = oracle.topk(logits, 4)
    assert idx.tolist() == [[0, 1, 2, 3]] * 2
    assert np.all(w == 0.25)


def test_weights_are_full_softmax_renormalised_over_topk():
    T, H, E, K = 6, 256, 32, 8
    x = synth.tokens(T, H, seed=5)
    wr = synth.router_weight(E, H, seed=5).numpy() * 10  # spread the logits
    logits, idx, w = oracle.route(oracle.as_u16(x), wr, None, K)
    l = logits.astype(np.float64)
    full = np.exp(l - l.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)  # softmax over all E experts
    sel = np.take_along_axis(full, idx.astype(np.int64), 1)
    ref = sel / sel.sum(1, keepdims=True)
    assert np.max(np.abs(w - ref)) < 1e-12
    assert np.max(np.abs(w.sum(1) - 1.0)) < 1e-12
    assert np.all(np.diff(w, axis=1) <= 0)  # ordered by logit descending
    _, w1 = oracle.topk(logits, 1)
    assert np.all(w1 == 1.0)


# ------------------------------------------------------------- permutation --

def test_permutation_against_numpy_stable_sort():
    rng = np.random.default_rng(1)
    for T, K, E in ((1, 1, 1), (7, 2, 8), (100, 8, 384), (33, 4, 5)):
        idx = np.stack([rng.choice(E, size=K, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm_src, perm_k, inv = oracle.permute(idx, E)
        flat_e = idx.reshape(-1).astype(np.int64)
        flat_t = np.repeat(np.arange(T), K)
        flat_k = np.tile(np.arange(K), T)
        order = np.argsort(flat_e * T + flat_t, kind="stable")
        assert np.array_equal(perm_src, flat_t[order])
        assert np.array_equal(perm_k, flat_k[order])
        assert np.array_equal(counts, np.bincount(flat_e, minlength=E))
        assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts) and offsets[-1] == T * K
        # permute then unpermute is the identity
        assert np.array_equal(perm_src[inv.reshape(-1)], flat_t)
        assert np.array_equal(perm_k[inv.reshape(-1)], flat_k)
        assert np.array_equal(np.sort(inv.reshape(-1)), np.arange(T * K))


# --------------------------------------------------------------------- FFN --

def _experts(E, H, I, seed):
    gu, dn = {}, {}
    for e in range(E):
        a, b = synth.expert_weights(e, H, I, seed=seed)
        gu[e], dn[e] = oracle.as_u16(a), oracle.as_u16(b)
    return gu, dn


def test_one_expert_top1_is_dense_swiglu_ffn():
    T, H, I = 6, 256, 128
    x = synth.tokens(T, H, seed=7)
    wr = synth.router_weight(1, H, seed=7).numpy()
    gu, dn = _experts(1, H, I, seed=7)
    res = oracle.forward(oracle.as_u16(x), wr, None, K=1, E=1, w_gu=gu, w_dn=dn)
    assert np.all(res["w"] == 1.0) and np.all(res["idx"] == 0)
    xf = x.to(torch.float64).numpy()
    Wg, Wu = f32(gu[0])[:I], f32(gu[0])[I:]
    Wd = f32(dn[0])
    hh = bf16_round_np(silu64(xf @ Wg.T) * (xf @ Wu.T))
    ref = bf16_round_np(hh @ Wd.T)
    got = f32(res["out"])
    err = np.abs(got - ref)
    # h may sit one bf16 ulp apart where fp32 and float64 dot products straddle a rounding boundary
    assert np.max(err) <= 2e-2 * np.max(np.abs(ref))
    assert np.mean(err) <= 2e-3 * np.mean(np.abs(ref))
    # swapping gate and up, or transposing the down projection, is far off
    bad = bf16_round_np(bf16_round_np(silu64(xf @ Wu.T) * (xf @ Wg.T)) @ Wd.T)
    assert np.max(np.abs(bad - ref)) > 10 * np.max(err)


def test_tiny_layer_against_float64_brute_force():
    """Tiny config (16 tokens, hidden 256, 8 experts, top-2, intermediate 512)."""
    T, H, E, K, I = 16, 256, 8, 2, 512
    x = synth.tokens(T, H, seed=0)
    wr = synth.router_weight(E, H, seed=0).numpy()
    gu, dn = _experts(E, H, I, seed=0)
    res = oracle.forward(oracle.as_u16(x), wr, None, K=K, E=E, w_gu=gu, w_dn=dn)
    xf = x.to(torch.float64).numpy()
    l64 = xf @ wr.astype(np.float64).T
    out = np.zeros((T, H))
    for t in range(T):
        order = np.argsort(-l64[t], kind="stable")[:K]
        assert order.tolist() == res["idx"][t].tolist()  # no near-ties in this seeded case
        p = np.exp(l64[t] - l64[t].max())
        p /= p.sum()
        wk = p[order] / p[order].sum()
        for k, e in enumerate(order):
            g = f32(gu[e])[:I] @ xf[t]
            u = f32(gu[e])[I:] @ xf[t]
            out[t] += wk[k] * (f32(dn[e]) @ (silu64(g) * u))
    got = f32(res["out"])
    assert np.max(np.abs(got - out)) <= 2e-2 * np.max(np.abs(out))
    assert np.sqrt(np.mean((got - out) ** 2)) <= 5e-3 * np.sqrt(np.mean(out ** 2))


def test_fp32_and_float64_accumulation_agree():
    T, H, I = 3, 512, 256
    x = synth.tokens(T, H, seed=11)
    gu, dn = _experts(2, H, I, seed=11)
    pt = np.array([0, 1, 2, 0], np.int32)
    pe = np.array([0, 1, 1, 1], np.int32)
    pw = np.array([0.5, 0.25, 1.0, 0.125], np.float32)
    y32 = oracle.ffn_bf16(oracle.as_u16(x), pt, pe, pw, gu, dn, 2)
    y64 = oracle.ffn_bf16(oracle.as_u16(x), pt, pe, pw, gu, dn, 2, acc64=True)
    assert np.max(np.abs(y32 - y64)) <= 1e-2 * np.max(np.abs(y64))


# ----------------------------------------------------------------- combine --

def test_combine_golden_cases():
    for c in json.load(open(os.path.join(GOLD, "order_cases.json")))["combine_cases"]:
        K = len(c["y"])
        y = np.array(c["y"], np.float32).reshape(K, 1)
        inv = np.arange(K, dtype=np.int32).reshape(1, K)
        got = oracle.combine(np.ascontiguousarray(y), inv)[0, 0]
        assert got == int(c["expected_bf16"], 16), c["why"]


def test_combine_gathers_through_inv():
    rng = np.random.default_rng(2)
    T, K, H = 9, 3, 16
    y = rng.standard_normal((T * K, H)).astype(np.float32)
    inv = rng.permutation(T * K).astype(np.int32).reshape(T, K)
    got = f32(oracle.combine(y, inv))
    ref = y.astype(np.float64)[inv].sum(1)
    assert np.max(np.abs(got - bf16_round_np(ref))) <= 2 ** -7 * np.max(np.abs(ref))


# -------------------------------------------------------------------- e4m3 --

def test_e4m3_golden_cases():
    for c in json.load(open(os.path.join(GOLD, "e4m3_cases.json")))["cases"]:
        assert oracle.f32_to_e4m3(c["x"]) == int(c["code"], 16), c["why"]


def test_e4m3_grid_round_trip_and_torch_cast():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            assert np.isnan(oracle.e4m3_to_f32(c))
            continue
        assert oracle.f32_to_e4m3(oracle.e4m3_to_f32(c)) == c
    table = oracle.e4m3_table()
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    ok = ~np.isnan(codes)
    assert np.array_equal(table[ok], codes[ok])
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.uniform(-447.9, 447.9, 3000), rng.standard_normal(3000) * 0.01,
                           (table[ok][:-1] + table[ok][1:]) / 2]).astype(np.float32)
    vals = vals[np.abs(vals) < 448]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.f32_to_e4m3(v) for v in vals], np.uint8)
    assert np.array_equal(mine, ref)


def test_block_quantiser():
    H = 384
    src = synth.tokens(130, H, seed=9)
    su = oracle.as_u16(src)
    su[5, 128:256] = 0  # an all-zero activation block
    for br in (1, 128):
        q, s = oracle.quant_e4m3(su, br)
        v = f32(su)
        nbr = s.shape[0]
        for rb in range(nbr):
            rows = slice(rb * br, min((rb + 1) * br, v.shape[0]))
            for cb in range(H // 128):
                blk = v[rows, cb * 128:(cb + 1) * 128]
                amax = np.float32(np.abs(blk).max())
                exp_s = np.float32(1.0) if amax == 0 else np.float32(amax) / np.float32(448.0)
                assert s[rb, cb] == exp_s
                qb = q[rows, cb * 128:(cb + 1) * 128]
                if amax > 0:
                    # the element with the block's amax lands on +-448 exactly
                    r, c = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
                    assert qb[r, c] & 0x7F == 0x7E
                deq = oracle.e4m3_table()[qb].astype(np.float64) * float(exp_s)
                assert np.all(np.abs(deq - blk) <= 2 ** -4 * np.abs(blk) + float(exp_s) * 2 ** -10)
    assert np.all(oracle.quant_e4m3(su, 1)[0][5, 128:256] == 0)
    # the whole quantiser equals torch's IEEE fp32 divide + float8_e4m3fn cast (RNE)
    v = torch.from_numpy(f32(su).astype(np.float32))
    for br in (1, 128):
        q, s = oracle.quant_e4m3(su, br)
        amax = torch.stack([torch.stack([v[r:r + br, c * 128:(c + 1) * 128].abs().max()
                                         for c in range(H // 128)]) for r in range(0, v.shape[0], br)])
        st = torch.where(amax == 0, torch.ones_like(amax), amax / torch.tensor(448.0))
        assert np.array_equal(st.numpy(), s)
        full = st.repeat_interleave(br, 0)[: v.shape[0]].repeat_interleave(128, 1)
        ref = (v / full).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(ref, q)


def test_fp8_ffn_against_float64_dequantised_math():
    T, H, I = 3, 256, 256
    x = synth.tokens(T, H, seed=13)
    gu, dn = _experts(1, H, I, seed=13)
    qgu, sgu = oracle.quant_e4m3(gu[0], 128)
    qdn, sdn = oracle.quant_e4m3(dn[0], 128)
    lut = oracle.e4m3_table().astype(np.float64)
    pt = np.arange(T, dtype=np.int32)
    pe = np.zeros(T, np.int32)
    pw = np.array([1.0, 0.5, 0.25], np.float32)
    y, h = oracle.ffn_fp8(oracle.as_u16(x), pt, pe, pw, {0: qgu}, {0: sgu}, {0: qdn}, {0: sdn}, 1, want_h=True)
    Wgu = lut[qgu] * np.repeat(np.repeat(sgu, 128, 0), 128, 1)
    Wdn = lut[qdn] * np.repeat(np.repeat(sdn, 128, 0), 128, 1)
    for t in range(T):
        qx, sx = oracle.quant_e4m3(oracle.as_u16(x)[t:t + 1], 1)
        xd = lut[qx[0]] * np.repeat(sx[0], 128)
        g = Wgu[:I] @ xd
        u = Wgu[I:] @ xd
        hh = bf16_round_np(silu64(g) * u)
        assert np.max(np.abs(f32(h[t]) - hh)) <= 2 ** -7 * np.max(np.abs(hh))
        qh, sh = oracle.quant_e4m3(h[t:t + 1], 1)
        hd = lut[qh[0]] * np.repeat(sh[0], 128)
        ref = pw[t] * (Wdn @ hd)
        assert np.max(np.abs(y[t] - ref)) <= 1e-4 * np.max(np.abs(ref))
    # and the fp8 layer stays near the bf16 one
    yb = oracle.ffn_bf16(oracle.as_u16(x), pt, pe, pw, gu, dn, 1)
    assert np.max(np.abs(y - yb)) <= 1e-1 * np.max(np.abs(yb))


# --------------------------------------------------------------------- MX --

MX = json.load(open(os.path.join(GOLD, "mx_cases.json")))


def test_e2m1_decode_table():
    """The OCP MX E2M1 element: sign, 2 exponent bits (bias 1), 1 mantissa bit."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    t = oracle.e2m1_table()
    assert t[:8].tolist() == mags
    assert t[8:].tolist() == [-m for m in mags]
    assert np.signbit(t[8])


def test_e2m1_golden_cases():
    for c in MX["e2m1_cases"]:
        assert oracle.f32_to_e2m1(c["x"]) == int(c["code"], 16), c["why"]


def test_e2m1_encoder_against_exhaustive_nearest():
    """Round to nearest even by exhaustive search over the 8 magnitudes (ties
    go to the code with mantissa bit 0), against the oracle's arithmetic
    encoder; saturation above 6."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    rng = np.random.default_rng(11)
    mids = (mags[:-1] + mags[1:]) / 2
    vals = np.concatenate([rng.uniform(-6.5, 6.5, 4000), mids, -mids, mags, rng.uniform(-0.6, 0.6, 500)])
    vals = vals.astype(np.float32)
    for v in vals:
        a = abs(float(v))
        if a >= 6.0:
            want = 7
        else:
            d = np.abs(mags - a)
            best = np.flatnonzero(d == d.min())
            want = int(best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0])
        want |= 8 if np.signbit(v) else 0
        assert oracle.f32_to_e2m1(float(v)) == want, float(v)


def test_mx_block_golden_cases():
    for c in MX["block_cases"]:
        blk = np.zeros((1, 32), np.uint16)
        if "values_bf16" in c:
            for i, hx in enumerate(c["values_bf16"]):
                blk[0, i] = int(hx, 16)
        else:
            vals = np.zeros(32, np.float32)
            vals[:len(c["values"])] = c["values"]
            blk[0] = bf16_bits_np(vals)
        q, s = oracle.quant_mx(blk, c["elem"])
        assert int(s[0, 0]) == c["scale"], c["why"]
        for i, code in c["codes"].items():
            assert int(q[0, int(i)]) == int(code, 16), c["why"]


def bf16_bits_np(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_mx_quantiser_properties():
    """For every 32-element block of seeded rows: the scale X is the power of
    two with 2^emax <= amax / X < 2^(emax+1); each element decodes to the
    nearest representable value of v / X (or the format's largest, when
    v / X lies beyond it); an all-zero block has X = 2^-127 and zero codes."""
    src = synth.tokens(6, 256, seed=19)
    su = oracle.as_u16(src)
    su[2, 64:96] = 0
    v = f32(su)
    for elem, emax, table, top in (("e2m1", 2, oracle.e2m1_table(), 6.0), ("e4m3", 8, oracle.e4m3_table(), 448.0)):
        q, s = oracle.quant_mx(su, elem)
        finite = table[~np.isnan(table)].astype(np.float64)
        for r in range(v.shape[0]):
            for b in range(v.shape[1] // 32):
                blk = v[r, b * 32:(b + 1) * 32]
                X = 2.0 ** (int(s[r, b]) - 127)
                amax = np.abs(blk).max()
                if amax == 0:
                    assert s[r, b] == 0 and np.all(q[r, b * 32:(b + 1) * 32] & 0x7F == 0)
                    continue
                assert 2.0 ** emax <= amax / X < 2.0 ** (emax + 1)
                deq = table[q[r, b * 32:(b + 1) * 32]].astype(np.float64)
                for vi, di in zip(blk / X, deq):
                    tgt = np.clip(vi, -top, top)
                    assert abs(di - tgt) == np.min(np.abs(finite - tgt))  # nearest (ties either way)


def test_mxfp4_ffn_against_float64_dequantised_math():
    T, H, I = 3, 256, 128
    x = synth.tokens(T, H, seed=23)
    gu, dn = _experts(1, H, I, seed=23)
    qgu, sgu = oracle.quant_mx(gu[0], "e2m1")
    qdn, sdn = oracle.quant_mx(dn[0], "e2m1")
    l4 = oracle.e2m1_table().astype(np.float64)
    l8 = oracle.e4m3_table().astype(np.float64)
    pt = np.arange(T, dtype=np.int32)
    pe = np.zeros(T, np.int32)
    pw = np.array([1.0, 0.5, 0.25], np.float32)
    y, h = oracle.ffn_mxfp4(oracle.as_u16(x), pt, pe, pw, {0: qgu}, {0: sgu}, {0: qdn}, {0: sdn}, 1, want_h=True)

    def deq(q, s, table):
        return table[q] * np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=1)

    Wgu, Wdn = deq(qgu, sgu, l4), deq(qdn, sdn, l4)
    for t in range(T):
        qx, sx = oracle.quant_mx(oracle.as_u16(x)[t:t + 1], "e4m3")
        xd = deq(qx, sx, l8)[0]
        g = Wgu[:I] @ xd
        u = Wgu[I:] @ xd
        hh = bf16_round_np(silu64(g) * u)
        assert np.max(np.abs(f32(h[t]) - hh)) <= 2 ** -7 * np.max(np.abs(hh))
        qh, sh = oracle.quant_mx(h[t:t + 1], "e4m3")
        hd = deq(qh, sh, l8)[0]
        ref = pw[t] * (Wdn @ hd)
        assert np.max(np.abs(y[t] - ref)) <= 1e-4 * np.max(np.abs(ref))
    # and the MXFP4 layer stays within a few tens of percent of the bf16 one (one mantissa bit per weight)
    yb = oracle.ffn_bf16(oracle.as_u16(x), pt, pe, pw, gu, dn, 1)
    rel = np.sqrt(np.mean((y - yb) ** 2)) / np.sqrt(np.mean(yb ** 2))
    assert rel <= 0.25, rel
