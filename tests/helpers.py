"""Shared test helpers: build a layer from seeded inputs, run the oracle on the
same bytes, compare. Inputs always come from ``synth``; expected values always
come from ``oracle``."""

from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


def f32_of_bf16_bits(u16: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f32(u16).astype(np.float64)


class LayerCase:
    """Seeded inputs of one MoE layer on a CUDA device, plus a MoeLayer holding them."""

    def __init__(self, T, H, E, K, I, seed=0, zipf=None, wdtype=0, n_spare=0, hot=None, device="cuda",
                 first_token=0, unregistered=()):
        import mixture_experts_layer_24_b200 as M
        self.T, self.H, self.E, self.K, self.I, self.seed, self.wdtype = T, H, E, K, I, seed, wdtype
        self.dev = torch.device(device)
        self.x = synth.tokens(T, H, seed=seed, device=self.dev, first_token=first_token)
        self.wr = synth.router_weight(E, H, seed=seed, device=self.dev)
        self.bias = None if zipf is None else synth.zipf_logit_bias(E, s=zipf, seed=seed).to(self.dev)
        self.w_gu, self.w_dn = [], []
        for e in range(E):
            a, b = synth.expert_weights(e, H, I, seed=seed, device=self.dev)
            self.w_gu.append(a)
            self.w_dn.append(b)
        self.q = None
        if wdtype == M.MOE_FP8_E4M3_B128:
            self.q = []
            for e in range(E):
                qg = torch.empty((2 * I, H), dtype=torch.uint8, device=self.dev)
                sg = torch.empty((2 * I // 128, H // 128), dtype=torch.float32, device=self.dev)
                qd = torch.empty((H, I), dtype=torch.uint8, device=self.dev)
                sd = torch.empty((H // 128, I // 128), dtype=torch.float32, device=self.dev)
                M.moe_quantize_e4m3(self.w_gu[e], 2 * I, H, 128, qg, sg)
                M.moe_quantize_e4m3(self.w_dn[e], H, I, 128, qd, sd)
                self.q.append((qg, sg, qd, sd))
            torch.cuda.synchronize()
        self.layer = M.MoeLayer(H, E, K, I, wdtype=wdtype, n_spare_slots=n_spare, device=self.dev)
        self.host = {}
        for e in range(E):
            if e in unregistered:
                continue
            resident = hot is None or e in hot
            if self.q is None:
                g, d, sg, sd = self.w_gu[e], self.w_dn[e], None, None
            else:
                g, sg, d, sd = self.q[e]
            if resident:
                self.layer.register(e, g, d, sg, sd, M.MOE_LOC_HBM)
            else:
                hg = g.cpu().pin_memory()
                hd = d.cpu().pin_memory()
                hsg = sg.cpu().pin_memory() if sg is not None else None
                hsd = sd.cpu().pin_memory() if sd is not None else None
                self.host[e] = (hg, hd, hsg, hsd)
                self.layer.register(e, hg, hd, hsg, hsd, M.MOE_LOC_HOST_PINNED)

    def forward(self, x=None):
        x = self.x if x is None else x
        return self.layer.forward(x, self.wr, self.bias)

    # ---- oracle side (numpy on the host, same bytes) ----
    def oracle_inputs(self):
        xu = oracle.as_u16(self.x)
        wr = self.wr.cpu().numpy()
        bias = None if self.bias is None else self.bias.cpu().numpy()
        return xu, wr, bias

    def expert_arrays(self, experts):
        """The oracle's copy of the experts' weights: the seeded bf16 draws, and for
        FP8 their codes and 128x128 block scales from the oracle's own quantiser
        (never the GPU's codes)."""
        gu, dn, sgu, sdn = {}, {}, {}, {}
        for e in experts:
            e = int(e)
            g, d = oracle.as_u16(self.w_gu[e]), oracle.as_u16(self.w_dn[e])
            if self.q is None:
                gu[e], dn[e] = g, d
            else:
                gu[e], sgu[e] = oracle.quant_e4m3(g, 128)
                dn[e], sdn[e] = oracle.quant_e4m3(d, 128)
        return gu, dn, sgu, sdn

    def oracle_forward(self, tokens=None, threads=0):
        xu, wr, bias = self.oracle_inputs()
        logits, idx, w = oracle.route(xu, wr, bias, self.K, threads)
        sel = np.arange(self.T) if tokens is None else np.asarray(tokens)
        gu, dn, sgu, sdn = self.expert_arrays(np.unique(idx[sel]))
        if self.q is None:
            res = oracle.forward(xu, wr, bias, self.K, self.E, gu, dn, threads=threads, tokens=tokens)
        else:
            res = oracle.forward(xu, wr, bias, self.K, self.E, gu, dn, dtype="fp8", scales=(sgu, sdn),
                                 threads=threads, tokens=tokens)
        return res

    def close(self):
        self.layer.close()


def assert_close_out(got_u16: np.ndarray, ref_u16: np.ndarray, rel: float):
    g = f32_of_bf16_bits(got_u16)
    r = f32_of_bf16_bits(ref_u16)
    err = np.max(np.abs(g - r))
    scale = np.max(np.abs(r))
    assert err <= rel * scale, f"max|err| {err:.4g} > {rel} * max|ref| {scale:.4g}"
    return err / scale


def oracle_layer_out(x_u16, wr, bias, K, E, H, I, seed, fp8=False, threads=0):
    """Oracle outputs [rows, H] (bf16 bits) of the layer whose experts are
    synth.expert_weights(e, H, I, seed) for the token rows x_u16 (uint16 [rows, H]).
    The weights are drawn again on the host for the experts these rows route to
    (and, for FP8, quantised by the oracle), so nothing comes from the GPU."""
    _, idx, _ = oracle.route(x_u16, wr, bias, K, threads)
    gu, dn, sgu, sdn = {}, {}, {}, {}
    for e in np.unique(idx):
        e = int(e)
        g, d = synth.expert_weights(e, H, I, seed=seed)
        g, d = oracle.as_u16(g), oracle.as_u16(d)
        if fp8:
            gu[e], sgu[e] = oracle.quant_e4m3(g, 128)
            dn[e], sdn[e] = oracle.quant_e4m3(d, 128)
        else:
            gu[e], dn[e] = g, d
    if fp8:
        return oracle.forward(x_u16, wr, bias, K, E, gu, dn, dtype="fp8", scales=(sgu, sdn), threads=threads)["out"]
    return oracle.forward(x_u16, wr, bias, K, E, gu, dn, threads=threads)["out"]

