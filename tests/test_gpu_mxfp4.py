"""MXFP4 experts (OCP MX: E2M1 weights, MX e4m3 activations, one E8M0 scale per
32 elements along K) on the block-scaled tensor cores, against the oracle.

- The MX quantiser is bit-exact (codes and scale bytes, both element types).
- Layer outputs: max|err| <= 4e-2 * max|ref|, the FP8 tolerance: as in the FP8
  path, the activations and h are quantised to 8-bit floats, and a
  one-ulp difference in h (the tensor core sums in another order) can move an
  e4m3 code by one step (2^-3 relative) or a block's scale by a power of two.
  The weights' E2M1 codes are the oracle's own on both sides.
- Routing is the bf16 router: bit-exact.
- Batch invariance: a token's output bits do not depend on the batch.
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_close_out

pytestmark = pytest.mark.gpu

TOL = 4e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mixture_experts_layer_24_b200 as M
    M.lib()
    yield


def _pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """One E2M1 code per byte [rows, cols] -> two per byte [rows, cols/2], element 2i in the low nibble."""
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def _unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


class MxCase:
    """A layer with MXFP4 experts quantised by the oracle (the same codes feed both sides)."""

    def __init__(self, T, H, E, K, I, seed, zipf=None, first_token=0):
        import mixture_experts_layer_24_b200 as M
        self.T, self.H, self.E, self.K, self.I = T, H, E, K, I
        dev = torch.device("cuda")
        self.dev = dev
        self.x = synth.tokens(T, H, seed=seed, device=dev, first_token=first_token)
        self.wr = synth.router_weight(E, H, seed=seed, device=dev)
        self.bias = None if zipf is None else synth.zipf_logit_bias(E, s=zipf, seed=seed).to(dev)
        self.layer = M.MoeLayer(H, E, K, I, wdtype=M.MOE_MXFP4, device=dev)
        self.codes = {}
        for e in range(E):
            g, d = synth.expert_weights(e, H, I, seed=seed)
            qg, sg = oracle.quant_mx(oracle.as_u16(g), "e2m1")
            qd, sd = oracle.quant_mx(oracle.as_u16(d), "e2m1")
            self.codes[e] = (qg, sg, qd, sd)
            t = [torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in (_pack_e2m1(qg), _pack_e2m1(qd), sg, sd)]
            self.layer.register(e, *t)
        torch.cuda.synchronize()

    def forward(self, x=None):
        return self.layer.forward(self.x if x is None else x, self.wr, self.bias)

    def oracle_out(self, x=None):
        x = self.x if x is None else x
        xu = oracle.as_u16(x)
        wr = self.wr.cpu().numpy()
        bias = None if self.bias is None else self.bias.cpu().numpy()
        gu = {e: c[0] for e, c in self.codes.items()}
        sgu = {e: c[1] for e, c in self.codes.items()}
        dn = {e: c[2] for e, c in self.codes.items()}
        sdn = {e: c[3] for e, c in self.codes.items()}
        return oracle.forward(xu, wr, bias, self.K, self.E, gu, dn, dtype="mxfp4", scales=(sgu, sdn))

    def close(self):
        self.layer.close()


@pytest.mark.parametrize("elem", [0, 1])
@pytest.mark.parametrize("rows,cols", [(7, 256), (130, 4096)])
def test_mx_quantizer_bit_exact(elem, rows, cols):
    import mixture_experts_layer_24_b200 as M
    src = synth.tokens(rows, cols, seed=rows + elem)
    src[0, :32] = 0.0                                # an all-zero block: scale 2^-127, codes 0
    src[1, :32] = src[1, :32] * 1e-38                # subnormal-range block
    src[2, 32:64] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4) * 2.0 ** -3  # ties after scaling
    src[3, 64:96] = -src[3, 64:96].abs() * 1e30      # large negative block
    dev = torch.device("cuda")
    d_src = src.to(dev)
    qcols = cols // 2 if elem == 0 else cols
    q = torch.empty((rows, qcols), dtype=torch.uint8, device=dev)
    s = torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
    M.moe_quantize_mx(d_src, rows, cols, elem, q, s)
    torch.cuda.synchronize()
    qo, so = oracle.quant_mx(oracle.as_u16(src), "e2m1" if elem == 0 else "e4m3")
    qg = q.cpu().numpy()
    if elem == 0:
        qg = _unpack_e2m1(qg)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(qg, qo)


@pytest.mark.parametrize("T,H,E,K,I,zipf", [(16, 256, 8, 2, 512, None), (1, 512, 8, 4, 256, None),
                                             (5, 1024, 16, 8, 512, 1.1), (100, 512, 12, 4, 768, None),
                                             (300, 256, 6, 3, 256, 1.1)])
def test_forward_mxfp4_matches_oracle(T, H, E, K, I, zipf):
    case = MxCase(T, H, E, K, I, seed=T + 7, zipf=zipf)
    out = case.forward()
    torch.cuda.synchronize()
    assert case.layer.status() == 0
    ref = case.oracle_out()
    rel = assert_close_out(oracle.as_u16(out), ref["out"], TOL)
    print(f"mxfp4 T={T} H={H} E={E} K={K} I={I}: max|err|/max|ref| = {rel:.3e}")
    idx, _ = case.layer.route(case.x, case.wr, case.bias)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    case.close()


def test_mxfp4_batch_invariance():
    case = MxCase(200, 512, 16, 4, 256, seed=3, zipf=1.1)
    full = oracle.as_u16(case.forward())
    for T in (1, 2, 7, 16, 33, 64, 65, 129):
        out = oracle.as_u16(case.forward(case.x[:T].contiguous()))
        assert np.array_equal(out, full[:T]), T
    assert case.layer.status() == 0
    case.close()


def test_mxfp4_full_size_sampled():
    """The 384-expert layer with MXFP4 experts (quantised on the GPU by the MX
    quantiser; the oracle quantises its own copy), decode and a 4096-token
    chunk, sampled tokens against the oracle."""
    import mixture_experts_layer_24_b200 as M
    H, E, K, I = 4096, 384, 8, 2048
    dev = torch.device("cuda")
    layer = M.MoeLayer(H, E, K, I, wdtype=M.MOE_MXFP4, device=dev)
    keep = []
    for e in range(E):
        g, d = synth.expert_weights(e, H, I, seed=6, device=dev)
        qg = torch.empty((2 * I, H // 2), dtype=torch.uint8, device=dev)
        sg = torch.empty((2 * I, H // 32), dtype=torch.uint8, device=dev)
        qd = torch.empty((H, I // 2), dtype=torch.uint8, device=dev)
        sd = torch.empty((H, I // 32), dtype=torch.uint8, device=dev)
        M.moe_quantize_mx(g, 2 * I, H, 0, qg, sg)
        M.moe_quantize_mx(d, H, I, 0, qd, sd)
        layer.register(e, qg, qd, sg, sd)
        keep.append((qg, qd, sg, sd))
        del g, d
    wr = synth.router_weight(E, H, seed=6, device=dev)
    bias = synth.zipf_logit_bias(E, 1.1, seed=6).to(dev)
    torch.cuda.synchronize()
    ocache = {}  # the oracle's own quantisation of each expert it needs
    for T, n_sample in ((1, 1), (8, 8), (64, 12), (4096, 16)):
        x = synth.tokens(T, H, seed=6, device=dev, first_token=4000)
        out = layer.forward(x, wr, bias)
        torch.cuda.synchronize()
        assert layer.status() == 0
        rng = np.random.default_rng(T)
        tok = np.sort(rng.choice(T, size=n_sample, replace=False))
        sub = oracle.as_u16(x)[tok]
        _, idx, _ = oracle.route(sub, wr.cpu().numpy(), bias.cpu().numpy(), K)
        gu, sgu, dn, sdn = {}, {}, {}, {}
        for e in np.unique(idx):
            e = int(e)
            if e not in ocache:
                g, d = synth.expert_weights(e, H, I, seed=6)
                ocache[e] = oracle.quant_mx(oracle.as_u16(g), "e2m1") + oracle.quant_mx(oracle.as_u16(d), "e2m1")
            gu[e], sgu[e], dn[e], sdn[e] = ocache[e]
        ref = oracle.forward(sub, wr.cpu().numpy(), bias.cpu().numpy(), K, E, gu, dn, dtype="mxfp4",
                             scales=(sgu, sdn))["out"]
        rel = assert_close_out(oracle.as_u16(out)[tok], ref, TOL)
        print(f"mxfp4 full size T={T}: max|err|/max|ref| = {rel:.3e}")
    # the same tokens in a smaller batch: identical bits
    x = synth.tokens(4096, H, seed=6, device=dev, first_token=4000)
    big = oracle.as_u16(layer.forward(x, wr, bias))
    small = oracle.as_u16(layer.forward(x[:8].contiguous(), wr, bias))
    assert np.array_equal(big[:8], small)
    layer.close()
