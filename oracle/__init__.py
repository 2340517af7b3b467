"""CPU oracle of the routed MoE layer forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. It wraps ``moe_oracle.c`` (plain C, built with gcc,
sharing no code with the CUDA library) through ctypes and adds nothing but
argument marshalling and the composition of the steps in the layer's order.

Arrays are numpy: bf16 data travels as uint16 bit patterns, e4m3 as uint8.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc, OpenMP, IEEE fp32)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_router_logits.argtypes = [P, P, P, I, I, I, P, I]
        lib.oracle_topk.argtypes = [P, I, I, I, P, P]
        lib.oracle_permute.argtypes = [P, I, I, I, P, P, P, P, P]
        lib.oracle_ffn_bf16.argtypes = [P, I, I, I, P, P, P, P, P, P, P, I, I]
        lib.oracle_ffn_bf16.restype = I
        lib.oracle_ffn_fp8.argtypes = [P, I, I, I, P, P, P, P, P, P, P, P, P, I]
        lib.oracle_ffn_fp8.restype = I
        lib.oracle_combine.argtypes = [P, P, I, I, I, P]
        lib.oracle_quant_e4m3.argtypes = [P, I, I, I, P, P]
        lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
        lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_f32_to_e2m1.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_e2m1.restype = ctypes.c_uint8
        lib.oracle_e2m1_to_f32.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_to_f32.restype = ctypes.c_float
        lib.oracle_quant_mx.argtypes = [P, I, I, I, P, P]
        lib.oracle_ffn_mxfp4.argtypes = [P, I, I, I, P, P, P, P, P, P, P, P, P, I]
        lib.oracle_ffn_mxfp4.restype = I
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def as_u16(t) -> np.ndarray:
    """bf16 torch tensor (any device) or uint16 array -> C-contiguous uint16 numpy."""
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.uint16)
    import torch
    return np.ascontiguousarray(t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------- steps --

def router_logits(x_u16: np.ndarray, wr: np.ndarray, bias=None, threads: int = 0) -> np.ndarray:
    """fp32 logits [T, E] in the specified 32-lane interleaved order (+ bias)."""
    lib = _load()
    T, H = x_u16.shape
    E = wr.shape[0]
    wr = np.ascontiguousarray(wr, dtype=np.float32)
    out = np.empty((T, E), dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    lib.oracle_router_logits(_p(x_u16), _p(wr), None if b is None else _p(b), T, H, E, _p(out), threads)
    return out


def topk(logits: np.ndarray, K: int):
    """(idx int32 [T, K], w float64 [T, K]) -- full sort by (logit desc, e asc)."""
    lib = _load()
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float64)
    lib.oracle_topk(_p(logits), T, E, K, _p(idx), _p(w))
    return idx, w


def permute(idx: np.ndarray, E: int):
    """(counts [E], offsets [E+1], perm_src [P], perm_k [P], inv [T, K])."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    P = T * K
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm_src = np.empty(P, np.int32)
    perm_k = np.empty(P, np.int32)
    inv = np.empty((T, K), np.int32)
    lib.oracle_permute(_p(idx), T, K, E, _p(counts), _p(offsets), _p(perm_src), _p(perm_k), _p(inv))
    return counts, offsets, perm_src, perm_k, inv


def _ptr_array(arrs, n, dtype):
    keep = []
    ptrs = (ctypes.c_void_p * n)()
    for e in range(n):
        a = arrs.get(e) if isinstance(arrs, dict) else (arrs[e] if e < len(arrs) else None)
        if a is None:
            ptrs[e] = None
        else:
            a = np.ascontiguousarray(a, dtype=dtype)
            keep.append(a)
            ptrs[e] = a.ctypes.data
    return ptrs, keep


def ffn_bf16(x_u16, pair_token, pair_expert, pair_weight, w_gu, w_dn, E, acc64=False, threads=0,
             want_h=False):
    """y [npairs, H] fp32 (and h [npairs, I] bf16 bits) for bf16 experts.

    w_gu / w_dn: dict or list expert -> uint16 array ([2I, H] / [H, I])."""
    lib = _load()
    T, H = x_u16.shape
    pair_token = np.ascontiguousarray(pair_token, np.int32)
    pair_expert = np.ascontiguousarray(pair_expert, np.int32)
    pair_weight = np.ascontiguousarray(pair_weight, np.float32)
    n = pair_token.shape[0]
    pg, k1 = _ptr_array(w_gu, E, np.uint16)
    pd, k2 = _ptr_array(w_dn, E, np.uint16)
    first = next(a for a in k1)
    I = first.shape[0] // 2
    y = np.empty((n, H), np.float32)
    h = np.empty((n, I), np.uint16) if want_h else None
    rc = lib.oracle_ffn_bf16(_p(x_u16), H, I, n, _p(pair_token), _p(pair_expert), _p(pair_weight), pg, pd,
                             _p(y), None if h is None else _p(h), int(acc64), threads)
    if rc != 0:
        raise ValueError("oracle_ffn_bf16: weights of a needed expert were not given")
    return (y, h) if want_h else y


def ffn_fp8(x_u16, pair_token, pair_expert, pair_weight, q_gu, s_gu, q_dn, s_dn, E, threads=0,
            want_h=False):
    """y [npairs, H] fp32 for e4m3 experts with 128x128 block scales."""
    lib = _load()
    T, H = x_u16.shape
    pair_token = np.ascontiguousarray(pair_token, np.int32)
    pair_expert = np.ascontiguousarray(pair_expert, np.int32)
    pair_weight = np.ascontiguousarray(pair_weight, np.float32)
    n = pair_token.shape[0]
    pqg, k1 = _ptr_array(q_gu, E, np.uint8)
    psg, k2 = _ptr_array(s_gu, E, np.float32)
    pqd, k3 = _ptr_array(q_dn, E, np.uint8)
    psd, k4 = _ptr_array(s_dn, E, np.float32)
    I = k1[0].shape[0] // 2
    y = np.empty((n, H), np.float32)
    h = np.empty((n, I), np.uint16) if want_h else None
    rc = lib.oracle_ffn_fp8(_p(x_u16), H, I, n, _p(pair_token), _p(pair_expert), _p(pair_weight), pqg, psg,
                            pqd, psd, _p(y), None if h is None else _p(h), threads)
    if rc != 0:
        raise ValueError("oracle_ffn_fp8: weights of a needed expert were not given")
    return (y, h) if want_h else y


def ffn_mxfp4(x_u16, pair_token, pair_expert, pair_weight, q_gu, s_gu, q_dn, s_dn, E, threads=0,
              want_h=False):
    """y [npairs, H] fp32 for MXFP4 experts (e2m1 codes [2I, H] / [H, I], one
    E8M0 scale byte per 32 elements along each row); activations MX e4m3."""
    lib = _load()
    T, H = x_u16.shape
    pair_token = np.ascontiguousarray(pair_token, np.int32)
    pair_expert = np.ascontiguousarray(pair_expert, np.int32)
    pair_weight = np.ascontiguousarray(pair_weight, np.float32)
    n = pair_token.shape[0]
    pqg, k1 = _ptr_array(q_gu, E, np.uint8)
    psg, k2 = _ptr_array(s_gu, E, np.uint8)
    pqd, k3 = _ptr_array(q_dn, E, np.uint8)
    psd, k4 = _ptr_array(s_dn, E, np.uint8)
    I = k1[0].shape[0] // 2
    y = np.empty((n, H), np.float32)
    h = np.empty((n, I), np.uint16) if want_h else None
    rc = lib.oracle_ffn_mxfp4(_p(x_u16), H, I, n, _p(pair_token), _p(pair_expert), _p(pair_weight), pqg, psg,
                              pqd, psd, _p(y), None if h is None else _p(h), threads)
    if rc != 0:
        raise ValueError("oracle_ffn_mxfp4: weights of a needed expert were not given")
    return (y, h) if want_h else y


def combine(y_pair: np.ndarray, inv: np.ndarray) -> np.ndarray:
    """out [T, H] bf16 bits = bf16(sum_k y_pair[inv[t,k]]) in k order."""
    lib = _load()
    y_pair = np.ascontiguousarray(y_pair, np.float32)
    inv = np.ascontiguousarray(inv, np.int32)
    T, K = inv.shape
    H = y_pair.shape[1]
    out = np.empty((T, H), np.uint16)
    lib.oracle_combine(_p(y_pair), _p(inv), T, K, H, _p(out))
    return out


def quant_e4m3(src_u16: np.ndarray, block_rows: int):
    """(q uint8 [rows, cols], scales fp32 [ceil(rows/br), cols/128])."""
    lib = _load()
    src_u16 = np.ascontiguousarray(src_u16, np.uint16)
    rows, cols = src_u16.shape
    assert cols % 128 == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty(((rows + block_rows - 1) // block_rows, cols // 128), np.float32)
    lib.oracle_quant_e4m3(_p(src_u16), rows, cols, block_rows, _p(q), _p(s))
    return q, s


def quant_mx(src_u16: np.ndarray, elem: str = "e2m1"):
    """(q uint8 [rows, cols] one code per byte, scales uint8 [rows, cols/32] E8M0)."""
    lib = _load()
    src_u16 = np.ascontiguousarray(src_u16, np.uint16)
    rows, cols = src_u16.shape
    assert cols % 32 == 0
    q = np.empty((rows, cols), np.uint8)
    s = np.empty((rows, cols // 32), np.uint8)
    lib.oracle_quant_mx(_p(src_u16), rows, cols, {"e2m1": 0, "e4m3": 1}[elem], _p(q), _p(s))
    return q, s


def f32_to_e2m1(v: float) -> int:
    return int(_load().oracle_f32_to_e2m1(float(v)))


def e2m1_to_f32(c: int) -> float:
    return float(_load().oracle_e2m1_to_f32(int(c)))


def e2m1_table() -> np.ndarray:
    return np.array([e2m1_to_f32(c) for c in range(16)], dtype=np.float32)


def f32_to_e4m3(v: float) -> int:
    return int(_load().oracle_f32_to_e4m3(float(v)))


def e4m3_to_f32(c: int) -> float:
    return float(_load().oracle_e4m3_to_f32(int(c)))


def e4m3_table() -> np.ndarray:
    return np.array([e4m3_to_f32(c) for c in range(256)], dtype=np.float32)


def f32_to_bf16_bits(v: float) -> int:
    return int(_load().oracle_f32_to_bf16(float(v)))


# ----------------------------------------------------- composed forward --

def route(x_u16, wr, bias, K, threads=0):
    """(logits, idx, w64) for tokens x."""
    logits = router_logits(x_u16, wr, bias, threads)
    idx, w = topk(logits, K)
    return logits, idx, w


def forward(x_u16, wr, bias, K, E, w_gu, w_dn, dtype="bf16", scales=None, threads=0, acc64=False,
            tokens=None):
    """The whole layer on the CPU. Returns a dict of every intermediate.

    tokens: optional index array; when given only those tokens' outputs are
    computed (routing of a token depends on that token alone, and its output
    on its own pairs alone), and 'out' has one row per listed token.
    For dtype 'fp8', w_gu/w_dn hold e4m3 codes and ``scales`` = (s_gu, s_dn);
    for 'mxfp4', e2m1 codes and their E8M0 scale bytes."""
    T, H = x_u16.shape
    logits, idx, w64 = route(x_u16, wr, bias, K, threads)
    counts, offsets, perm_src, perm_k, inv = permute(idx, E)
    sel = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    pt = np.repeat(sel, K).astype(np.int32)
    pk = np.tile(np.arange(K), len(sel))
    pe = idx[sel].reshape(-1)
    pw = w64[sel].reshape(-1).astype(np.float32)
    if dtype == "bf16":
        y = ffn_bf16(x_u16, pt, pe, pw, w_gu, w_dn, E, acc64=acc64, threads=threads)
    elif dtype == "mxfp4":
        s_gu, s_dn = scales
        y = ffn_mxfp4(x_u16, pt, pe, pw, w_gu, s_gu, w_dn, s_dn, E, threads=threads)
    else:
        s_gu, s_dn = scales
        y = ffn_fp8(x_u16, pt, pe, pw, w_gu, s_gu, w_dn, s_dn, E, threads=threads)
    inv_local = np.arange(len(sel) * K, dtype=np.int32).reshape(len(sel), K)
    out = combine(y, inv_local)
    return dict(logits=logits, idx=idx, w=w64, counts=counts, offsets=offsets, perm_src=perm_src,
                perm_k=perm_k, inv=inv, y_sel=y, out=out, tokens=sel)
