"""Seeded synthetic inputs for the routed MoE layer.

This module produces the layer's inputs (token activations, router weights,
router logit bias, expert weights) and nothing else: it holds none of the
layer's arithmetic. It is the one module that both the CPU oracle's tests and
the CUDA path use, so that both read the same bytes.

Generator (counter-based, so any slice of any tensor can be produced on its own,
on any device, with identical bits):

* ``mix32`` is the 32-bit integer finaliser x ^= x>>16; x *= 0x7feb352d;
  x ^= x>>15; x *= 0x846ca68b; x ^= x>>16 (C. Wellons' "lowbias32", from his
  published hash-prospector results).
* Element ``i`` of tensor ``(seed, tensor_id)`` draws four 32-bit words
  ``w_j = mix32(mix32(lo(i) ^ K_j) ^ mix32(hi(i) ^ K_hi))`` where ``K_j`` and
  ``K_hi`` are per-tensor keys; the eight 16-bit halves ``u_0..u_7`` are
  uniform on [0, 65535].
* The normal draw is the Irwin-Hall approximation
  ``z = (sum(u) - 262140) * sigma * sqrt(1.5) / 65536`` (mean 0, variance
  sigma^2 up to the rounding of the constant; support +-4.9 sigma), computed as
  one exact integer sum, one exact int->fp32 conversion and ONE fp32 multiply,
  then one RNE rounding to the storage dtype. Every step is an integer op or a
  single correctly-rounded IEEE operation, so CPU and GPU give identical bits.
  (A Box-Muller draw would need log/cos, whose last bits differ between the
  host and device maths libraries.)

The Zipf(s) router prior is ``bias[e] = ln p_{rank(e)}``,
``p_r = r^-s / sum_{r'} r'^-s``, with ``rank`` a seeded permutation of the
experts; it is computed in float64 on the host and rounded to fp32 once.
"""

from __future__ import annotations

import math

import numpy as np
import torch

M32 = 0xFFFFFFFF

# tensor ids (one per logical tensor; expert weights get a range)
TID_X = 1
TID_ROUTER = 2
TID_ZIPF_PERM = 3
TID_YPAIR = 4
TID_H = 5
TID_EXPERT_BASE = 1000  # expert e: gate/up = BASE + 2e, down = BASE + 2e + 1

_CHUNK = 1 << 24  # elements per generation chunk (bounds temporaries)


def _mix32_int(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & M32
    x ^= x >> 16
    return x


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 tensors holding uint32 values, overflow-free."""
    lo = c & 0xFFFF
    hi = c >> 16
    return ((x * lo) + (((x * hi) & 0xFFFF) << 16)) & M32


def _mix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _keys(seed: int, tensor_id: int):
    k0 = _mix32_int(_mix32_int(seed ^ 0x9E3779B9) ^ (tensor_id * 0x85EBCA6B))
    kj = [_mix32_int(k0 + 0x27D4EB2F * (j + 1)) for j in range(4)]
    khi = _mix32_int(k0 ^ 0x165667B1)
    return kj, khi


def _irwin_hall8(idx: torch.Tensor, seed: int, tensor_id: int) -> torch.Tensor:
    """int64 tensor of sum(u_0..u_7) - 262140 for element indices ``idx``."""
    kj, khi = _keys(seed, tensor_id)
    lo = idx & M32
    hi = _mix32((idx >> 32) ^ khi)
    s = torch.zeros_like(idx)
    for j in range(4):
        w = _mix32(_mix32(lo ^ kj[j]) ^ hi)
        s = s + (w & 0xFFFF) + (w >> 16)
    return s - 262140


_clib = None


def _c_generator():
    """ctypes handle of _gen.c (built on first use with gcc), or None."""
    global _clib
    if _clib is None:
        import ctypes
        import os
        import subprocess
        here = os.path.dirname(os.path.abspath(__file__))
        src, so = os.path.join(here, "_gen.c"), os.path.join(here, "_gen.so")
        try:
            if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
                subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                                       "-o", so + ".tmp", src])
                os.replace(so + ".tmp", so)
            lib = ctypes.CDLL(so)
            lib.synth_normal.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_uint32, ctypes.c_float]
            _clib = lib
        except Exception:  # no compiler: the torch path below gives the same bits
            _clib = False
    return _clib or None


def normal(shape, seed: int, tensor_id: int, sigma: float, dtype: torch.dtype,
           device="cpu", offset: int = 0, use_c: bool = True) -> torch.Tensor:
    """Seeded approx-N(0, sigma^2) tensor; element i uses counter ``offset + i``."""
    shape = tuple(int(s) for s in shape)
    n = 1
    for s in shape:
        n *= s
    cval = float(np.float32(sigma * math.sqrt(1.5) / 65536.0))
    if use_c and torch.device(device).type == "cpu" and dtype in (torch.float32, torch.bfloat16) \
            and _c_generator() is not None:
        import ctypes
        kj, khi = _keys(seed, tensor_id)
        keys = (ctypes.c_uint32 * 4)(*kj)
        out = torch.empty(n, dtype=dtype)
        _c_generator().synth_normal(ctypes.c_void_p(out.data_ptr()), 0 if dtype == torch.float32 else 1, n,
                                    offset, keys, khi, cval)
        return out.view(shape)
    out = torch.empty(n, dtype=dtype, device=device)
    c = torch.tensor(cval, dtype=torch.float32, device=device)
    for start in range(0, n, _CHUNK):
        stop = min(n, start + _CHUNK)
        idx = torch.arange(offset + start, offset + stop, dtype=torch.int64, device=device)
        num = _irwin_hall8(idx, seed, tensor_id).to(torch.float32)  # exact: |num| < 2^19
        out[start:stop] = (num * c).to(dtype)
    return out.view(shape)


def tokens(T: int, H: int, seed: int = 0, device="cpu", first_token: int = 0) -> torch.Tensor:
    """x ~ N(0, 1) bf16 [T, H]; token ``first_token + t`` is row t (same row for
    the same token index whatever T is)."""
    return normal((T, H), seed, TID_X, 1.0, torch.bfloat16, device, offset=first_token * H)


def router_weight(E: int, H: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Wr ~ N(0, 0.02) fp32 [E, H]."""
    return normal((E, H), seed, TID_ROUTER, 0.02, torch.float32, device)


def expert_weights(e: int, H: int, I: int, seed: int = 0, device="cpu"):
    """(w_gu [2I, H], w_dn [H, I]) bf16 ~ N(0, 0.02) for expert e.

    Rows 0..I-1 of w_gu are the gate projection, rows I..2I-1 the up
    projection; both matrices are [out, in] row-major."""
    w_gu = normal((2 * I, H), seed, TID_EXPERT_BASE + 2 * e, 0.02, torch.bfloat16, device)
    w_dn = normal((H, I), seed, TID_EXPERT_BASE + 2 * e + 1, 0.02, torch.bfloat16, device)
    return w_gu, w_dn


def zipf_permutation(E: int, seed: int = 0) -> np.ndarray:
    """rank_of[e] in 1..E: a seeded permutation (expert with rank 1 is the head)."""
    keys = np.array([_mix32_int(_mix32_int(seed ^ 0x51ED270B) ^ _mix32_int(e * 0x9E3779B9 + TID_ZIPF_PERM))
                     for e in range(E)], dtype=np.int64)
    order = np.lexsort((np.arange(E), keys))  # by key, ties by index
    rank_of = np.empty(E, dtype=np.int64)
    rank_of[order] = np.arange(1, E + 1)
    return rank_of


def zipf_logit_bias(E: int, s: float = 1.1, seed: int = 0) -> torch.Tensor:
    """fp32 [E] bias = ln p_rank(e), p_r = r^-s / sum r'^-s."""
    rank_of = zipf_permutation(E, seed)
    r = np.arange(1, E + 1, dtype=np.float64)
    z = np.sum(r ** (-s))
    logp = -s * np.log(rank_of.astype(np.float64)) - np.log(z)
    return torch.from_numpy(logp.astype(np.float32))


def normal_f32(shape, seed: int, tensor_id: int, device="cpu") -> torch.Tensor:
    """Seeded approx-N(0,1) fp32 (used for synthetic intermediate tensors such as
    y_pair or h in single-kernel tests)."""
    return normal(shape, seed, tensor_id, 1.0, torch.float32, device)
