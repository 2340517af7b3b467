"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (or None) where the C side takes pointers, and passes the current torch
CUDA stream unless one is given. Nothing is computed in Python; if
``libmoe.so`` cannot be loaded the first call raises -- there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_BF16 = 0
MOE_FP8_E4M3_B128 = 1
MOE_MXFP4 = 2
MOE_LOC_HBM = 0
MOE_LOC_HOST_PINNED = 1
MOE_SLOTS_LRU = 0
MOE_SLOTS_PER_CALL = 1
MOE_DEV_BAD_EXPERT = 1
MOE_DEV_NO_SLOT = 2
MOE_DEV_TIMEOUT = 4

STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
                4: "MOE_ERR_SLOT", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_OOM"}

EXPORTS = ["moe_ctx_create", "moe_ctx_destroy", "moe_workspace_size", "moe_route", "moe_permute",
           "moe_expert_ffn", "moe_combine", "moe_forward", "moe_quantize_e4m3", "moe_slots_create",
           "moe_slots_destroy", "moe_slots_register", "moe_slots_query", "moe_slots_stats",
           "moe_plan_hot_set", "moe_get_device_status", "moe_last_error", "moe_launch_count",
           "moe_profile_enable", "moe_profile_read", "moe_route_noalloc", "moe_slots_set_policy",
           "moe_debug_wait_flag", "moe_ep_pack", "moe_ep_recv_plan", "moe_ep_gather_rows", "moe_quantize_mx",
           "moe_debug_fail_allocs"]

PROF_KINDS = ["router", "topk", "permute", "gather", "gate_up", "down", "quant", "combine", "ffn_fused"]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


class MoeConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("intermediate", ctypes.c_int), ("wdtype", ctypes.c_int), ("flags", ctypes.c_int)]


class MoeSlotsStats(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_int64), ("cold_staged", ctypes.c_int64), ("bytes_staged", ctypes.c_int64),
                ("last_cold", ctypes.c_int32), ("last_touched", ctypes.c_int32), ("cache_hits", ctypes.c_int64),
                ("last_hits", ctypes.c_int32), ("last_routed_cold", ctypes.c_int32)]


_lib = None


def lib():
    """Loads libmoe.so (built by ``python -m mixture_experts_layer_24_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with python -m mixture_experts_layer_24_b200.build")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, S, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_size_t
    sig = {
        "moe_ctx_create": ([ctypes.POINTER(P), ctypes.POINTER(MoeConfig)], S),
        "moe_ctx_destroy": ([P], S),
        "moe_workspace_size": ([P, I], Z),
        "moe_route": ([P, P, P, P, I, P, P, P, Z, P], S),
        "moe_permute": ([P, P, I, P, P, P, P, P, P, Z, P], S),
        "moe_expert_ffn": ([P, P, P, P, P, P, P, I, P, P, Z, P], S),
        "moe_combine": ([P, P, P, I, P, P], S),
        "moe_forward": ([P, P, P, P, P, I, P, P, Z, P], S),
        "moe_quantize_e4m3": ([P, I, I, I, P, P, P], S),
        "moe_slots_create": ([ctypes.POINTER(P), P, I], S),
        "moe_slots_destroy": ([P], S),
        "moe_slots_register": ([P, I, P, P, P, P, I], S),
        "moe_slots_query": ([P, I, ctypes.POINTER(I), ctypes.POINTER(I)], S),
        "moe_slots_stats": ([P, ctypes.POINTER(MoeSlotsStats)], S),
        "moe_slots_set_policy": ([P, I], S),
        "moe_plan_hot_set": ([P, I, I, P], S),
        "moe_get_device_status": ([P, ctypes.POINTER(ctypes.c_int32), I], S),
        "moe_last_error": ([], ctypes.c_char_p),
        "moe_launch_count": ([P], ctypes.c_int64),
        "moe_profile_enable": ([P, I], S),
        "moe_profile_read": ([P, I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), I], S),
        "moe_route_noalloc": ([P, P, P, I, I, I, I, P, P, P], S),
        "moe_debug_wait_flag": ([P, P, ctypes.c_int64, P], S),
        "moe_ep_pack": ([P, P, P, P, P, P, I, P, P, P], S),
        "moe_ep_recv_plan": ([P, P, I, P, P, P, P, P], S),
        "moe_ep_gather_rows": ([P, P, P, I, P, P], S),
        "moe_quantize_mx": ([P, I, I, I, P, P, P], S),
        "moe_debug_fail_allocs": ([I, I, I], S),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(st: int, where: str):
    if st != 0:
        raise MoeError(st, where, lib().moe_last_error().decode())


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        if not torch.cuda.is_available():
            return None  # the call will fail its own checks; there is no CPU path
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# ------------------------------------------------------------ C entry points --

MOE_FLAG_NO_PDL = 1


def moe_ctx_create(hidden, n_experts, top_k, intermediate, wdtype=MOE_BF16, flags=0):
    cfg = MoeConfig(hidden, n_experts, top_k, intermediate, wdtype, flags)
    h = ctypes.c_void_p()
    _check(lib().moe_ctx_create(ctypes.byref(h), ctypes.byref(cfg)), "moe_ctx_create")
    return h


def moe_ctx_destroy(ctx):
    _check(lib().moe_ctx_destroy(ctx), "moe_ctx_destroy")


def moe_workspace_size(ctx, T: int) -> int:
    return int(lib().moe_workspace_size(ctx, T))


def moe_route(ctx, x, w_router, logit_bias, T, topk_idx, topk_w, ws, stream=None):
    _check(lib().moe_route(ctx, _p(x), _p(w_router), _p(logit_bias), T, _p(topk_idx), _p(topk_w), _p(ws),
                           _nbytes(ws), _s(stream)), "moe_route")


def moe_permute(ctx, topk_idx, T, counts, offsets, perm_src, perm_k, inv, ws, stream=None):
    _check(lib().moe_permute(ctx, _p(topk_idx), T, _p(counts), _p(offsets), _p(perm_src), _p(perm_k), _p(inv),
                             _p(ws), _nbytes(ws), _s(stream)), "moe_permute")


def moe_expert_ffn(ctx, slots, x, perm_src, perm_k, offsets, topk_w, T, y_pair, ws, stream=None):
    _check(lib().moe_expert_ffn(ctx, slots, _p(x), _p(perm_src), _p(perm_k), _p(offsets), _p(topk_w), T,
                                _p(y_pair), _p(ws), _nbytes(ws), _s(stream)), "moe_expert_ffn")


def moe_route_noalloc(x, w_router, logit_bias, T, H, E, K, topk_idx, topk_w, stream=None):
    """Router without a context or workspace (static scratch inside libmoe)."""
    _check(lib().moe_route_noalloc(_p(x), _p(w_router), _p(logit_bias), T, H, E, K, _p(topk_idx), _p(topk_w),
                                   _s(stream)), "moe_route_noalloc")


def moe_combine(ctx, y_pair, inv, T, out, stream=None):
    _check(lib().moe_combine(ctx, _p(y_pair), _p(inv), T, _p(out), _s(stream)), "moe_combine")


def moe_forward(ctx, slots, x, w_router, logit_bias, T, out, ws, stream=None):
    _check(lib().moe_forward(ctx, slots, _p(x), _p(w_router), _p(logit_bias), T, _p(out), _p(ws), _nbytes(ws),
                             _s(stream)), "moe_forward")


def moe_ep_pack(ctx, x, topk_w, perm_src, perm_k, offsets, T, x_send, w_send, stream=None):
    _check(lib().moe_ep_pack(ctx, _p(x), _p(topk_w), _p(perm_src), _p(perm_k), _p(offsets), T, _p(x_send),
                             _p(w_send), _s(stream)), "moe_ep_pack")


def moe_ep_recv_plan(ctx, recv_counts, n_src, offsets, perm_src, perm_k, inv, stream=None):
    _check(lib().moe_ep_recv_plan(ctx, _p(recv_counts), n_src, _p(offsets), _p(perm_src), _p(perm_k), _p(inv),
                                  _s(stream)), "moe_ep_recv_plan")


def moe_ep_gather_rows(ctx, src, idx, n_rows, dst, stream=None):
    _check(lib().moe_ep_gather_rows(ctx, _p(src), _p(idx), n_rows, _p(dst), _s(stream)), "moe_ep_gather_rows")


def moe_quantize_e4m3(src, rows, cols, block_rows, q, scales, stream=None):
    _check(lib().moe_quantize_e4m3(_p(src), rows, cols, block_rows, _p(q), _p(scales), _s(stream)),
           "moe_quantize_e4m3")


def moe_quantize_mx(src, rows, cols, elem, q, scales, stream=None):
    """MX quantiser: elem 0 = E2M1 (q packed two per byte), 1 = E4M3; E8M0 scales per 32 elements."""
    _check(lib().moe_quantize_mx(_p(src), rows, cols, elem, _p(q), _p(scales), _s(stream)), "moe_quantize_mx")


def moe_slots_create(ctx, n_spare_slots: int):
    h = ctypes.c_void_p()
    _check(lib().moe_slots_create(ctypes.byref(h), ctx, n_spare_slots), "moe_slots_create")
    return h


def moe_slots_destroy(slots):
    _check(lib().moe_slots_destroy(slots), "moe_slots_destroy")


def moe_slots_register(slots, expert, w_gu, w_dn, s_gu=None, s_dn=None, location=MOE_LOC_HBM):
    _check(lib().moe_slots_register(slots, expert, _p(w_gu), _p(w_dn), _p(s_gu), _p(s_dn), location),
           "moe_slots_register")


def moe_slots_query(slots, expert):
    loc, slot = ctypes.c_int(), ctypes.c_int()
    _check(lib().moe_slots_query(slots, expert, ctypes.byref(loc), ctypes.byref(slot)), "moe_slots_query")
    return loc.value, slot.value


def moe_slots_stats(slots) -> dict:
    st = MoeSlotsStats()
    _check(lib().moe_slots_stats(slots, ctypes.byref(st)), "moe_slots_stats")
    return {k: getattr(st, k) for k, _ in MoeSlotsStats._fields_}


def moe_slots_set_policy(slots, policy: int) -> None:
    _check(lib().moe_slots_set_policy(slots, int(policy)), "moe_slots_set_policy")


def moe_plan_hot_set(hist, n_hot: int):
    """hist: int64 CPU tensor [E] -> int32 CPU tensor [n_hot]."""
    hist = hist.to(torch.int64).contiguous()
    hot = torch.empty(n_hot, dtype=torch.int32)
    _check(lib().moe_plan_hot_set(_p(hist), hist.numel(), n_hot, _p(hot)), "moe_plan_hot_set")
    return hot


def moe_get_device_status(ctx, reset: bool = True) -> int:
    v = ctypes.c_int32()
    _check(lib().moe_get_device_status(ctx, ctypes.byref(v), int(reset)), "moe_get_device_status")
    return v.value


def moe_debug_wait_flag(ctx, flag, limit_ns: int, stream=None):
    """Test hook: one thread waits (bounded by limit_ns) for the device int32
    ``flag`` to become nonzero; on time-out the status word gets MOE_DEV_TIMEOUT."""
    _check(lib().moe_debug_wait_flag(ctx, _p(flag), int(limit_ns), _s(stream)), "moe_debug_wait_flag")


MOE_ALLOC_ANY, MOE_ALLOC_DEVICE, MOE_ALLOC_PINNED = 0, 1, 2


def moe_debug_fail_allocs(kind: int, skip: int, n: int):
    """Test hook: of the library's own allocations of `kind` (MOE_ALLOC_DEVICE,
    MOE_ALLOC_PINNED or MOE_ALLOC_ANY), let `skip` succeed and fail the next `n`
    as an exhausted device or host would; n = 0 disarms it."""
    _check(lib().moe_debug_fail_allocs(int(kind), int(skip), int(n)), "moe_debug_fail_allocs")


def moe_launch_count(ctx) -> int:
    return int(lib().moe_launch_count(ctx))


def moe_profile_enable(ctx, enable: bool = True):
    _check(lib().moe_profile_enable(ctx, int(enable)), "moe_profile_enable")


def moe_profile_read(ctx, reset: bool = True) -> dict:
    """{kind: (total_ms, launches)} for every kernel kind (synchronises)."""
    out = {}
    for k, name in enumerate(PROF_KINDS):
        ms, n = ctypes.c_double(), ctypes.c_int64()
        _check(lib().moe_profile_read(ctx, k, ctypes.byref(ms), ctypes.byref(n), int(reset)), "moe_profile_read")
        out[name] = (ms.value, n.value)
    return out


# ------------------------------------------------------------- convenience --

def check_tensor(t, name, dtype, shape, device=None, pinned=False):
    """Raises unless t is a contiguous tensor of this dtype and shape, on this
    device (a CUDA torch.device with its index, or "cpu"), and in pinned
    memory when asked. The C ABI takes raw pointers and cannot see any of it."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (row-major)")
    if device is not None:
        d = torch.device(device)
        if t.device.type != d.type or (d.type == "cuda" and t.device.index != d.index):
            raise ValueError(f"{name}: on {t.device}, expected {d}")
    if pinned and not t.is_pinned():
        raise ValueError(f"{name}: host-resident weights must be in pinned memory")


def _rows(x, name):
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{name}: expected a 2-D [tokens, hidden] tensor")
    return x.shape[0]


class MoeLayer:
    """One MoE layer: a context, its slot table and a reusable workspace.

    Registered weight tensors are kept referenced here because the library
    borrows them. Every method checks its tensors' dtype, shape, layout and
    device before the call (``check_tensor``)."""

    def __init__(self, hidden, n_experts, top_k, intermediate, wdtype=MOE_BF16, n_spare_slots=0, device=None,
                 flags=0):
        self.H, self.E, self.K, self.I, self.wdtype = hidden, n_experts, top_k, intermediate, wdtype
        d = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        if d.type == "cuda" and d.index is None:
            d = torch.device("cuda", torch.cuda.current_device())
        self.device = d
        with torch.cuda.device(self.device):
            self.ctx = moe_ctx_create(hidden, n_experts, top_k, intermediate, wdtype, flags)
            try:
                self.slots = moe_slots_create(self.ctx, n_spare_slots)
            except MoeError:
                moe_ctx_destroy(self.ctx)  # nothing of a half-built layer stays allocated
                self.ctx = None
                raise
        self._keep = {}
        self._ws = None

    def register(self, e, w_gu, w_dn, s_gu=None, s_dn=None, location=MOE_LOC_HBM):
        if not 0 <= int(e) < self.E:
            raise ValueError(f"expert {e} out of range [0, {self.E})")
        if location == MOE_LOC_HBM:
            dev, pinned = self.device, False
        elif location == MOE_LOC_HOST_PINNED:
            dev, pinned = "cpu", True
        else:
            raise ValueError(f"unknown location {location}")
        H, I = self.H, self.I
        if self.wdtype == MOE_MXFP4:
            check_tensor(w_gu, "w_gu", torch.uint8, (2 * I, H // 2), dev, pinned)
            check_tensor(w_dn, "w_dn", torch.uint8, (H, I // 2), dev, pinned)
            check_tensor(s_gu, "s_gu", torch.uint8, (2 * I, H // 32), dev, pinned)
            check_tensor(s_dn, "s_dn", torch.uint8, (H, I // 32), dev, pinned)
        elif self.wdtype == MOE_FP8_E4M3_B128:
            check_tensor(w_gu, "w_gu", torch.uint8, (2 * I, H), dev, pinned)
            check_tensor(w_dn, "w_dn", torch.uint8, (H, I), dev, pinned)
            check_tensor(s_gu, "s_gu", torch.float32, (2 * I // 128, H // 128), dev, pinned)
            check_tensor(s_dn, "s_dn", torch.float32, (H // 128, I // 128), dev, pinned)
        else:
            check_tensor(w_gu, "w_gu", torch.bfloat16, (2 * I, H), dev, pinned)
            check_tensor(w_dn, "w_dn", torch.bfloat16, (H, I), dev, pinned)
            if s_gu is not None or s_dn is not None:
                raise ValueError("bf16 experts take no block scales")
        self._keep[e] = (w_gu, w_dn, s_gu, s_dn)
        moe_slots_register(self.slots, e, w_gu, w_dn, s_gu, s_dn, location)

    def workspace(self, T: int) -> torch.Tensor:
        need = moe_workspace_size(self.ctx, T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def _check_route_inputs(self, x, w_router, logit_bias):
        T = _rows(x, "x")
        check_tensor(x, "x", torch.bfloat16, (T, self.H), self.device)
        check_tensor(w_router, "w_router", torch.float32, (self.E, self.H), self.device)
        if logit_bias is not None:
            check_tensor(logit_bias, "logit_bias", torch.float32, (self.E,), self.device)
        return T

    def forward(self, x, w_router, logit_bias=None, out=None, stream=None, ws=None):
        T = self._check_route_inputs(x, w_router, logit_bias)
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        else:
            check_tensor(out, "out", torch.bfloat16, (T, self.H), self.device)
        if ws is not None:
            check_tensor(ws, "ws", torch.uint8, (ws.numel(),), self.device)
            if ws.numel() < moe_workspace_size(self.ctx, T):
                raise ValueError(f"ws: {ws.numel()} bytes, the call needs {moe_workspace_size(self.ctx, T)}")
        moe_forward(self.ctx, self.slots, x, w_router, logit_bias, T, out, self.workspace(T) if ws is None else ws,
                    stream)
        return out

    def route(self, x, w_router, logit_bias=None, stream=None):
        T = self._check_route_inputs(x, w_router, logit_bias)
        idx = torch.empty((T, self.K), dtype=torch.int32, device=self.device)
        w = torch.empty((T, self.K), dtype=torch.float32, device=self.device)
        moe_route(self.ctx, x, w_router, logit_bias, T, idx, w, self.workspace(T), stream)
        return idx, w

    def permute(self, topk_idx, stream=None):
        T = _rows(topk_idx, "topk_idx")
        check_tensor(topk_idx, "topk_idx", torch.int32, (T, self.K), self.device)
        P = T * self.K
        d = self.device
        counts = torch.empty(self.E, dtype=torch.int32, device=d)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=d)
        perm_src = torch.empty(P, dtype=torch.int32, device=d)
        perm_k = torch.empty(P, dtype=torch.int32, device=d)
        inv = torch.empty((T, self.K), dtype=torch.int32, device=d)
        moe_permute(self.ctx, topk_idx, T, counts, offsets, perm_src, perm_k, inv, self.workspace(T), stream)
        return counts, offsets, perm_src, perm_k, inv

    def expert_ffn(self, x, perm_src, perm_k, offsets, topk_w, stream=None):
        T = _rows(x, "x")
        P = T * self.K
        check_tensor(x, "x", torch.bfloat16, (T, self.H), self.device)
        check_tensor(perm_src, "perm_src", torch.int32, (P,), self.device)
        check_tensor(perm_k, "perm_k", torch.int32, (P,), self.device)
        check_tensor(offsets, "offsets", torch.int32, (self.E + 1,), self.device)
        check_tensor(topk_w, "topk_w", torch.float32, (T, self.K), self.device)
        y = torch.empty((T * self.K, self.H), dtype=torch.float32, device=self.device)
        moe_expert_ffn(self.ctx, self.slots, x, perm_src, perm_k, offsets, topk_w, T, y, self.workspace(T), stream)
        return y

    def combine(self, y_pair, inv, stream=None):
        T = _rows(inv, "inv")
        check_tensor(inv, "inv", torch.int32, (T, self.K), self.device)
        check_tensor(y_pair, "y_pair", torch.float32, (T * self.K, self.H), self.device)
        out = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        moe_combine(self.ctx, y_pair, inv, T, out, stream)
        return out

    def capture(self, x, w_router, logit_bias=None):
        """Captures one forward over the fixed tensor x into a CUDA graph.

        Returns (graph, out): graph.replay() recomputes out from the current
        contents of x. Valid while x, w_router, logit_bias and the registered
        weights stay where they are. With host-resident experts, only batches
        whose T * top_k fits in the spare slots can be captured (their cache
        bookkeeping and copies run on the device); larger ones synchronise with
        the host."""
        T = x.shape[0]
        ws = torch.empty(max(moe_workspace_size(self.ctx, T), 256), dtype=torch.uint8, device=self.device)
        out = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        self.forward(x, w_router, logit_bias, out=out, ws=ws)  # first call outside capture (kernel attributes)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.forward(x, w_router, logit_bias, out=out, ws=ws)
        g.moe_workspace = ws  # the graph's own workspace lives as long as the graph
        return g, out

    def status(self, reset=True) -> int:
        return moe_get_device_status(self.ctx, reset)

    def stats(self) -> dict:
        return moe_slots_stats(self.slots)

    def launches(self) -> int:
        return moe_launch_count(self.ctx)

    def close(self):
        if getattr(self, "slots", None) is not None:
            moe_slots_destroy(self.slots)
            self.slots = None
        if getattr(self, "ctx", None) is not None:
            moe_ctx_destroy(self.ctx)
            self.ctx = None
        self._keep = {}
        self._ws = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
