"""The C-ABI library (CPU-side checks, no GPU): it builds, loads, exports every
function include/moe.h declares, and its host-only paths behave."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from mixture_experts_layer_24_b200 import build as B
    B.build()
    import mixture_experts_layer_24_b200 as M
    return M.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 18
    so = os.path.join(ROOT, "mixture_experts_layer_24_b200", "libmoe.so")
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)  # resolvable through ctypes too


def test_binding_covers_every_declared_function(lib):
    from mixture_experts_layer_24_b200 import binding
    assert set(declared_functions()) == set(binding.EXPORTS)


def test_library_is_built_for_sm100a():
    """The in-tree build compiles and links every source for sm_100a only, and the library is newer than them."""
    from mixture_experts_layer_24_b200 import build as B
    assert "arch=compute_100a,code=sm_100a" in B.FLAGS
    assert sum(f.startswith("arch=") for f in B.FLAGS) == 1
    assert B.up_to_date()


def test_host_side_argument_checks(lib):
    import mixture_experts_layer_24_b200 as M
    with pytest.raises(M.MoeError) as e:
        M.moe_route(None, None, None, None, 1, None, None, None)
    assert e.value.status == 1
    # quantiser rejects shapes before touching any device memory
    st = lib.moe_quantize_e4m3(None, 4, 100, 1, None, None, None)
    assert st == 1
    st = lib.moe_quantize_e4m3(None, 4, 128, 7, None, None, None)
    assert st == 2
    assert lib.moe_workspace_size(None, 5) == 0
    assert lib.moe_quantize_e4m3(None, 0, 128, 1, None, None, None) == 0  # empty input is a no-op
    assert lib.moe_slots_set_policy(None, M.MOE_SLOTS_LRU) == 1  # NULL table
    assert lib.moe_debug_wait_flag(None, None, 1000, None) == 1  # NULL context
    assert M.MOE_SLOTS_LRU != M.MOE_SLOTS_PER_CALL


def test_mxfp4_shape_limits_checked_on_the_host(lib):
    """MXFP4 stages hold two 128-deep K blocks: H and I must be multiples of 256,
    refused before any CUDA call."""
    import mixture_experts_layer_24_b200 as M
    for H, I in ((384, 256), (256, 384)):
        with pytest.raises(M.MoeError) as e:
            M.moe_ctx_create(H, 8, 2, I, M.MOE_MXFP4)
        assert e.value.status == 2 and b"256" in lib.moe_last_error()


def test_ctx_create_without_gpu_fails_cleanly(lib):
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    import mixture_experts_layer_24_b200 as M
    with pytest.raises(M.MoeError) as e:
        M.moe_ctx_create(4096, 384, 8, 2048)
    assert e.value.status in (2, 3)


def test_config_validation(lib):
    import mixture_experts_layer_24_b200 as M
    bad = [(100, 8, 2, 256, 0, 2), (256, 8, 2, 100, 0, 2), (256, 8, 40, 256, 0, 2), (256, 4, 8, 256, 0, 2),
           (256, 8, 2, 256, 5, 1), (256, 2000, 2, 256, 0, 2)]
    # unknown flag bits are rejected before any device call
    cfg = M.binding.MoeConfig(256, 8, 2, 256, 0, 8)
    h = ctypes.c_void_p()
    assert lib.moe_ctx_create(ctypes.byref(h), ctypes.byref(cfg)) == 1
    for H, E, K, I, dt, want in bad:
        cfg = M.binding.MoeConfig(H, E, K, I, dt, 0)
        h = ctypes.c_void_p()
        assert lib.moe_ctx_create(ctypes.byref(h), ctypes.byref(cfg)) == want, (H, E, K, I, dt)


def test_hot_set_planner():
    import mixture_experts_layer_24_b200 as M
    rng = np.random.default_rng(0)
    hist = rng.integers(0, 20, size=384)
    hot = M.moe_plan_hot_set(torch.from_numpy(hist), 120).numpy()
    ref = np.lexsort((np.arange(384), -hist))[:120]  # count desc, ties -> lower index
    assert hot.tolist() == ref.tolist()
    assert M.moe_plan_hot_set(torch.zeros(10, dtype=torch.int64), 3).tolist() == [0, 1, 2]


def test_tensor_checks_of_the_binding():
    """MoeLayer's methods pass raw pointers to the C ABI, so the binding checks
    dtype, shape, layout, device and pinning first (CPU-checkable part)."""
    from mixture_experts_layer_24_b200.binding import check_tensor
    t = torch.zeros((4, 8), dtype=torch.bfloat16)
    check_tensor(t, "x", torch.bfloat16, (4, 8), "cpu")
    with pytest.raises(TypeError):
        check_tensor(t, "x", torch.float32, (4, 8))
    with pytest.raises(ValueError):
        check_tensor(t, "x", torch.bfloat16, (8, 4))
    with pytest.raises(ValueError):
        check_tensor(t.t(), "x", torch.bfloat16, (8, 4))  # a transposed view is not row-major
    with pytest.raises(ValueError):
        check_tensor(t, "x", torch.bfloat16, (4, 8), torch.device("cuda", 0))  # wrong device
    with pytest.raises(ValueError):
        check_tensor(t, "w_gu", torch.bfloat16, (4, 8), "cpu", pinned=True)  # pageable host memory
    with pytest.raises(TypeError):
        check_tensor(np.zeros((4, 8)), "x", torch.bfloat16, (4, 8))
    check_tensor(t[:0], "x", torch.bfloat16, (0, 8), "cpu")  # an empty batch is fine


def test_layer_methods_accept_valid_calls_and_reject_bad_ones(monkeypatch):
    """The checked MoeLayer methods, driven on the CPU: the C calls are replaced
    by no-ops and the layer's device is the host, so only the argument checks
    and the output allocation run. Valid calls of every method pass; each kind
    of bad argument is refused before any C call."""
    from mixture_experts_layer_24_b200 import binding as B
    calls = []
    for name in ("moe_forward", "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_slots_register"):
        monkeypatch.setattr(B, name, lambda *a, _n=name, **k: calls.append(_n))
    monkeypatch.setattr(B, "moe_workspace_size", lambda ctx, T: 4096)

    def layer(wdtype):
        L = object.__new__(B.MoeLayer)
        L.H, L.E, L.K, L.I, L.wdtype = 256, 8, 2, 128, wdtype
        L.device, L.ctx, L.slots, L._keep, L._ws = torch.device("cpu"), None, None, {}, None
        return L

    L = layer(B.MOE_BF16)
    T, H, E, K, I = 5, 256, 8, 2, 128
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    wr = torch.zeros((E, H), dtype=torch.float32)
    bias = torch.zeros(E, dtype=torch.float32)
    L.register(3, torch.zeros((2 * I, H), dtype=torch.bfloat16), torch.zeros((H, I), dtype=torch.bfloat16))
    assert L.forward(x, wr, bias).shape == (T, H)
    L.forward(x, wr, None, out=torch.empty((T, H), dtype=torch.bfloat16), ws=torch.empty(4096, dtype=torch.uint8))
    L.forward(x[:0], wr, None, out=torch.empty((0, H), dtype=torch.bfloat16))
    idx, w = L.route(x, wr, bias)
    assert idx.shape == (T, K) and idx.dtype == torch.int32 and w.dtype == torch.float32
    counts, offsets, ps, pk, inv = L.permute(idx)
    assert offsets.shape == (E + 1,) and ps.shape == (T * K,) and inv.shape == (T, K)
    y = L.expert_ffn(x, ps, pk, offsets, w)
    assert y.shape == (T * K, H) and y.dtype == torch.float32
    assert L.combine(y, inv).shape == (T, H)
    n_ok = len(calls)

    bad = [
        lambda: L.forward(x.float(), wr, bias),                                     # x not bf16
        lambda: L.forward(x[:, :128], wr, bias),                                    # wrong hidden size
        lambda: L.forward(x, wr.t().contiguous().t(), bias),                        # w_router not row-major
        lambda: L.forward(x, wr[:4], bias),                                         # wrong expert count
        lambda: L.forward(x, wr, bias.double()),                                    # bias not fp32
        lambda: L.forward(x, wr, bias, out=torch.empty((T, H), dtype=torch.float32)),
        lambda: L.forward(x, wr, bias, ws=torch.empty(16, dtype=torch.uint8)),      # workspace too small
        lambda: L.forward(x[0], wr, bias),                                          # 1-D x
        lambda: L.permute(idx.long()),
        lambda: L.permute(idx[:, :1].contiguous()),
        lambda: L.expert_ffn(x, ps[:-1], pk, offsets, w),
        lambda: L.combine(y[:, :128].contiguous(), inv),
        lambda: L.register(8, torch.zeros((2 * I, H), dtype=torch.bfloat16), torch.zeros((H, I), dtype=torch.bfloat16)),
        lambda: L.register(0, torch.zeros((H, I), dtype=torch.bfloat16), torch.zeros((H, I), dtype=torch.bfloat16)),
        lambda: L.register(0, torch.zeros((2 * I, H), dtype=torch.bfloat16), torch.zeros((H, I), dtype=torch.bfloat16),
                           torch.zeros((2, 2)), None),                              # scales on bf16 experts
        lambda: L.register(0, torch.zeros((2 * I, H), dtype=torch.bfloat16), torch.zeros((H, I), dtype=torch.bfloat16),
                           location=B.MOE_LOC_HOST_PINNED),                         # host weights, not pinned
        lambda: L.register(0, torch.zeros((2 * I, H), dtype=torch.bfloat16), torch.zeros((H, I), dtype=torch.bfloat16),
                           location=7),
    ]
    for i, f in enumerate(bad):
        with pytest.raises((TypeError, ValueError)):
            f()
        assert len(calls) == n_ok, f"bad call {i} reached the C ABI"

    F = layer(B.MOE_FP8_E4M3_B128)
    qg, qd = torch.zeros((2 * I, H), dtype=torch.uint8), torch.zeros((H, I), dtype=torch.uint8)
    sg, sd = torch.zeros((2 * I // 128, H // 128)), torch.zeros((H // 128, I // 128))
    F.register(0, qg, qd, sg, sd)
    with pytest.raises(TypeError):
        F.register(0, qg, qd, sg.double(), sd)
    with pytest.raises(TypeError):
        F.register(0, qg, qd, None, sd)


def test_allocation_failure_hook_argument_checks(lib):
    """The host-side allocation hook (moe_debug_fail_allocs) refuses unknown
    kinds and negative counts, and arming or disarming it needs no device."""
    import mixture_experts_layer_24_b200 as M
    for args in ((-1, 0, 1), (3, 0, 1), (0, -1, 1), (0, 0, -1)):
        with pytest.raises(M.MoeError) as ei:
            M.moe_debug_fail_allocs(*args)
        assert ei.value.status == 1  # MOE_ERR_INVALID_ARG
    M.moe_debug_fail_allocs(M.MOE_ALLOC_PINNED, 2, 1)
    M.moe_debug_fail_allocs(M.MOE_ALLOC_ANY, 0, 0)  # disarmed
