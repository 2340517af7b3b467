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
    assert M.MOE_SLOTS_LRU != M.MOE_SLOTS_PER_CALL


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
