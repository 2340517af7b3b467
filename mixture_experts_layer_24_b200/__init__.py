"""B200 (sm_100a) routed Mixture-of-Experts layer forward.

The compute lives in ``libmoe.so`` (hand-written CUDA for sm_100a behind the C
ABI in ``include/moe.h``); this package is argument marshalling only:

* :mod:`.binding` -- ctypes declarations of every C entry point plus thin
  wrappers that take torch tensors (PyTorch supplies device memory and
  streams, nothing else).
* :mod:`.build`   -- nvcc build of ``libmoe.so`` in-tree.
* :mod:`.ep`      -- the expert-parallel schedule over several GPUs (which
  libmoe call comes when, and the NCCL all-to-alls between them).

Importing the package does not load the library; the first call of a binding
function does, and raises if ``libmoe.so`` is missing (there is no fallback).
"""

from .binding import (  # noqa: F401
    MOE_BF16,
    MOE_FP8_E4M3_B128,
    MOE_MXFP4,
    MOE_LOC_HBM,
    MOE_LOC_HOST_PINNED,
    MOE_SLOTS_LRU,
    MOE_SLOTS_PER_CALL,
    MoeError,
    MoeLayer,
    lib,
    moe_combine,
    moe_ctx_create,
    moe_ctx_destroy,
    MOE_ALLOC_ANY,
    MOE_ALLOC_DEVICE,
    MOE_ALLOC_PINNED,
    moe_debug_fail_allocs,
    moe_debug_wait_flag,
    moe_ep_gather_rows,
    moe_ep_pack,
    moe_ep_recv_plan,
    moe_expert_ffn,
    moe_forward,
    moe_get_device_status,
    moe_launch_count,
    moe_permute,
    moe_plan_hot_set,
    moe_profile_enable,
    moe_profile_read,
    moe_quantize_e4m3,
    moe_quantize_mx,
    moe_route,
    moe_route_noalloc,
    moe_slots_create,
    moe_slots_destroy,
    moe_slots_query,
    moe_slots_register,
    moe_slots_set_policy,
    moe_slots_stats,
    moe_workspace_size,
)
