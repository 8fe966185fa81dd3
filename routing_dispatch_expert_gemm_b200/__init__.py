"""MoE layer forward (route + pack + compute + combine) on one B200, sm_100a.

The work runs in libmoe.so (CUDA kernels behind a C ABI, include/moe.h); this package is
its thin ctypes binding (``native``) plus the seeded synthetic workloads (``inputs``).
"""
from .native import (  # noqa: F401
    DTYPES, EXPORTS, GATE_MODES, MoeConfig, MoeError, make_config, moe_abi_version,
    moe_capacity, moe_combine, moe_debug_bounded_wait, moe_dispatch, moe_dispatch_noalloc,
    moe_expert_ffn,
    moe_forward, moe_forward_profiled, moe_get_device_status, moe_max_rows, moe_route, moe_status_string,
    moe_workspace_bytes, moe_workspace_init, workspace,
)
