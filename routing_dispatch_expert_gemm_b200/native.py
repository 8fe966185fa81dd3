"""Thin ctypes binding of libmoe.so: the C ABI of include/moe.h under the same names.

Argument marshalling only: torch tensors become device pointers, ``None`` becomes NULL,
the stream defaults to torch's current stream.  Every step of the path runs in the CUDA
kernels of libmoe.so; there is no CPU fallback.  If the library is missing the first call
raises ``ImportError`` (build it with ``routing_dispatch_expert_gemm_b200.build.build()``).
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_OK = 0
ABI_VERSION = 5  # moe_abi_version() of the library this binding mirrors
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_BAD_EXPERT_ID",
                6: "MOE_ERR_TIMEOUT"}
DTYPES = {"f32": 0, "bf16": 1}
GATE_MODES = {"softmax_topk": 0, "softmax_topk_renorm": 1, "topk_softmax": 2}
LAYOUTS = {"ragged": 0, "padded": 1}
OVERFLOWS = {"drop": 0, "reroute": 1}
TILES = {"auto": 0, "rows": 1, "columns": 2, "pairs": 3, "row_pairs": 4}
FUSE = {"none": 0, "gather": 1, "combine": 2, "gather+combine": 3}

# Every symbol include/moe.h declares (checked by the CPU test suite).
EXPORTS = ("moe_capacity", "moe_max_rows", "moe_workspace_bytes", "moe_workspace_init",
           "moe_ffn_tile_shape", "moe_ffn_launches",
           "moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_forward",
           "moe_forward_profiled", "moe_get_device_status", "moe_debug_bounded_wait",
           "moe_dispatch_noalloc", "moe_routing_stats", "moe_status_string",
           "moe_abi_version")


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({moe_status_string(code)})")


class MoeConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "d", "E", "k", "d_ff", "dtype", "gate_mode", "capacity",
                 "has_shared", "add_residual", "stats", "layout", "overflow", "tiles",
                 "fuse")]

    def __repr__(self):
        return "MoeConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_config(T, d, E, k, d_ff, dtype="bf16", gate_mode="topk_softmax", capacity=-1,
                has_shared=False, add_residual=False, stats=False, layout="ragged",
                overflow="drop", tiles="auto", fuse="none") -> MoeConfig:
    return MoeConfig(int(T), int(d), int(E), int(k), int(d_ff), DTYPES[dtype],
                     GATE_MODES[gate_mode], int(capacity), int(bool(has_shared)),
                     int(bool(add_residual)), int(bool(stats)), LAYOUTS[layout],
                     OVERFLOWS[overflow], TILES[tiles], FUSE[fuse])


def offsets_len(cfg: MoeConfig) -> int:
    """Entries of the segment table moe_dispatch writes: E + 2, plus E filled-slot counts
    with the padded layout."""
    return cfg.E + 2 + (cfg.E if cfg.layout == LAYOUTS["padded"] else 0)


class MoeRoutingSummary(ctypes.Structure):
    """moe_routing_summary; moe_routing_stats writes one into device memory."""
    _fields_ = [("aux_loss", ctypes.c_float), ("imbalance", ctypes.c_float),
                ("drop_rate", ctypes.c_float), ("padding_rate", ctypes.c_float),
                ("kept", ctypes.c_int32), ("dropped", ctypes.c_int32),
                ("max_demand", ctypes.c_int32), ("busiest_expert", ctypes.c_int32)]


def summary_dict(buf) -> dict:
    """Decode a moe_routing_summary copied to the host (bytes, or a uint8 tensor/array)."""
    raw = bytes(buf.cpu().numpy().tobytes()) if hasattr(buf, "cpu") else bytes(buf)
    s = MoeRoutingSummary.from_buffer_copy(raw[:ctypes.sizeof(MoeRoutingSummary)])
    return {n: getattr(s, n) for n, _ in s._fields_}


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_CFG = ctypes.POINTER(MoeConfig)


def lib() -> ctypes.CDLL:
    """Load libmoe.so once; raise loudly if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m routing_dispatch_expert_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "moe_capacity": (_I32, [_I32] * 5),
            "moe_max_rows": (ctypes.c_int64, [_CFG]),
            "moe_workspace_bytes": (ctypes.c_size_t, [_CFG]),
            "moe_workspace_init": (_I32, [_P, _P]),
            "moe_ffn_tile_shape": (_I32, [_CFG]),
            "moe_ffn_launches": (_I32, [_CFG]),
            "moe_route": (_I32, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
            "moe_dispatch": (_I32, [_CFG] + [_P] * 10),
            "moe_expert_ffn": (_I32, [_CFG] + [_P] * 12 + [_P]),
            "moe_combine": (_I32, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
            "moe_forward": (_I32, [_CFG] + [_P] * 15 + [_P]),
            "moe_forward_profiled": (_I32, [_CFG] + [_P] * 14 + [ctypes.POINTER(_P), _I32, _P, _P]),
            "moe_get_device_status": (_I32, [_P, _P, _I32, ctypes.POINTER(_I32)]),
            "moe_debug_bounded_wait": (_I32, [_P, ctypes.c_int64, _P]),
            "moe_dispatch_noalloc": (_I32, [_CFG] + [_P] * 8 + [_P]),
            "moe_routing_stats": (_I32, [_CFG, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P]),
            "moe_status_string": (ctypes.c_char_p, [_I32]),
            "moe_abi_version": (_I32, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        if L.moe_abi_version() != ABI_VERSION:
            raise ImportError(f"{LIB_PATH} has ABI version {L.moe_abi_version()}, the binding "
                              f"expects {ABI_VERSION}: rebuild the library")
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoeError(code, where)


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_capacity(T, k, E, phi_num, phi_den) -> int:
    return lib().moe_capacity(T, k, E, phi_num, phi_den)


def moe_max_rows(cfg: MoeConfig) -> int:
    return lib().moe_max_rows(ctypes.byref(cfg))


def moe_ffn_tile_shape(cfg: MoeConfig) -> str:
    """'rows', 'columns', 'pairs' or 'row_pairs': the FFN tile shape the config runs with."""
    v = lib().moe_ffn_tile_shape(ctypes.byref(cfg))
    if v == 0:
        raise MoeError(1, "moe_ffn_tile_shape")
    return {1: "rows", 2: "columns", 3: "pairs", 4: "row_pairs"}[v]


def moe_ffn_launches(cfg: MoeConfig) -> int:
    """Kernel launches of the expert FFN for the config (2, or 4 with the shared expert's
    segment on SM pairs next to row tiles)."""
    v = lib().moe_ffn_launches(ctypes.byref(cfg))
    if v == 0:
        raise MoeError(1, "moe_ffn_launches")
    return v


def moe_workspace_bytes(cfg: MoeConfig) -> int:
    return lib().moe_workspace_bytes(ctypes.byref(cfg))


def moe_workspace_init(ws, stream=None):
    _check(lib().moe_workspace_init(_ptr(ws), _stream(stream)), "moe_workspace_init")


def moe_route(cfg, x, w_router, logit_bias, ids, gates, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(logit_bias),
                           _ptr(ids), _ptr(gates), _ptr(ws), _stream(stream)), "moe_route")


def moe_dispatch(cfg, x, ids, gates, x_packed, row_token, route_row, offsets, demand, ws,
                 stream=None):
    """``gates`` is read and rewritten with the reroute policy; otherwise it may be None."""
    _check(lib().moe_dispatch(ctypes.byref(cfg), _ptr(x), _ptr(ids), _ptr(gates),
                              _ptr(x_packed), _ptr(row_token), _ptr(route_row), _ptr(offsets),
                              _ptr(demand), _ptr(ws), _stream(stream)), "moe_dispatch")


def moe_expert_ffn(cfg, x, x_packed, offsets, w_gate, w_up, w_down, shared_gate, shared_up,
                   shared_down, h, y_packed, ws, stream=None):
    _check(lib().moe_expert_ffn(ctypes.byref(cfg), _ptr(x), _ptr(x_packed), _ptr(offsets),
                                _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(shared_gate),
                                _ptr(shared_up), _ptr(shared_down), _ptr(h), _ptr(y_packed),
                                _ptr(ws), _stream(stream)), "moe_expert_ffn")


def moe_combine(cfg, y_packed, route_row, gates, offsets, residual, y, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _ptr(y_packed), _ptr(route_row), _ptr(gates),
                             _ptr(offsets), _ptr(residual), _ptr(y), _stream(stream)),
           "moe_combine")


def moe_forward(cfg, x, w_router, logit_bias, w_gate, w_up, w_down, shared_gate, shared_up,
                shared_down, y, ids_out, gates_out, demand_out, offsets_out, ws, stream=None):
    _check(lib().moe_forward(ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(logit_bias),
                             _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(shared_gate),
                             _ptr(shared_up), _ptr(shared_down), _ptr(y), _ptr(ids_out),
                             _ptr(gates_out), _ptr(demand_out), _ptr(offsets_out), _ptr(ws),
                             _stream(stream)), "moe_forward")


def moe_forward_profiled(cfg, x, w_router, logit_bias, w_gate, w_up, w_down, shared_gate,
                         shared_up, shared_down, y, ids_out, gates_out, demand_out, offsets_out,
                         events, ws, stream=None):
    """``events``: six (or seven) torch.cuda.Event objects, or raw cudaEvent_t handles as
    ints; see moe_forward_profiled in include/moe.h."""
    for e in events:  # torch creates an event's handle at its first record
        if not isinstance(e, int) and e.cuda_event == 0:
            e.record()
    handles = (_P * len(events))(*[e if isinstance(e, int) else e.cuda_event for e in events])
    _check(lib().moe_forward_profiled(ctypes.byref(cfg), _ptr(x), _ptr(w_router),
                                      _ptr(logit_bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                      _ptr(shared_gate), _ptr(shared_up), _ptr(shared_down),
                                      _ptr(y), _ptr(ids_out), _ptr(gates_out), _ptr(demand_out),
                                      _ptr(offsets_out), handles, len(events), _ptr(ws),
                                      _stream(stream)), "moe_forward_profiled")


def moe_get_device_status(ws, stream=None, clear=False) -> int:
    out = _I32(0)
    _check(lib().moe_get_device_status(_ptr(ws), _stream(stream), int(bool(clear)),
                                       ctypes.byref(out)), "moe_get_device_status")
    return out.value


def moe_debug_bounded_wait(ws, limit_ns, stream=None):
    _check(lib().moe_debug_bounded_wait(_ptr(ws), int(limit_ns), _stream(stream)),
           "moe_debug_bounded_wait")


def moe_dispatch_noalloc(cfg, x, ids, x_packed, row_token, route_row, offsets, demand,
                         status=None, stream=None):
    """moe_dispatch without a workspace: for callers that cannot allocate device memory.
    Its scratch is a fixed array inside libmoe.so (see include/moe.h)."""
    _check(lib().moe_dispatch_noalloc(ctypes.byref(cfg), _ptr(x), _ptr(ids), _ptr(x_packed),
                                      _ptr(row_token), _ptr(route_row), _ptr(offsets),
                                      _ptr(demand), _ptr(status), _stream(stream)),
           "moe_dispatch_noalloc")


def moe_routing_stats(cfg, demand, offsets, alpha, f, P, summary, ws, stream=None):
    """``summary``: a device uint8 tensor of at least 32 bytes (decode with summary_dict)."""
    _check(lib().moe_routing_stats(ctypes.byref(cfg), _ptr(demand), _ptr(offsets),
                                   float(alpha), _ptr(f), _ptr(P), _ptr(summary), _ptr(ws),
                                   _stream(stream)), "moe_routing_stats")


def workspace(cfg: MoeConfig, device="cuda"):
    """Allocate (with torch) and zero-initialise a workspace for ``cfg``."""
    import torch
    n = moe_workspace_bytes(cfg)
    if n == 0:
        raise MoeError(1, "moe_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws
