"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the
fp64 oracle on the same inputs, and compare.  Only the seeded inputs are shared."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_gemm_b200 import inputs as I
from routing_dispatch_expert_gemm_b200 import native as N

NEAR_TIE = 1e-4       # top-k margin under which a token's ids may legitimately differ
GATE_ATOL = 1e-5      # fp32 gates against fp64
BF16_REL = 2e-2       # max|err| <= 2e-2 * max|y_oracle| for bf16 with fp32 accumulation
F32_REL = 1e-4        # max|err| <= 1e-4 * max|y_oracle| for the fp32 configuration


def oracle_capacity(wl: I.Workload):
    return None if wl.phi is None else O.capacity(wl.T, wl.k, wl.E, *wl.phi)


def config_for(wl: I.Workload, capacity=None, stats=False, tiles="auto",
               fuse="none") -> N.MoeConfig:
    """The GPU-side config; capacity from the library's own moe_capacity."""
    if capacity is None:
        capacity = -1 if wl.phi is None else N.moe_capacity(wl.T, wl.k, wl.E, *wl.phi)
    return N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, dtype=wl.dtype, gate_mode=wl.gate_mode,
                         capacity=capacity, has_shared=wl.has_shared, add_residual=wl.add_residual,
                         stats=stats, layout=wl.layout, overflow=wl.overflow, tiles=tiles,
                         fuse=fuse)


def oracle_params(p: dict) -> dict:
    """The oracle reads the same tensors (converted to fp64 where it uses them)."""
    return {k: v for k, v in p.items()}


def forward_gpu(cfg, x, p, ws=None):
    """moe_forward; returns y and the routing metadata as torch tensors on the GPU."""
    dev = x.device
    T, k, E = cfg.T, cfg.k, cfg.E
    ws = N.workspace(cfg) if ws is None else ws
    y = torch.empty_like(x)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    demand = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 2, dtype=torch.int32, device=dev)
    N.moe_forward(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"], p["w_down"],
                  p["shared_gate"], p["shared_up"], p["shared_down"], y, ids, gates, demand,
                  offsets, ws)
    status = N.moe_get_device_status(ws)
    return dict(y=y, ids=ids, gates=gates, demand=demand, offsets=offsets, status=status, ws=ws)


def staged_gpu(cfg, x, p, ids, gates, ws=None):
    """moe_dispatch -> moe_expert_ffn -> moe_combine on a given routing."""
    dev = x.device
    T, k, E = cfg.T, cfg.k, cfg.E
    ws = N.workspace(cfg) if ws is None else ws
    rmax = N.moe_max_rows(cfg)
    rows_h = rmax + (T if cfg.has_shared else 0)
    xp = torch.empty((rmax, cfg.d), dtype=x.dtype, device=dev)
    row_token = torch.full((rmax,), -7, dtype=torch.int32, device=dev)
    route_row = torch.empty((T, k), dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 2, dtype=torch.int32, device=dev)
    demand = torch.empty(E, dtype=torch.int32, device=dev)
    N.moe_dispatch(cfg, x, ids, None, xp, row_token, route_row, offsets, demand, ws)
    h = torch.empty((rows_h, cfg.d_ff), dtype=x.dtype, device=dev)
    yp = torch.empty((rows_h, cfg.d), dtype=x.dtype, device=dev)
    N.moe_expert_ffn(cfg, x, xp, offsets, p["w_gate"], p["w_up"], p["w_down"], p["shared_gate"],
                     p["shared_up"], p["shared_down"], h, yp, ws)
    y = torch.empty_like(x)
    N.moe_combine(cfg, yp, route_row, gates, offsets, x if cfg.add_residual else None, y)
    status = N.moe_get_device_status(ws)
    return dict(y=y, x_packed=xp, row_token=row_token, route_row=route_row, offsets=offsets,
                demand=demand, h=h, y_packed=yp, status=status)


def err_bound(y_gpu, y_ref: np.ndarray, dtype: str):
    y = y_gpu.detach().to("cpu", torch.float64).numpy() if hasattr(y_gpu, "detach") else y_gpu
    err = float(np.max(np.abs(y - y_ref))) if y_ref.size else 0.0
    scale = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    rel = BF16_REL if dtype == "bf16" else F32_REL
    return err, rel * scale


def assert_close(y_gpu, y_ref, dtype, what=""):
    err, bound = err_bound(y_gpu, y_ref, dtype)
    assert err <= bound, f"{what}: max|err| {err:.3e} > bound {bound:.3e}"
    return err, bound


def order_margin(z, k):
    """Smallest gap between consecutive logits among the k+1 largest of each token.

    Any change of the ordered top-k list (a different set, or the same set in another
    order) needs a perturbation of the logits at least this large."""
    s = -np.sort(-np.asarray(z, dtype=np.float64), axis=1)[:, :k + 1]
    if s.shape[1] < 2:
        return np.full(s.shape[0], np.inf)
    return np.min(s[:, :-1] - s[:, 1:], axis=1)


def ids_agree(ids_gpu, ids_ref, margin, z=None, k=None):
    """Per token: GPU ids equal the oracle's ordered ids exactly.

    Excluded and counted: tokens whose k-th and (k+1)-th oracle logits are within NEAR_TIE
    (``margin``), and, when the logits ``z`` are given, tokens whose top-k SET agrees but
    whose order differs between two selected logits that are within NEAR_TIE of each other
    (several orders are then correct)."""
    g = ids_gpu.cpu().numpy().astype(np.int64)
    ok = (g == ids_ref).all(axis=1)
    near = margin < NEAR_TIE
    if z is not None:
        same_set = np.array([set(a) == set(b) for a, b in zip(g, ids_ref)])
        near |= same_set & (order_margin(z, k) < NEAR_TIE)
    bad = np.where(~ok & ~near)[0]
    return bad, int((near & ~ok).sum()), ok   # count: near-tie tokens that did differ
