"""Routing statistics on the GPU (moe_routing_stats) against the fp64 oracle.

f, kept/dropped counts, imbalance, drop and padding rates are functions of the expert ids.
The oracle routes on its own; where the GPU chose the same expert set for every token (the
usual case) they are compared exactly: f bit-exact (the same correctly rounded quotient), the
counts exact, the rates to fp32 rounding.  Where near-tie tokens (logits within 1e-4) chose a
different set, each such token moves at most k routes, which bounds the differences.
P (mean full-softmax probability) is compared with the oracle's fp64 softmax of the same
stored inputs within P_RTOL: the kernel's logits carry fp32 accumulation error (|dz| well
under 1e-5 for these shapes), a probability moves by p * |dz| to first order, and the fp32
tile sums add a relative 128 * 2^-24.  The auxiliary value inherits P's tolerance.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_gemm_b200 import inputs as I
from routing_dispatch_expert_gemm_b200 import native as N

from harness import config_for, forward_gpu, ids_agree, oracle_capacity

pytestmark = pytest.mark.gpu
W = I.WORKLOADS
P_RTOL = 1e-4
ALPHA = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from routing_dispatch_expert_gemm_b200 import build
    build.build()
    N.lib()


CASES = {
    "tiny_fp32": W["tiny_fp32"],                                       # CUDA-core router
    "granite24": W["granite24"],                                       # E=32, top-k softmax
    "switch_phi125": W["switch_phi125"],                               # E=4, k=1, capacity
    "switch_phi050": W["switch_phi050"],                               # heavy drops
    "shared64_T4096_phi1": W["shared64_T4096_phi1"],                   # E=64, renormalised
    "mixtral_decode": W["mixtral_decode"],                             # T=16: one partial tile
    "E128_k8_T1000": W["granite24"].with_(E=128, k=8, T=1000),         # general epilogue path
    "E200_k6_T777_cap": W["granite24"].with_(E=200, k=6, T=777, phi=(1, 1),
                                             gate_mode="softmax_topk"),  # E not a multiple of 16
    "many_tiles": W["mixtral_decode"].with_(T=307200, d=128, phi=(1, 1)),  # 2400 tiles, 148 CTAs
    "T1": W["shared64_T1_phi2"],
}


def _check_against_oracle(wl, x, p, C, ids, f, P, s, demand):
    """Compare the GPU's statistics with the oracle's, computed from the oracle's own routing."""
    ref_ids, _, z = O.route(x, p["w_router"], p["logit_bias"], wl.k, wl.gate_mode)
    bad, _, _ = ids_agree(ids, ref_ids, O.topk_margin(z, wl.k), z, wl.k)
    assert len(bad) == 0
    ref = O.routing_stats(x, p["w_router"], p["logit_bias"], wl.k, C, alpha=ALPHA)
    dem_ref = O.dispatch(ref_ids, wl.E, C)["demand"]
    # P is the full softmax, whatever experts were chosen
    Pg = P.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(Pg - ref["P"]) <= P_RTOL * ref["P"] + 1e-9), np.max(np.abs(Pg - ref["P"]))
    g = ids.cpu().numpy().astype(np.int64)
    moved = int((np.sort(g, axis=1) != np.sort(ref_ids, axis=1)).any(axis=1).sum())
    dem = demand.cpu().numpy().astype(np.int64)
    Tk = wl.T * wl.k
    if moved == 0:
        assert dem.tolist() == dem_ref.tolist()
        if f is not None:
            assert np.array_equal(f.cpu().numpy(), ref["f"].astype(np.float32))
        assert abs(s["aux_loss"] - ref["aux"]) <= P_RTOL * ref["aux"] + 1e-9
        assert s["kept"] == ref["kept"] and s["dropped"] == Tk - ref["kept"]
        assert s["imbalance"] == np.float32(ref["imbalance"])
        assert s["drop_rate"] == np.float32(ref["drop_rate"])
        assert s["padding_rate"] == np.float32(ref["padding_rate"])
    else:  # each differing token shifts at most k routes between experts
        assert np.abs(dem - dem_ref).sum() <= 2 * wl.k * moved
        assert abs(s["kept"] - ref["kept"]) <= 2 * wl.k * moved
        bound = ALPHA * wl.E * float(np.sum(np.abs(dem - dem_ref) / Tk * ref["P"]))
        assert abs(s["aux_loss"] - ref["aux"]) <= P_RTOL * ref["aux"] + bound + 1e-9
    # the summary is consistent with the GPU's own counts in every case
    assert s["max_demand"] == dem.max() and s["busiest_expert"] == int(np.argmax(dem))
    assert s["dropped"] == Tk - s["kept"]
    if f is not None:
        assert np.array_equal(f.cpu().numpy(), (dem / Tk).astype(np.float32))


def _route_dispatch_stats(wl, cfg, x, p, ws):
    dev = x.device
    T, k, E = wl.T, wl.k, wl.E
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    N.moe_route(cfg, x, p["w_router"], p["logit_bias"], ids, gates, ws)
    rmax = N.moe_max_rows(cfg)
    xp = torch.empty((rmax, wl.d), dtype=x.dtype, device=dev)
    row_token = torch.empty(rmax, dtype=torch.int32, device=dev)
    route_row = torch.empty((T, k), dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 2, dtype=torch.int32, device=dev)
    demand = torch.empty(E, dtype=torch.int32, device=dev)
    N.moe_dispatch(cfg, x, ids, None, xp, row_token, route_row, offsets, demand, ws)
    f = torch.full((E,), -1.0, device=dev)
    P = torch.full((E,), -1.0, device=dev)
    summ = torch.zeros(32, dtype=torch.uint8, device=dev)
    N.moe_routing_stats(cfg, demand, offsets, ALPHA, f, P, summ, ws)
    assert N.moe_get_device_status(ws) == 0
    return ids, demand, offsets, f, P, summ


@pytest.mark.parametrize("name", list(CASES))
def test_routing_stats_parity(name):
    wl = CASES[name]
    x, (p,) = I.make_inputs(wl, seed=4, device="cuda", experts=False)
    cfg = config_for(wl, stats=True)
    ws = N.workspace(cfg)
    ids, demand, _, f, P, summ = _route_dispatch_stats(wl, cfg, x, p, ws)
    s = N.summary_dict(summ)
    _check_against_oracle(wl, x, p, oracle_capacity(wl), ids, f, P, s, demand)


def test_routing_stats_repeatable():
    """Repeated calls on one workspace give the same bits (the ticket counter is reset)."""
    wl = CASES["many_tiles"].with_(T=40000)
    x, (p,) = I.make_inputs(wl, seed=1, device="cuda", experts=False)
    cfg = config_for(wl, stats=True)
    ws = N.workspace(cfg)
    _, demand, offsets, f1, P1, s1 = _route_dispatch_stats(wl, cfg, x, p, ws)
    for _ in range(2):
        f2, P2, s2 = torch.empty_like(f1), torch.empty_like(P1), torch.zeros_like(s1)
        N.moe_routing_stats(cfg, demand, offsets, ALPHA, f2, P2, s2, ws)
        assert torch.equal(f1, f2) and torch.equal(P1, P2) and torch.equal(s1, s2)
    assert N.moe_get_device_status(ws) == 0


def test_forward_with_stats():
    """cfg.stats changes no output of moe_forward, and moe_routing_stats with NULL demand /
    offsets reads the copies moe_forward kept in the workspace."""
    wl = W["granite24"].with_(layers=1, T=700, phi=(1, 1))
    x, (p,) = I.make_inputs(wl, seed=3, device="cuda", layers=1)
    plain = forward_gpu(config_for(wl), x, p)
    cfg = config_for(wl, stats=True)
    ws = N.workspace(cfg)
    withs = forward_gpu(cfg, x, p, ws)
    for key in ("y", "ids", "gates", "demand", "offsets"):
        assert torch.equal(plain[key], withs[key]), key
    # forward again without the *_out copies, so that demand/offsets stay in the workspace
    y = torch.empty_like(x)
    N.moe_forward(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"], p["w_down"],
                  None, None, None, y, None, None, None, None, ws)
    assert torch.equal(y, plain["y"])
    f = torch.empty(wl.E, device="cuda")
    P = torch.empty(wl.E, device="cuda")
    summ = torch.zeros(32, dtype=torch.uint8, device="cuda")
    N.moe_routing_stats(cfg, None, None, ALPHA, f, P, summ, ws)
    f_ref = torch.empty_like(f)
    summ_ref = torch.zeros_like(summ)
    N.moe_routing_stats(cfg, withs["demand"], withs["offsets"], ALPHA, f_ref, None, summ_ref, ws)
    assert N.moe_get_device_status(ws) == 0
    assert torch.equal(f, f_ref) and torch.equal(summ, summ_ref)
    s = N.summary_dict(summ)
    _check_against_oracle(wl, x, p, oracle_capacity(wl), plain["ids"], f, P, s, plain["demand"])
