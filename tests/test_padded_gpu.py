"""The padded [E, C, d] dispatch buffer and the reroute overflow policy on the GPU, against
the fp64 oracle.

Bars: slot assignment (route_row, row_token incl. padding = -1, filled-slot counts, demand)
and the packed rows bit-exact; gates within 1e-5 (GATE_ATOL); layer outputs within the
bf16 bar of the other parity tests.  The reroute cascade depends on each overflowed
token's whole expert ranking, so its bit-exact tests use integer-valued router inputs
(every fp32 logit exact, so both sides rank identically, exact ties included); with
Gaussian inputs the tests check the policy's invariants instead.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_gemm_b200 import inputs as I
from routing_dispatch_expert_gemm_b200 import native as N

from harness import GATE_ATOL, assert_close, oracle_capacity

pytestmark = pytest.mark.gpu
W = I.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from routing_dispatch_expert_gemm_b200 import build
    build.build()
    N.lib()


def _buffers(cfg, d, dtype, dev="cuda"):
    rmax = N.moe_max_rows(cfg)
    return dict(x_packed=torch.zeros((rmax, d), dtype=dtype, device=dev),
                row_token=torch.full((rmax,), -7, dtype=torch.int32, device=dev),
                route_row=torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev),
                offsets=torch.empty(N.offsets_len(cfg), dtype=torch.int32, device=dev),
                demand=torch.empty(cfg.E, dtype=torch.int32, device=dev))


def _dispatch(cfg, x, ids, gates, ws):
    b = _buffers(cfg, x.shape[1], x.dtype)
    N.moe_dispatch(cfg, x, ids, gates, b["x_packed"], b["row_token"], b["route_row"],
                   b["offsets"], b["demand"], ws)
    b["status"] = N.moe_get_device_status(ws)
    return b


def _check_against(b, ref, x, E, C):
    assert b["status"] == 0
    off = b["offsets"].cpu().numpy()
    assert off[:E + 1].tolist() == [e * C for e in range(E + 1)]
    assert off[E + 2:].tolist() == ref["counts"].tolist()
    assert b["demand"].cpu().numpy().tolist() == ref["demand"].tolist()
    assert b["route_row"].cpu().numpy().tolist() == ref["route_row"].tolist()
    assert b["row_token"].cpu().numpy()[:E * C].tolist() == ref["row_token"].tolist()
    filled = np.where(ref["row_token"] >= 0)[0]
    got = b["x_packed"][torch.from_numpy(filled).cuda()].cpu()
    want = x.cpu()[torch.from_numpy(ref["row_token"][filled])]
    assert torch.equal(got.view(torch.int16) if got.dtype == torch.bfloat16 else got,
                       want.view(torch.int16) if want.dtype == torch.bfloat16 else want)


# ------------------------------------------------------------------------- drop policy

@pytest.mark.parametrize("T,E,k,skew,C", [
    (37, 8, 2, 1.5, 3), (300, 32, 8, 2.0, 40), (4096, 4, 1, 1.0, 512), (4096, 64, 2, 1.2, 128),
    (1000, 64, 2, 0.0, 0), (200, 16, 16, 0.5, 150), (5, 4, 2, 0.0, 7), (1, 1, 1, 0.0, 1)])
def test_padded_dispatch_bit_exact(T, E, k, skew, C):
    d = 128
    ids = I.random_ids(T, E, k, seed=T + E, skew=skew)
    x = torch.randn((T, d), generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).cuda()
    cfg = N.make_config(T, d, E, k, 128, capacity=C, layout="padded")
    b = _dispatch(cfg, x, ids.cuda(), None, N.workspace(cfg))
    _check_against(b, O.dispatch_padded(ids.numpy(), None, E, C), x, E, C)


# ------------------------------------------------------------------------- reroute, exact logits

REROUTE_CASES = {
    # name: (T, d, E, k, phi, bias, gate_mode, dtype)
    "E4_k1_skewed": (512, 128, 4, 1, (1, 1), [2, 0, 0, -2], "softmax_topk", "bf16"),
    "E8_k2_renorm": (600, 256, 8, 2, (1, 1), [3, 2, 1, 0, 0, 0, -1, -2], "softmax_topk_renorm", "bf16"),
    "E8_k2_topk_softmax_phi125": (999, 128, 8, 2, (5, 4), [60, 0, 0, 0, 0, 0, 0, 0], "topk_softmax", "bf16"),
    "E40_k6": (700, 128, 40, 6, (1, 1), None, "topk_softmax", "bf16"),
    "E100_k4_general_path": (300, 128, 100, 4, (1, 1), [1] * 10 + [0] * 90, "softmax_topk_renorm", "bf16"),
    "E200_k8_tight": (257, 128, 200, 8, (1, 2), None, "softmax_topk", "bf16"),
    "fp32_router": (200, 64, 6, 2, (1, 1), [2, 1, 0, 0, 0, -1], "softmax_topk_renorm", "f32"),
    "C0": (64, 128, 4, 2, (0, 1), None, "topk_softmax", "bf16"),
    # 16384 routes, many overflowing: a long cascade of placement phases
    "E16_k4_many_phases": (4096, 128, 16, 4, (1, 1), [3, 2, 1] + [0] * 13, "softmax_topk_renorm", "bf16"),
    # 24000 routes: above what the placement keeps in shared memory, so its pending-route
    # arrays live in global memory
    "E16_k4_global_arrays": (6000, 128, 16, 4, (1, 1), [2, 2, 1] + [0] * 13, "topk_softmax", "bf16"),
}


def _reroute_case(name):
    T, d, E, k, phi, bias, mode, dtype = REROUTE_CASES[name]
    wl = I.Workload(name=name, T=T, d=d, E=E, k=k, d_ff=128, dtype=dtype, gate_mode=mode, phi=phi)
    x, w, b = I.integer_router(wl, seed=T, device="cuda", bias=bias)
    C = O.capacity(T, k, E, *phi)
    return wl, x, w, b, C


@pytest.mark.parametrize("name", list(REROUTE_CASES))
def test_reroute_dispatch_exact_logits(name):
    wl, x, w, b, C = _reroute_case(name)
    E, k = wl.E, wl.k
    cfg = N.make_config(wl.T, wl.d, E, k, 128, dtype=wl.dtype, gate_mode=wl.gate_mode,
                        capacity=C, layout="padded", overflow="reroute")
    ws = N.workspace(cfg)
    ids = torch.empty((wl.T, k), dtype=torch.int32, device="cuda")
    gates = torch.empty((wl.T, k), dtype=torch.float32, device="cuda")
    N.moe_route(cfg, x, w, b, ids, gates, ws)
    g_route = gates.clone()
    buf = _dispatch(cfg, x, ids, gates, ws)

    ids_ref, g_ref, z = O.route(x, w, b, k, wl.gate_mode)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)            # exact logits: exact ids
    ref = O.dispatch_padded(ids_ref, z, E, C, O.OVERFLOW_REROUTE)
    _check_against(buf, ref, x, E, C)
    moved = ref["rerouted"].any(axis=1)
    if name != "C0":
        assert moved.any(), "the case should exercise the reroute"
    g = gates.cpu().numpy().astype(np.float64)
    g_want = O.reroute_gates(z, ref["final_ids"], g_ref, ref["rerouted"], wl.gate_mode)
    assert np.max(np.abs(g - g_want)) <= GATE_ATOL
    # tokens without a moved route keep the router's gates bit for bit
    assert torch.equal(gates[torch.from_numpy(~moved).cuda()], g_route[torch.from_numpy(~moved).cuda()])


@pytest.mark.parametrize("overflow", ["drop", "reroute"])
def test_padded_forward_parity(overflow):
    """Whole layer through the padded buffer (both policies) against the oracle, with exact
    router logits, Gaussian experts and the shared expert (residual off, so that the
    comparison sees the experts' contribution)."""
    wl = W["shared64_T256_phi1"].with_(T=300, d=512, d_ff=1024)
    x_g, (p,) = I.make_inputs(wl, seed=3, device="cuda", layers=1)
    x, w, b = I.integer_router(wl, seed=5, device="cuda", bias=[2] * 8 + [0] * 56)
    p = dict(p, w_router=w, logit_bias=b)
    C = oracle_capacity(wl)
    cfg = N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, gate_mode=wl.gate_mode, capacity=C,
                        has_shared=True, layout="padded", overflow=overflow)
    ws = N.workspace(cfg)
    y = torch.empty_like(x)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    offsets = torch.empty(N.offsets_len(cfg), dtype=torch.int32, device="cuda")
    N.moe_forward(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"], p["w_down"],
                  p["shared_gate"], p["shared_up"], p["shared_down"], y, ids, gates, None,
                  offsets, ws)
    assert N.moe_get_device_status(ws) == 0
    y_ref, info = O.moe_layer(x, p, wl.k, wl.gate_mode, C, layout="padded", overflow=overflow)
    assert np.array_equal(ids.cpu().numpy(), info["ids"])
    assert offsets.cpu().numpy()[wl.E + 2:].tolist() == info["counts"].tolist()
    if overflow == "reroute":
        assert info["rerouted"].any()
    assert np.max(np.abs(gates.cpu().numpy() - info["gates"])) <= GATE_ATOL
    assert_close(y, y_ref, "bf16", f"padded/{overflow}")
    # the layout alone changes no bit of the output
    if overflow == "drop":
        cfg_r = N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, gate_mode=wl.gate_mode,
                              capacity=C, has_shared=True)
        y_r = torch.empty_like(x)
        N.moe_forward(cfg_r, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"],
                      p["w_down"], p["shared_gate"], p["shared_up"], p["shared_down"], y_r,
                      None, None, None, None, N.workspace(cfg_r))
        assert torch.equal(y, y_r)


# ------------------------------------------------------------------------- Gaussian inputs

@pytest.mark.parametrize("name", ["switch_phi050", "switch_phi125", "shared64_T4096_phi1"])
def test_reroute_invariants(name):
    """Full-size layers with Gaussian inputs: the reroute result obeys the policy's rules
    (checked on the GPU's own routing), keeps at least the drop policy's routes, and
    repeats bit for bit."""
    wl = W[name]
    x, (p,) = I.make_inputs(wl, seed=0, device="cuda", layers=1)
    C = oracle_capacity(wl)
    drop = N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, gate_mode=wl.gate_mode, capacity=C,
                         has_shared=wl.has_shared, layout="padded", stats=True)
    rr = N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, gate_mode=wl.gate_mode, capacity=C,
                       has_shared=wl.has_shared, layout="padded", overflow="reroute", stats=True)
    outs = {}
    for tag, cfg in (("drop", drop), ("rr", rr), ("rr2", rr)):
        ws = N.workspace(cfg)
        y = torch.empty_like(x)
        ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        gates = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        offsets = torch.empty(N.offsets_len(cfg), dtype=torch.int32, device="cuda")
        N.moe_forward(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"],
                      p["w_down"], p["shared_gate"], p["shared_up"], p["shared_down"], y, ids,
                      gates, None, offsets, ws)
        summ = torch.zeros(32, dtype=torch.uint8, device="cuda")
        N.moe_routing_stats(cfg, None, offsets, 1e-2, None, None, summ, ws)
        assert N.moe_get_device_status(ws) == 0
        outs[tag] = dict(y=y, ids=ids.cpu().numpy(), gates=gates, summ=N.summary_dict(summ),
                         counts=offsets.cpu().numpy()[wl.E + 2:])
    a, r = outs["drop"], outs["rr"]
    assert torch.equal(r["y"], outs["rr2"]["y"]) and torch.equal(r["gates"], outs["rr2"]["gates"])
    assert np.array_equal(a["ids"], r["ids"])
    assert (r["counts"] <= C).all() and r["counts"].sum() >= a["counts"].sum()
    assert r["summ"]["kept"] == int(r["counts"].sum()) and a["summ"]["kept"] == int(a["counts"].sum())
    assert r["summ"]["padding_rate"] == np.float32((wl.E * C - r["counts"].sum()) / (wl.E * C))
    # the oracle's own reroute must give the same filled-slot counts when the GPU chose the
    # same expert set for every token and no overflowed token has two logits within 1e-4
    # (otherwise two rankings are both correct)
    ids_ref, _, z = O.route(x, p["w_router"], p["logit_bias"], wl.k, wl.gate_mode)
    ref = O.dispatch_padded(ids_ref, z, wl.E, C, O.OVERFLOW_REROUTE)
    over = (O.dispatch_padded(ids_ref, None, wl.E, C)["route_row"] < 0).any(axis=1)
    s = -np.sort(-z, axis=1)
    gap = np.min(s[:, :-1] - s[:, 1:], axis=1)
    same_sets = np.array_equal(np.sort(r["ids"], axis=1), np.sort(ids_ref, axis=1))
    if same_sets and (gap[over] > 1e-4).all():
        assert r["counts"].tolist() == ref["counts"].tolist()
    assert int(ref["rerouted"].sum()) > 0


@pytest.mark.parametrize("overflow", ["drop", "reroute"])
def test_padded_forward_parity_fp32(overflow):
    """The fp32 layer (CUDA-core router and grouped GEMMs) through the padded buffer: the
    GEMMs compute only each expert's filled slots."""
    wl = W["tiny_fp32"].with_(T=96, E=6, k=2, phi=(1, 1))
    x_g, (p,) = I.make_inputs(wl, seed=2, device="cuda", layers=1)
    x, w, b = I.integer_router(wl, seed=8, device="cuda", bias=[3, 2, 0, 0, -1, -2])
    p = dict(p, w_router=w, logit_bias=b)
    C = oracle_capacity(wl)
    cfg = N.make_config(wl.T, wl.d, wl.E, wl.k, wl.d_ff, dtype="f32", gate_mode=wl.gate_mode,
                        capacity=C, layout="padded", overflow=overflow)
    ws = N.workspace(cfg)
    y = torch.empty_like(x)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    offsets = torch.empty(N.offsets_len(cfg), dtype=torch.int32, device="cuda")
    N.moe_forward(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"], p["w_down"],
                  None, None, None, y, ids, gates, None, offsets, ws)
    assert N.moe_get_device_status(ws) == 0
    y_ref, info = O.moe_layer(x, p, wl.k, wl.gate_mode, C, layout="padded", overflow=overflow)
    assert np.array_equal(ids.cpu().numpy(), info["ids"])
    assert offsets.cpu().numpy()[wl.E + 2:].tolist() == info["counts"].tolist()
    assert int(info["counts"].sum()) < wl.T * wl.k or overflow == "reroute"
    if overflow == "reroute":
        assert info["rerouted"].any()
    assert np.max(np.abs(gates.cpu().numpy() - info["gates"])) <= GATE_ATOL
    assert_close(y, y_ref, "f32", f"padded fp32/{overflow}")
