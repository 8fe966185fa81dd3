"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on seeded inputs.

Bars: expert ids, packed positions, offsets, drop masks and packed rows bit-exact (tokens
whose k-th and (k+1)-th oracle logits are closer than 1e-4 are excluded from the id
comparison and counted); gates within 1e-5; outputs within max|err| <= 2e-2 max|y_oracle|
(bf16, fp32 accumulation) or 1e-4 max|y_oracle| (fp32 configuration).
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from routing_dispatch_expert_gemm_b200 import inputs as I
from routing_dispatch_expert_gemm_b200 import native as N

from harness import (GATE_ATOL, assert_close, config_for, forward_gpu, ids_agree,
                     oracle_capacity, order_margin, staged_gpu)

pytestmark = pytest.mark.gpu
W = I.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from routing_dispatch_expert_gemm_b200 import build
    build.build()
    N.lib()
    torch.manual_seed(0)


# Sizes the oracle finishes in seconds, still spanning several tiles and a ragged tail.
SMALL = {
    "tiny_fp32": W["tiny_fp32"],
    "granite_layer": W["granite24"].with_(layers=1, add_residual=True),
    "switch_dropless": W["switch_dropless"],
    "switch_phi050": W["switch_phi050"],
    "switch_phi100": W["switch_phi100"],
    "switch_phi125": W["switch_phi125"],
    "mixtral_T300": W["mixtral_prefill"].with_(T=300),
    "mixtral_decode": W["mixtral_decode"],
    "shared64_narrow_phi1": W["shared64_T256_phi1"].with_(T=300, d=512, d_ff=1024),
    "shared64_narrow_dropless": W["shared64_T256_dropless"].with_(T=300, d=512, d_ff=1024),
    "shared64_narrow_phi2_T1": W["shared64_T1_phi2"].with_(d=512, d_ff=1024),
    # about 128 rows per routed expert: segments just above one 128-row tile (two tiles, the
    # second nearly empty) next to smaller and larger ones, and a 1024-row shared segment
    "shared16_narrow": W["shared16_T1024_F8192"].with_(d=512, d_ff=1024),
}


# ------------------------------------------------------------------------- route

@pytest.mark.parametrize("name", ["tiny_fp32", "granite24", "switch_dropless", "mixtral_prefill",
                                  "mixtral_decode", "shared64_T4096_dropless", "shared64_T1_phi1"])
def test_route_parity(name):
    wl = W[name]
    x, (p,) = I.make_inputs(wl, seed=0, device="cuda", experts=False)
    cfg = config_for(wl)
    ws = N.workspace(cfg)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    N.moe_route(cfg, x, p["w_router"], p["logit_bias"], ids, gates, ws)
    assert N.moe_get_device_status(ws) == 0
    ids_ref, g_ref, z = O.route(x, p["w_router"], p["logit_bias"], wl.k, wl.gate_mode)
    margin = O.topk_margin(z, wl.k)
    bad, n_near, ok = ids_agree(ids, ids_ref, margin, z, wl.k)
    assert len(bad) == 0, f"{len(bad)} tokens with different top-{wl.k} (near ties excluded: {n_near})"
    g = gates.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g[ok] - g_ref[ok])) <= GATE_ATOL
    if wl.gate_mode != "softmax_topk":
        assert np.max(np.abs(g.sum(1) - 1)) <= 1e-6


def test_route_ties_go_to_lowest_index():
    wl = W["tiny_fp32"].with_(T=40, E=8, k=3, dtype="bf16", d=128, d_ff=128)
    cfg = config_for(wl)
    x = torch.zeros((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    x[20:] = 1.0
    w = torch.zeros((wl.E, wl.d), dtype=torch.bfloat16, device="cuda")
    bias = torch.tensor([0.5, 2.0, 2.0, 0.5, 2.0, 1.0, 2.0, 0.0], device="cuda")
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    ws = N.workspace(cfg)
    N.moe_route(cfg, x, w, bias, ids, gates, ws)
    assert (ids.cpu() == torch.tensor([1, 2, 4], dtype=torch.int32)).all()
    assert torch.allclose(gates.cpu(), torch.full((wl.T, 3), 1 / 3))


# ------------------------------------------------------------------------- dispatch

@pytest.mark.parametrize("T,E,k,skew,cap", [
    (1, 4, 2, 1.0, None), (37, 8, 2, 1.5, None), (37, 8, 2, 1.5, 3), (300, 32, 8, 1.0, None),
    (300, 32, 8, 2.0, 40), (4096, 4, 1, 1.0, 512), (4096, 64, 2, 1.2, 128), (1000, 64, 2, 0.0, 0),
    (5000, 256, 4, 1.0, None), (513, 1, 1, 0.0, None), (200, 16, 16, 0.5, 150)])
def test_dispatch_bit_exact(T, E, k, skew, cap):
    d = 128
    ids = I.random_ids(T, E, k, seed=T + E, skew=skew)
    gen = torch.Generator().manual_seed(1)
    x = torch.randn((T, d), generator=gen).to(torch.bfloat16)
    cfg = N.make_config(T, d, E, k, 128, capacity=-1 if cap is None else cap)
    ws = N.workspace(cfg)
    rmax = N.moe_max_rows(cfg)
    xd, idsd = x.cuda(), ids.cuda()
    xp = torch.zeros((rmax, d), dtype=torch.bfloat16, device="cuda")
    row_token = torch.full((rmax,), -7, dtype=torch.int32, device="cuda")
    route_row = torch.empty((T, k), dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    demand = torch.empty(E, dtype=torch.int32, device="cuda")
    N.moe_dispatch(cfg, xd, idsd, None, xp, row_token, route_row, offsets, demand, ws)
    assert N.moe_get_device_status(ws) == 0
    ref = O.dispatch(ids.numpy(), E, cap)
    R = int(ref["offsets"][E])
    assert demand.cpu().numpy().tolist() == ref["demand"].tolist()
    assert offsets.cpu().numpy()[:E + 1].tolist() == ref["offsets"].tolist()
    assert int(offsets[E + 1]) == R
    assert route_row.cpu().numpy().tolist() == ref["route_row"].tolist()
    assert row_token.cpu().numpy()[:R].tolist() == ref["row_token"].tolist()
    # packed rows are byte copies of the token rows
    xp_h = xp[:R].cpu().view(torch.int16)
    assert torch.equal(xp_h, x.view(torch.int16)[torch.from_numpy(ref["row_token"])])


def test_dispatch_rejects_bad_ids():
    T, E, k, d = 20, 8, 2, 128
    ids = I.random_ids(T, E, k, seed=3)
    ids[3, 1] = 99           # out of range
    ids[5, 1] = ids[5, 0]    # repeated within a token
    ids[7, 0] = -1
    cfg = N.make_config(T, d, E, k, 128)
    ws = N.workspace(cfg)
    x = torch.randn((T, d), device="cuda").to(torch.bfloat16)
    rmax = N.moe_max_rows(cfg)
    xp = torch.empty((rmax, d), dtype=torch.bfloat16, device="cuda")
    row_token = torch.empty(rmax, dtype=torch.int32, device="cuda")
    route_row = torch.empty((T, k), dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    demand = torch.empty(E, dtype=torch.int32, device="cuda")
    N.moe_dispatch(cfg, x, ids.cuda(), None, xp, row_token, route_row, offsets, demand, ws)
    assert N.moe_get_device_status(ws, clear=True) == 5      # MOE_ERR_BAD_EXPERT_ID
    assert N.moe_get_device_status(ws) == 0
    rr = route_row.cpu()
    assert rr[3, 1] == -1 and rr[5, 1] == -1 and rr[7, 0] == -1
    assert int(demand.sum()) == T * k - 3
    assert rr[5, 0] >= 0 and rr[3, 0] >= 0


# ------------------------------------------------------------------------- whole layer

def _run_oracle_routing(wl, seed=0, tiles="auto"):
    x, (p,) = I.make_inputs(wl, seed=seed, device="cuda", layers=1)
    cfg = config_for(wl, tiles=tiles)
    C = oracle_capacity(wl)
    ids_ref, g_ref, _ = O.route(x, p["w_router"], p["logit_bias"], wl.k, wl.gate_mode)
    g32 = torch.from_numpy(g_ref.astype(np.float32))
    out = staged_gpu(cfg, x, p, torch.from_numpy(ids_ref.astype(np.int32)).cuda(), g32.cuda())
    return wl, x, p, C, ids_ref, g32, out


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_parity_on_oracle_routing(name):
    wl, x, p, C, ids_ref, g32, out = _run_oracle_routing(SMALL[name])
    assert out["status"] == 0
    y_ref, info = O.moe_layer(x, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual,
                              routing=(ids_ref, g32.double().numpy()))
    assert out["route_row"].cpu().numpy().tolist() == info["route_row"].tolist()
    assert out["offsets"].cpu().numpy()[:wl.E + 1].tolist() == info["offsets"].tolist()
    if wl.add_residual:  # the MoE contribution alone, allowing one bf16 ulp of y's rounding
        moe_ref = y_ref - O.as_f64(x)
        moe_gpu = out["y"].double().cpu().numpy() - O.as_f64(x)
        bound = 2e-2 * np.max(np.abs(moe_ref)) + 2.0 ** -8 * np.max(np.abs(y_ref))
        assert np.max(np.abs(moe_gpu - moe_ref)) <= bound
    assert_close(out["y"], y_ref, wl.dtype, name)


@pytest.mark.parametrize("tiles", ["rows", "columns", "pairs", "row_pairs"])
@pytest.mark.parametrize("name", ["granite_layer", "switch_phi125", "switch_phi050", "mixtral_T300",
                                  "mixtral_decode", "shared64_narrow_phi1",
                                  "shared64_narrow_phi2_T1", "shared16_narrow"])
def test_every_tile_shape_on_oracle_routing(name, tiles):
    """The row-tile, column-tile, column-pair and row-pair FFN kernels, forced on the same
    inputs and routing, each against the oracle (segments of 1 to a few thousand rows,
    ragged tails, the shared expert, capacity drops; the Switch-shaped layers' d = 768 runs
    row tiles when column pairs are asked for)."""
    wl, x, p, C, ids_ref, g32, out = _run_oracle_routing(SMALL[name], tiles=tiles)
    assert out["status"] == 0
    y_ref, _ = O.moe_layer(x, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual,
                           routing=(ids_ref, g32.double().numpy()))
    if wl.add_residual:
        moe_ref = y_ref - O.as_f64(x)
        moe_gpu = out["y"].double().cpu().numpy() - O.as_f64(x)
        bound = 2e-2 * np.max(np.abs(moe_ref)) + 2.0 ** -8 * np.max(np.abs(y_ref))
        assert np.max(np.abs(moe_gpu - moe_ref)) <= bound
    assert_close(out["y"], y_ref, wl.dtype, f"{name} {tiles}")


def test_shared_expert_on_pairs_matches_row_tiles_bit_for_bit():
    """With a shared expert of T >= 512 rows the automatic choice runs that segment on row
    tiles over SM pairs in launches of its own (4 FFN launches); forcing row tiles runs every
    segment on one-SM row tiles (2 launches).  Both sum each output element over K in the
    same order, so the outputs are the same bits; and both meet the oracle."""
    wl = SMALL["shared16_narrow"]
    assert N.moe_ffn_launches(config_for(wl)) == 4
    assert N.moe_ffn_launches(config_for(wl, tiles="rows")) == 2
    wl_, x, p, C, ids_ref, g32, auto = _run_oracle_routing(wl)
    _, _, _, _, _, _, rows = _run_oracle_routing(wl, tiles="rows")
    assert auto["status"] == 0 and rows["status"] == 0
    assert torch.equal(auto["y"].view(torch.int16), rows["y"].view(torch.int16))
    y_ref, _ = O.moe_layer(x, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual,
                           routing=(ids_ref, g32.double().numpy()))
    assert_close(auto["y"], y_ref, wl.dtype, "shared16_narrow auto")


FUSED_CASES = ["tiny_bf16", "granite_layer", "switch_phi050", "mixtral_T300", "mixtral_decode",
               "shared64_narrow_phi1", "shared64_narrow_dropless", "shared64_narrow_phi2_T1"]


@pytest.mark.parametrize("fuse", ["gather", "combine", "gather+combine"])
@pytest.mark.parametrize("name", FUSED_CASES)
def test_fused_steps(name, fuse):
    """moe_forward with the gather fused into the gate/up GEMM and/or the combine fused into
    the down GEMM's epilogue: bit-identical to the unfused column-tile forward (the same
    rows are summed in the same order), and within the bar against the oracle."""
    wl = SMALL[name] if name in SMALL else W["tiny_fp32"].with_(dtype="bf16", d=128, d_ff=128,
                                                                 add_residual=True)
    x, (p,) = I.make_inputs(wl, seed=3, device="cuda", layers=1)
    ref = forward_gpu(config_for(wl, tiles="columns"), x, p)
    out = forward_gpu(config_for(wl, fuse=fuse), x, p)
    assert ref["status"] == 0 and out["status"] == 0
    for key in ("ids", "gates", "demand", "offsets"):
        assert torch.equal(out[key], ref[key]), key
    assert torch.equal(out["y"].view(torch.int16), ref["y"].view(torch.int16))
    C = oracle_capacity(wl)
    y_ref, info = O.moe_layer(x, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual)
    bad, n_near, ok = ids_agree(out["ids"], info["ids"], O.topk_margin(info["logits"], wl.k),
                                info["logits"], wl.k)
    assert len(bad) == 0
    keep = _robust_tokens(info, ok, n_near, C)
    assert_close(out["y"][torch.from_numpy(keep).cuda()], y_ref[keep], wl.dtype, f"{name} {fuse}")


def test_fused_combine_with_every_route_dropped():
    """Capacity 0: no token has a contribution, so the pack writes y = x (residual) itself."""
    wl = W["switch_phi100"].with_(T=100, add_residual=True)
    x, (p,) = I.make_inputs(wl, seed=0, device="cuda", layers=1)
    for fuse in ("combine", "gather+combine"):
        out = forward_gpu(config_for(wl, capacity=0, fuse=fuse), x, p)
        assert out["status"] == 0
        assert torch.equal(out["y"], x)
    wl0 = wl.with_(add_residual=False)
    out = forward_gpu(config_for(wl0, capacity=0, fuse="combine"), x, p)
    assert out["status"] == 0 and not out["y"].any()


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_parity(name):
    wl = SMALL[name]
    x, (p,) = I.make_inputs(wl, seed=1, device="cuda", layers=1)
    out = forward_gpu(config_for(wl), x, p)
    assert out["status"] == 0
    C = oracle_capacity(wl)
    y_ref, info = O.moe_layer(x, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual)
    margin = O.topk_margin(info["logits"], wl.k)
    bad, n_near, ok = ids_agree(out["ids"], info["ids"], margin, info["logits"], wl.k)
    assert len(bad) == 0
    if n_near == 0:
        assert out["demand"].cpu().numpy().tolist() == info["demand"].tolist()
    keep = _robust_tokens(info, ok, n_near, C)
    assert keep.sum() >= 0.9 * wl.T
    assert_close(out["y"][torch.from_numpy(keep).cuda()], y_ref[keep], wl.dtype, name)


def test_granite_stack_24_layers():
    """24 layers chained by the residual, bf16 activations between layers.

    Tokens are independent rows, so a routing change only affects that token.  The GPU's
    and the oracle's layer inputs drift apart by bf16 rounding of each layer's output, so
    a token may change its top-k at a layer only where the drift allows it: for the set,
    its k-th/(k+1)-th oracle margin, and for the order, its smallest adjacent gap among
    the k+1 largest logits, must be below 2 ||dx_t|| max_e ||w_e|| + 1e-4 (Cauchy-Schwarz
    on the measured input difference dx_t).  Tokens whose expert SET changed at some layer
    are left out of the final comparison (an order change alone leaves the math
    unchanged); every other token must match, and there must be enough of them."""
    wl = W["granite24"]
    x0, layers = I.make_inputs(wl, seed=0, device="cuda")
    cfg = config_for(wl)
    ws = N.workspace(cfg)
    xs = [x0]
    ids_gpu = []
    routes = 0
    for p in layers:
        out = forward_gpu(cfg, xs[-1], p, ws)
        assert out["status"] == 0
        xs.append(out["y"])
        ids_gpu.append(out["ids"].cpu().numpy().astype(np.int64))
        routes += int(out["demand"].sum())
    assert routes == 1412 * 24 * 8 == 271104
    xL_ref, infos = O.moe_stack(x0, layers, wl.k, wl.gate_mode)
    flagged = np.zeros(wl.T, dtype=bool)
    n_set = n_order = 0
    for l, info in enumerate(infos):
        g, r = ids_gpu[l], info["ids"]
        same_order = (g == r).all(axis=1)
        same_set = np.array([set(a) == set(b) for a, b in zip(g, r)])
        dx = np.linalg.norm(xs[l].double().cpu().numpy() - info["x_in"], axis=1)
        wmax = float(np.max(np.linalg.norm(O.as_f64(layers[l]["w_router"]), axis=1)))
        drift = 2 * dx * wmax + 1e-4
        set_flip = ~same_set & ~flagged
        order_flip = same_set & ~same_order & ~flagged
        bad_set = np.where(set_flip & ~(O.topk_margin(info["logits"], wl.k) < drift))[0]
        bad_order = np.where(order_flip & ~(order_margin(info["logits"], wl.k) < drift))[0]
        assert len(bad_set) == 0, f"layer {l}: tokens {bad_set[:10]} changed experts beyond drift"
        assert len(bad_order) == 0, f"layer {l}: tokens {bad_order[:10]} reordered beyond drift"
        n_set += int(set_flip.sum())
        n_order += int(order_flip.sum())
        flagged |= ~same_set
        assert int(info["demand"].sum()) == wl.T * wl.k
    keep = ~flagged
    assert keep.sum() >= 100, f"only {keep.sum()} tokens kept the oracle's experts in all layers"
    err, bound = assert_close(xs[-1][torch.from_numpy(keep).cuda()], xL_ref[keep], "bf16",
                              "granite stack")
    print(f"stack: {keep.sum()} tokens compared, {n_set} expert-set and {n_order} order changes "
          f"explained by drift; max|err| {err:.3e} <= {bound:.3e}")


def _robust_tokens(info, ok, n_near, C):
    """Tokens whose own routing agrees and whose kept/dropped status cannot be changed by
    the n_near near-tie tokens (each can move a later position by at most one)."""
    if C is None:
        return ok
    pos = info["pos"]
    safe = ((pos + n_near < C) | (pos - n_near >= C)).all(axis=1)
    return ok & safe


# ------------------------------------------------------------------------- full size

@pytest.mark.parametrize("name,sample,tiles", [
    ("mixtral_prefill", None, ("auto", "rows", "columns", "pairs")),
    ("mixtral_decode", None, ("auto", "pairs", "row_pairs")),
    ("shared64_T16_dropless", None, ("auto", "fused")),
    ("shared64_T4096_dropless", 512, ("auto", "columns", "pairs", "fused")),
    ("shared64_T4096_phi1", 64, ("auto",)), ("switch_phi050", None, ("auto", "rows"))])
def test_full_size(name, sample, tiles):
    """Full-size layer in the bench's launch configuration.  The oracle routes every token
    and computes the output of every token (sample None) or of a seeded sample of tokens
    (the 64+1 layer at T=4096, whose 52 GB of weights the oracle converts to fp64 expert
    by expert).  Every compared token's routing agrees (near ties excluded) and, with a
    capacity, its kept/dropped status cannot be changed by a near-tie token elsewhere."""
    wl = W[name]
    x, (p,) = I.make_inputs(wl, seed=0, device="cuda", layers=1)
    outs = {t: forward_gpu(config_for(wl, tiles="auto", fuse="gather+combine") if t == "fused"
                           else config_for(wl, tiles=t), x, p) for t in tiles}
    out = outs["auto"]
    for o in outs.values():
        assert o["status"] == 0
        assert torch.equal(o["ids"], out["ids"])
    C = oracle_capacity(wl)
    ids_ref, g_ref, z = O.route(x, p["w_router"], p["logit_bias"], wl.k, wl.gate_mode)
    margin = O.topk_margin(z, wl.k)
    bad, n_near, ok = ids_agree(out["ids"], ids_ref, margin, z, wl.k)
    assert len(bad) == 0
    g = out["gates"].cpu().numpy().astype(np.float64)
    assert np.max(np.abs(g[ok] - g_ref[ok])) <= GATE_ATOL
    disp = O.dispatch(ids_ref, wl.E, C)
    if n_near == 0:
        assert out["demand"].cpu().numpy().tolist() == disp["demand"].tolist()
        assert out["offsets"].cpu().numpy()[:wl.E + 1].tolist() == disp["offsets"].tolist()
    cand = np.where(_robust_tokens(disp, ok, n_near, C))[0]
    if sample is None:
        assert len(cand) >= 0.99 * wl.T
        toks = cand
    else:
        rng = np.random.default_rng(0)
        toks = np.sort(rng.choice(cand, size=min(sample, len(cand)), replace=False))
    y_ref, _ = O.moe_layer(x, p, wl.k, wl.gate_mode, C, add_residual=wl.add_residual,
                           tokens=toks, routing=(ids_ref, g_ref))
    for t, o in outs.items():
        err, bound = assert_close(o["y"][torch.from_numpy(toks).cuda()], y_ref, wl.dtype,
                                  f"{name} tiles={t}")
        print(f"{name} tiles={t}: {len(toks)} of {wl.T} tokens, max|err| {err:.3e} <= {bound:.3e}")


# ------------------------------------------------------------------------- edge cases

def test_capacity_zero_drops_everything():
    wl = W["switch_phi100"].with_(T=100, has_shared=False, add_residual=True)
    x, (p,) = I.make_inputs(wl, seed=0, device="cuda", layers=1)
    cfg = config_for(wl, capacity=0)
    out = forward_gpu(cfg, x, p)
    assert out["status"] == 0
    assert int(out["offsets"][wl.E]) == 0
    assert torch.equal(out["y"], x)    # residual only


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (3, 4, 4), (130, 8, 8), (129, 2, 1)])
def test_degenerate_shapes(T, E, k):
    wl = I.Workload(name="edge", T=T, d=256, E=E, k=k, d_ff=256, gate_mode="softmax_topk_renorm",
                    has_shared=(T == 130), add_residual=(T == 3))
    x, (p,) = I.make_inputs(wl, seed=5, device="cuda", layers=1)
    out = forward_gpu(config_for(wl), x, p)
    assert out["status"] == 0
    y_ref, info = O.moe_layer(x, p, k, wl.gate_mode, None, add_residual=wl.add_residual)
    bad, n_near, ok = ids_agree(out["ids"], info["ids"], O.topk_margin(info["logits"], k),
                                info["logits"], k)
    assert len(bad) == 0
    assert_close(out["y"][torch.from_numpy(ok).cuda()], y_ref[ok], "bf16", f"T={T} E={E} k={k}")


def test_deterministic():
    wl = W["granite24"].with_(layers=1)
    x, (p,) = I.make_inputs(wl, seed=2, device="cuda", layers=1)
    cfg = config_for(wl)
    a = forward_gpu(cfg, x, p)
    b = forward_gpu(cfg, x, p)
    for key in ("y", "ids", "gates", "demand", "offsets"):
        assert torch.equal(a[key], b[key]), key


def test_bounded_wait_reports_timeout_and_context_survives():
    cfg = config_for(W["tiny_fp32"])
    ws = N.workspace(cfg)
    N.moe_debug_bounded_wait(ws, 2_000_000)         # 2 ms, nothing ever arrives
    assert N.moe_get_device_status(ws, clear=True) == 6   # MOE_ERR_TIMEOUT
    x, (p,) = I.make_inputs(W["tiny_fp32"], seed=0, device="cuda", layers=1)
    out = forward_gpu(cfg, x, p, ws)
    assert out["status"] == 0


def test_forward_profiled_matches_forward_and_times_kernels():
    """moe_forward_profiled gives the same bits as moe_forward, called directly and when
    captured into a CUDA graph, and its events time every kernel."""
    wl = W["granite24"].with_(layers=1)
    x, (p,) = I.make_inputs(wl, seed=4, device="cuda", layers=1)
    cfg = config_for(wl)
    ref = forward_gpu(cfg, x, p)
    ws = N.workspace(cfg)
    args = lambda y: (cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"], p["w_down"],
                      p["shared_gate"], p["shared_up"], p["shared_down"], y, None, None, None, None)
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
    y1 = torch.empty_like(x)
    N.moe_forward_profiled(*args(y1), evs, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, ref["y"])
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    assert all(t > 0 for t in times), times
    y2 = torch.empty_like(x)
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cs):
        N.moe_forward_profiled(*args(y2), evs, ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y2, ref["y"])
    assert all(evs[i].elapsed_time(evs[i + 1]) > 0 for i in range(5))
    assert N.moe_get_device_status(ws) == 0


def test_forward_profiled_seven_events_times_the_reroute():
    """With seven events the reroute policy's kernels get their own interval; the bits are
    those of moe_forward."""
    wl = W["switch_phi125_reroute"].with_(T=512)
    x, (p,) = I.make_inputs(wl, seed=6, device="cuda", layers=1)
    cfg = config_for(wl)
    ref = forward_gpu(cfg, x, p)
    ws = N.workspace(cfg)
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(7)]
    y = torch.empty_like(x)
    N.moe_forward_profiled(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"],
                           p["w_down"], p["shared_gate"], p["shared_up"], p["shared_down"], y,
                           None, None, None, None, evs, ws)
    torch.cuda.synchronize()
    assert torch.equal(y, ref["y"])
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(6)]
    assert all(t > 0 for t in times), times
    assert N.moe_get_device_status(ws) == 0
