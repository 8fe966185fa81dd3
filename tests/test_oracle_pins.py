"""Pins for the fp64 oracle against what the pages and the mathematics fix.

Each test ties one oracle function to a value printed on the pages (fixtures under
tests/golden/, each carrying its citation), a closed form, a brute-force count, a
library routine, or an independent formulation, so that a dropped term, a wrong sign
or index, or a transposed operand in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O


# ---------------------------------------------------------------- softmax / gates

def test_softmax_worked_example(golden):
    g = golden("softmax_worked_example.json")
    p = O.softmax(g["logits"])
    assert np.round(p, 3).tolist() == g["softmax_3dp"]
    # exps and their sum, as printed (3 decimals): p * sum(exp) = exp
    assert abs(math.fsum(np.exp(g["logits"])) - g["exp_sum"]) < 5e-4
    assert np.allclose(p * g["exp_sum"], g["exp"], atol=2e-3)
    ids = O.top_k(np.array([g["logits"]]), 2)
    assert ids[0].tolist() == g["top2"]
    sel = O.gates(np.array([g["logits"]]), ids, O.GATE_SOFTMAX_TOPK)[0]
    assert round(float(sel.sum()), 3) == g["selected_mass_3dp"]
    assert np.round(sel, 3).tolist() == g["softmax_3dp"][:2]
    for mode in (O.GATE_SOFTMAX_TOPK_RENORM, O.GATE_TOPK_SOFTMAX):
        w = O.gates(np.array([g["logits"]]), ids, mode)[0]
        assert np.round(w, 3).tolist() == g["renormalised_3dp"]
    # exact values behind the 3-decimal print: e^0.3 / (1 + e^0.3)
    assert abs(O.gates(np.array([g["logits"]]), ids, O.GATE_TOPK_SOFTMAX)[0][0]
               - math.exp(0.3) / (1 + math.exp(0.3))) < 1e-15


def test_flipped_logit_changes_top2(golden):
    g = golden("softmax_worked_example.json")
    p = O.softmax(g["flipped_logits"])
    assert np.round(p, 3).tolist() == g["flipped_softmax_3dp"]
    assert O.top_k(np.array([g["flipped_logits"]]), 2)[0].tolist() == g["flipped_top2"]


def test_gate_sums_and_modes():
    rng = np.random.default_rng(0)
    z = rng.normal(size=(200, 32))
    ids = O.top_k(z, 8)
    g0 = O.gates(z, ids, O.GATE_SOFTMAX_TOPK)
    g1 = O.gates(z, ids, O.GATE_SOFTMAX_TOPK_RENORM)
    g2 = O.gates(z, ids, O.GATE_TOPK_SOFTMAX)
    assert np.max(np.abs(g1.sum(1) - 1)) < 1e-12
    assert np.max(np.abs(g2.sum(1) - 1)) < 1e-12
    assert np.all(g0.sum(1) < 1)             # the unselected experts keep some mass
    assert np.max(np.abs(g1 - g2)) < 1e-14   # equal in exact arithmetic
    # gates are non-increasing along the slots (largest logit first)
    assert np.all(np.diff(g1, axis=1) <= 0)
    # softmax_topk: each gate is exactly the full softmax probability of its expert
    p = np.exp(z - z.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    assert np.allclose(g0, np.take_along_axis(p, ids, 1), rtol=1e-14, atol=0)


def test_softmax_shift_invariance_and_extremes():
    v = np.array([1000.0, 999.0, -1000.0])
    p = O.softmax(v)
    assert np.isfinite(p).all() and abs(p.sum() - 1) < 1e-15
    assert abs(p[0] / p[1] - math.e) < 1e-12
    assert np.allclose(O.softmax(v - 17.0), p, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- top-k

def test_top_k_ties_go_to_lower_index():
    z = np.array([[1.0, 3.0, 3.0, 2.0], [0.0, 0.0, 0.0, 0.0], [5.0, 1.0, 5.0, 5.0]])
    assert O.top_k(z, 2).tolist() == [[1, 2], [0, 1], [0, 2]]
    assert O.top_k(z, 4)[2].tolist() == [0, 2, 3, 1]


def test_top_k_matches_stable_argsort():
    rng = np.random.default_rng(1)
    z = np.round(rng.normal(size=(300, 16)), 1)   # many exact ties
    for k in (1, 2, 5, 16):
        ref = np.argsort(-z, axis=1, kind="stable")[:, :k]
        assert np.array_equal(O.top_k(z, k), ref)


def test_router_logits_layout_and_bias():
    # nn.Linear storage: W [E, d]; z[t, e] = x[t] . W[e] + b[e]
    x = np.array([[1.0, 2.0, 3.0]])
    W = np.array([[1.0, 0.0, 0.0], [0.0, 0.0, 1.0]])
    z = O.router_logits(x, W, np.array([0.5, -1.0]))
    assert z.tolist() == [[1.5, 2.0]]
    with pytest.raises(ValueError):
        O.router_logits(x, W.T)   # [d, E] is the math form, not the stored form


def test_topk_margin():
    z = np.array([[3.0, 1.0, 2.0, 0.5]])
    assert O.topk_margin(z, 1)[0] == 1.0
    assert O.topk_margin(z, 2)[0] == 1.0
    assert O.topk_margin(z, 3)[0] == 0.5
    assert O.topk_margin(z, 4)[0] == np.inf


# ---------------------------------------------------------------- capacity / dispatch

def test_capacity_formula(golden):
    g = golden("capacity_worked_case.json")
    assert O.capacity(8, 2, 4, *g["phi"]) == g["C"] == 5
    for v in g["variants"]:
        assert O.capacity(8, v["k"], 4, *v["phi"]) == v["C"]
    # Switch-shaped top-1 layer, T = 4096, E = 4
    assert [O.capacity(4096, 1, 4, n, dn) for n, dn in ((1, 2), (1, 1), (5, 4))] == [512, 1024, 1280]
    # 64 routed experts, top-2
    assert [O.capacity(T, 2, 64, 1, 1) for T in (1, 16, 256, 4096)] == [1, 1, 8, 128]
    assert [O.capacity(T, 2, 64, 2, 1) for T in (1, 16, 256, 4096)] == [1, 1, 16, 256]
    # exact ceil, no float rounding: phi*T*k/E = 2.5 -> 3 and 3.0 -> 3
    assert O.capacity(8, 1, 4, 5, 4) == 3 and O.capacity(12, 1, 4, 1, 1) == 3


def test_capacity_worked_case_trace(golden):
    g = golden("capacity_worked_case.json")
    ids = np.array(g["assignments"])
    d = O.dispatch(ids, g["E"], g["C"])
    assert d["demand"].tolist() == g["demand"]
    assert int(d["demand"].sum()) == g["T"] * g["k"]
    dropped = [[t, int(ids[t, j])] for t in range(g["T"]) for j in range(g["k"])
               if d["route_row"][t, j] < 0]
    assert dropped == g["dropped_routes"]
    for e, toks in enumerate(g["slot_table"]):
        lo, hi = d["offsets"][e], d["offsets"][e + 1]
        assert d["row_token"][lo:hi].tolist() == toks
    assert int(d["kept"].sum()) == g["filled"]
    assert g["E"] * g["C"] == g["slots"]
    assert [round(100 * kc / g["C"]) for kc in d["kept"]] == g["utilisation_pct"]


def test_capacity_variants(golden):
    g = golden("capacity_worked_case.json")
    full = np.array(g["assignments"])
    for v in g["variants"]:
        ids = full[:, :v["k"]]            # k = 1 keeps the first expert of each pair
        C = O.capacity(g["T"], v["k"], g["E"], *v["phi"])
        d = O.dispatch(ids, g["E"], C)
        assert int((d["route_row"] < 0).sum()) == v["dropped"]
        assert O.drop_count(d["demand"], C) == v["dropped"]
        if "demand" in v:
            assert d["demand"].tolist() == v["demand"]
        if "filled" in v:
            assert int(d["kept"].sum()) == v["filled"] and g["E"] * C == v["slots"]
    # f = 1.0: arrival order drops the 5th and 6th arrivals at E1 (t5, t6)
    d = O.dispatch(full, 4, 4)
    assert [t for t in range(8) if d["route_row"][t, 0] < 0] == [4, 5]


def test_lesson_capacity_overflow(golden):
    g = golden("lesson_capacity_overflow.json")
    C = O.capacity(g["T"], g["k"], g["E"], *g["phi"])
    assert C == g["C"]
    ids = np.array([[e] for e, n in enumerate(g["demand"]) for _ in range(n)])
    d = O.dispatch(ids, g["E"], C)
    assert d["demand"].tolist() == g["demand"]
    assert int((d["route_row"] < 0).sum()) == g["dropped"]


def test_permutation_example(golden):
    g = golden("permutation_example.json")
    ids = np.array(g["expert_ids"])
    d = O.dispatch(ids, g["E"], None)
    assert d["row_token"].tolist() == g["packed_token_order"]
    assert d["offsets"][1:].tolist() == g["expert_ends"]
    for e, toks in g["groups"].items():
        e = int(e)
        assert d["row_token"][d["offsets"][e]:d["offsets"][e + 1]].tolist() == toks
    # the packed order is the stable argsort of the flattened ids (a library routine)
    flat = ids.flatten()
    order = np.argsort(flat, kind="stable")
    assert np.array_equal(np.repeat(np.arange(3), 2)[order], d["row_token"])
    # restore: scattering the packed rows back by route_row gives the duplicated rows
    x = np.array(g["x"])
    packed = x[d["row_token"]]
    restored = packed[d["route_row"].flatten()]
    assert np.array_equal(restored, np.repeat(x, 2, axis=0))


def test_dispatch_brute_force():
    rng = np.random.default_rng(2)
    T, E, k = 97, 6, 3
    # skewed distinct choices per token
    pr = np.array([0.4, 0.25, 0.15, 0.1, 0.06, 0.04])
    ids = np.array([rng.choice(E, size=k, replace=False, p=pr) for _ in range(T)])
    for C in (None, 0, 1, 7, 30, 1000):
        d = O.dispatch(ids, E, C)
        for e in range(E):
            toks = [t for t in range(T) if e in ids[t]]          # O(T*E) recount
            assert d["demand"][e] == len(toks)
            keep = toks if C is None else toks[:C]               # lowest token index first
            seg = d["row_token"][d["offsets"][e]:d["offsets"][e + 1]].tolist()
            assert seg == keep
        R = int(d["offsets"][-1])
        assert R == int((d["route_row"] >= 0).sum()) == len(d["row_token"])
        # route_row is a bijection from kept routes onto 0..R-1
        rows = np.sort(d["route_row"][d["route_row"] >= 0])
        assert np.array_equal(rows, np.arange(R))
        for t in range(T):
            for j in range(k):
                r = d["route_row"][t, j]
                if r >= 0:
                    assert d["row_token"][r] == t
                    e = ids[t, j]
                    assert d["offsets"][e] <= r < d["offsets"][e + 1]


def test_top1_drops_exactly_the_overflow():
    rng = np.random.default_rng(3)
    T, E = 400, 4
    z = rng.normal(size=(T, E)) + np.array([1.0, 0.0, 0.0, -1.0])
    ids = O.top_k(z, 1)
    for phi in ((1, 2), (1, 1), (5, 4)):
        C = O.capacity(T, 1, E, *phi)
        d = O.dispatch(ids, E, C)
        over = sum(max(0, int(D) - C) for D in d["demand"])
        assert int((d["route_row"] < 0).sum()) == over
        # the dropped routes of each expert are its highest-index tokens
        for e in range(E):
            toks = [t for t in range(T) if ids[t, 0] == e]
            dropped = [t for t in toks if d["route_row"][t, 0] < 0]
            assert dropped == toks[C:]


def test_route_count(golden):
    g = golden("route_count.json")
    rng = np.random.default_rng(4)
    total = 0
    for _ in range(g["layers"]):
        ids = O.top_k(rng.normal(size=(g["T"], g["E"])), g["k"])
        total += int(O.dispatch(ids, g["E"], None)["demand"].sum())
    assert total == g["routes"] == g["T"] * g["layers"] * g["k"]
    # one expert in every token's top-8 of 32: four times the mean load, the ceiling
    z = rng.normal(size=(g["T"], g["E"]))
    z[:, 5] += 100.0
    d = O.dispatch(O.top_k(z, g["k"]), g["E"], None)
    assert O.imbalance(d["demand"]) == g["max_imbalance"] == g["E"] / g["k"]


def test_imbalance_bound(golden):
    g = golden("imbalance_bound.json")
    E, k = g["E"], g["k"]
    rng = np.random.default_rng(5)
    for _ in range(20):
        ids = O.top_k(rng.normal(size=(64, E)) * rng.uniform(0.1, 5), k)
        I = O.imbalance(O.dispatch(ids, E, None)["demand"])
        assert 1.0 <= I <= E / k + 1e-12
    ids = np.tile([3, 6], (64, 1))       # collapsed router: every token picks the same two
    assert O.imbalance(O.dispatch(ids, E, None)["demand"]) == g["worst_case"]
    assert O.imbalance([5, 5, 5, 5]) == 1.0


# ---------------------------------------------------------------- SwiGLU expert

def test_swiglu_closed_form():
    # sigmoid(ln 3) = 3/4, so SiLU(ln 3) = 0.75 ln 3.  d = 2, F = 3 (non-square, so a
    # transposed weight cannot pass silently).
    l3 = math.log(3.0)
    wg = np.array([[l3, 0.0], [0.0, 0.0], [0.0, l3]])     # [F, d]
    wu = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, 0.0]])   # [F, d]
    wd = np.array([[1.0, 10.0, 100.0], [0.0, 1.0, 0.0]])  # [d, F]
    y = O.swiglu_expert(np.array([[1.0, 1.0]]), wg, wu, wd)
    assert np.allclose(y, [[150.75 * l3, 0.0]], rtol=1e-15, atol=1e-15)
    # SiLU itself: 0 at 0, odd part a/2, large |a| limits
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(l3) - 0.75 * l3) < 1e-15
    assert O.silu(800.0) == 800.0 and O.silu(-800.0) == 0.0
    a = np.linspace(-5, 5, 11)
    assert np.allclose(O.silu(a) - O.silu(-a), a, atol=1e-14)
    with pytest.raises(ValueError):
        O.swiglu_expert(np.array([[1.0, 1.0]]), wg, wu, wd.T)


def _tiny_params(rng, E, d, F, shared=False):
    s = 1.0 / math.sqrt(d)
    p = dict(w_router=rng.normal(size=(E, d)) * s, logit_bias=None,
             w_gate=rng.normal(size=(E, F, d)) * s, w_up=rng.normal(size=(E, F, d)) * s,
             w_down=rng.normal(size=(E, d, F)) * s)
    if shared:
        p.update(shared_gate=rng.normal(size=(F, d)) * s, shared_up=rng.normal(size=(F, d)) * s,
                 shared_down=rng.normal(size=(d, F)) * s)
    return p


@pytest.mark.parametrize("mode", O.GATE_MODES)
def test_dense_equivalence(mode):
    """Dropless layer == dense loop over ALL experts with gates zero off the top-k."""
    rng = np.random.default_rng(6)
    T, d, E, k, F = 9, 8, 5, 2, 12
    p = _tiny_params(rng, E, d, F, shared=True)
    x = rng.normal(size=(T, d))
    y, info = O.moe_layer(x, p, k, mode, None, add_residual=True)
    G = np.zeros((T, E))
    for t in range(T):
        G[t, info["ids"][t]] = info["gates"][t]
    dense = x.copy()
    for e in range(E):
        dense += G[:, e:e + 1] * O.swiglu_expert(x, p["w_gate"][e], p["w_up"][e], p["w_down"][e])
    dense += O.swiglu_expert(x, p["shared_gate"], p["shared_up"], p["shared_down"])
    assert np.allclose(y, dense, rtol=1e-12, atol=1e-12)
    assert y.shape == x.shape


def test_single_expert_is_a_plain_swiglu_mlp():
    rng = np.random.default_rng(7)
    p = _tiny_params(rng, 1, 6, 10)
    x = rng.normal(size=(5, 6))
    for mode in (O.GATE_SOFTMAX_TOPK_RENORM, O.GATE_TOPK_SOFTMAX, O.GATE_SOFTMAX_TOPK):
        y, _ = O.moe_layer(x, p, 1, mode)
        assert np.allclose(y, O.swiglu_expert(x, p["w_gate"][0], p["w_up"][0], p["w_down"][0]),
                           rtol=1e-14, atol=1e-14)


def test_dropped_route_contributes_zero():
    """Worked case: t6 loses E1 at C = 5 and keeps only 0.426 of the mixture."""
    rng = np.random.default_rng(8)
    T, d, E, k, F = 8, 4, 4, 2, 6
    p = _tiny_params(rng, E, d, F)
    x = rng.normal(size=(T, d))
    ids = np.array([[0, 1], [0, 2], [0, 1], [0, 3], [0, 2], [0, 1], [1, 3], [2, 3]])
    g = O.gates(np.tile([2.1, 1.8, 0.2, -5.0], (T, 1)), np.tile([0, 1], (T, 1)),
                O.GATE_SOFTMAX_TOPK_RENORM)
    y, info = O.moe_layer(x, p, k, O.GATE_SOFTMAX_TOPK_RENORM, C=5, routing=(ids, g))
    e2 = O.swiglu_expert(x[5:6], p["w_gate"][1], p["w_up"][1], p["w_down"][1])[0]
    assert round(g[5, 1], 3) == 0.426
    assert np.allclose(y[5], g[5, 1] * e2, rtol=1e-14, atol=1e-14)
    # the same routing without capacity restores the E1 share
    y_free, _ = O.moe_layer(x, p, k, O.GATE_SOFTMAX_TOPK_RENORM, C=None, routing=(ids, g))
    e1 = O.swiglu_expert(x[5:6], p["w_gate"][0], p["w_up"][0], p["w_down"][0])[0]
    assert np.allclose(y_free[5] - y[5], g[5, 0] * e1, rtol=1e-12, atol=1e-12)
    # top-1 with every route dropped leaves the residual alone
    y0, _ = O.moe_layer(x, p, 1, O.GATE_SOFTMAX_TOPK, C=0, add_residual=True)
    assert np.array_equal(y0, x)


def test_layer_token_subset_matches_full():
    rng = np.random.default_rng(9)
    p = _tiny_params(rng, 4, 8, 16, shared=True)
    x = rng.normal(size=(20, 8))
    y, _ = O.moe_layer(x, p, 2, O.GATE_TOPK_SOFTMAX, C=6, add_residual=True)
    sub = [0, 7, 19, 3]
    ys, _ = O.moe_layer(x, p, 2, O.GATE_TOPK_SOFTMAX, C=6, add_residual=True, tokens=sub)
    assert np.allclose(ys, y[sub], rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- bf16 rounding, stack

def test_round_to_bf16_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(10)
    v = np.concatenate([rng.normal(size=4000) * 10.0 ** rng.integers(-8, 8, 4000),
                        [0.0, -0.0, 1.0, 65504.0]])
    v32 = v.astype(np.float32).astype(np.float64)   # fp32-representable: one rounding only
    ref = torch.from_numpy(v32).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(v32), ref)
    # ties go to even; just above a tie rounds up
    assert O.round_to_bf16(1.0 + 2.0 ** -8) == 1.0
    assert O.round_to_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.round_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7


def test_stack_route_count_and_residual():
    rng = np.random.default_rng(11)
    layers = [_tiny_params(rng, 8, 16, 8) for _ in range(3)]
    x0 = rng.normal(size=(12, 16))
    xL, infos = O.moe_stack(x0, layers, 2, O.GATE_TOPK_SOFTMAX)
    assert sum(int(i["demand"].sum()) for i in infos) == 12 * 3 * 2
    # one layer by hand
    y1, _ = O.moe_layer(x0, layers[0], 2, O.GATE_TOPK_SOFTMAX, add_residual=True)
    x1 = O.round_to_bf16(y1)
    y2, _ = O.moe_layer(x1, layers[1], 2, O.GATE_TOPK_SOFTMAX, add_residual=True)
    x2 = O.round_to_bf16(y2)
    y3, _ = O.moe_layer(x2, layers[2], 2, O.GATE_TOPK_SOFTMAX, add_residual=True)
    assert np.array_equal(xL, O.round_to_bf16(y3))


# ---------------------------------------------------------------- routing statistics

def test_routing_stats_worked_case(golden):
    """[S19] worked case: demand 6/4/3/3, C = 5, one drop, 15 of 20 slots used (25% padding)."""
    g = golden("capacity_worked_case.json")
    ids = np.array(g["assignments"])
    T, E, k = g["T"], g["E"], g["k"]
    rng = np.random.default_rng(12)
    x, w = rng.normal(size=(T, 8)), rng.normal(size=(E, 8))
    st = O.routing_stats(x, w, None, k, g["C"], ids=ids)
    assert st["kept"] == g["filled"] == 15
    assert st["padding_rate"] == (g["slots"] - g["filled"]) / g["slots"] == 0.25
    assert st["drop_rate"] == 1 / 16
    assert st["imbalance"] == 6 / 4
    assert np.allclose(st["f"], np.array(g["demand"]) / 16, rtol=0, atol=0)
    assert abs(st["P"].sum() - 1) < 1e-12


def test_aux_loss_closed_forms():
    """Uniform routing gives aux = alpha; a collapsed router gives aux -> alpha * E."""
    T, E, d = 64, 8, 4
    x = np.zeros((T, d))
    w = np.zeros((E, d))
    ids = np.array([[t % E] for t in range(T)])          # every expert gets T/E routes
    st = O.routing_stats(x, w, None, 1, None, alpha=0.01, ids=ids)
    assert np.allclose(st["f"], 1 / E) and np.allclose(st["P"], 1 / E)
    assert abs(st["aux"] - 0.01) < 1e-15
    bias = np.zeros(E)
    bias[0] = 60.0                                        # softmax ~ one-hot on expert 0
    st = O.routing_stats(np.ones((T, d)), np.zeros((E, d)), bias, 1, None, alpha=0.01)
    assert st["f"][0] == 1.0 and st["P"][0] > 1 - 1e-12
    assert abs(st["aux"] - 0.01 * E) < 1e-12
    assert st["imbalance"] == E / 1


def test_routing_stats_drop_and_padding_brute_force():
    """Drop and padding rates against a slot-by-slot count, including C = 0 (no slots)."""
    rng = np.random.default_rng(3)
    T, E, k, d = 50, 6, 2, 5
    x, w = rng.normal(size=(T, d)), rng.normal(size=(E, d))
    ids = O.top_k(O.router_logits(x, w), k)
    for C in (None, 0, 3, 17, 100):
        st = O.routing_stats(x, w, None, k, C, ids=ids)
        used = [0] * E
        kept = 0
        for t in range(T):                 # arrival order = token order
            for j in range(k):
                e = int(ids[t, j])
                if C is None or used[e] < C:
                    used[e] += 1
                    kept += 1
        assert st["kept"] == kept
        assert st["drop_rate"] == (T * k - kept) / (T * k)
        assert st["padding_rate"] == (0.0 if not C else sum(C - u for u in used) / (E * C))
        # P: the mean of the full softmax, one token at a time
        z = O.router_logits(x, w)
        P = sum(np.exp(z[t] - z[t].max()) / np.exp(z[t] - z[t].max()).sum() for t in range(T)) / T
        assert np.allclose(st["P"], P, rtol=1e-13, atol=0)
        assert abs(st["aux"] - 1e-2 * E * sum(st["f"][e] * P[e] for e in range(E))) < 1e-15


# ---------------------------------------------------------------- padded buffer, reroute

def _worked_logits(g, soft):
    """Logits consistent with the worked case's assignments: each token's two experts
    get t1's top-2 logits; t6 (index 5) shares t1's logits, E4 absent from the
    three-expert reduction (logit -inf)."""
    z = np.full((g["T"], g["E"]), -np.inf)
    for t, (a, b) in enumerate(g["assignments"]):
        z[t, a], z[t, b] = soft["logits"][0], soft["logits"][1]
    z[5, :3] = soft["logits"]
    return z


def test_padded_buffer_worked_case(golden):
    """[S19] Visual support - Capacity: the [E, C, d] buffer row by row, 15 of 20 filled."""
    g = golden("capacity_worked_case.json")
    d = O.dispatch_padded(np.array(g["assignments"]), None, g["E"], g["C"])
    for e, toks in enumerate(g["slot_table"]):
        row = d["row_token"][e * g["C"]:(e + 1) * g["C"]].tolist()
        assert row == toks + [-1] * (g["C"] - len(toks))
    assert d["counts"].tolist() == [len(t) for t in g["slot_table"]]
    assert int(d["counts"].sum()) == g["filled"] and (d["row_token"] < 0).sum() == 5
    assert [[t, 0] for t in range(g["T"]) if d["route_row"][t, 0] < 0] == g["dropped_routes"]
    assert not d["rerouted"].any()


def test_reroute_worked_case(golden):
    """[S19] Overflow policies: with reroute, t6's overflowing E1 route is handled by its
    third-best expert (E3, which has free slots); nothing is dropped, 16 of 20 slots."""
    g = golden("capacity_worked_case.json")
    soft = golden("softmax_worked_example.json")
    ids = np.array(g["assignments"])
    z = _worked_logits(g, soft)
    assert np.array_equal(O.top_k(z, 2), ids)       # the logits reproduce the trace
    d = O.dispatch_padded(ids, z, g["E"], g["C"], O.OVERFLOW_REROUTE)
    assert d["rerouted"].sum() == 1 and d["rerouted"][5, 0]
    assert d["final_ids"][5].tolist() == [2, 1]
    assert d["route_row"][5, 0] == 2 * g["C"] + 3   # E3's 4th slot (3 were filled)
    assert d["counts"].tolist() == [5, 4, 4, 3] and (d["route_row"] >= 0).all()
    # gates of t6 over its final experts {E3, E2}, from the printed probabilities
    p = soft["softmax_3dp"]
    g_in = O.gates(z, ids, O.GATE_SOFTMAX_TOPK_RENORM)
    g1 = O.reroute_gates(z, d["final_ids"], g_in, d["rerouted"], O.GATE_SOFTMAX_TOPK_RENORM)
    assert np.allclose(g1[5], [p[2] / (p[2] + p[1]), p[1] / (p[2] + p[1])], atol=2e-3)
    g0 = O.reroute_gates(z, d["final_ids"], g_in, d["rerouted"], O.GATE_SOFTMAX_TOPK)
    assert np.allclose(g0[5], [p[2], p[1]], atol=5e-4)
    g2 = O.reroute_gates(z, d["final_ids"], g_in, d["rerouted"], O.GATE_TOPK_SOFTMAX)
    assert abs(g2[5, 0] - 1 / (1 + math.exp(1.6))) < 1e-15   # softmax of (0.2, 1.8)
    others = np.arange(g["T"]) != 5
    assert np.array_equal(g1[others], g_in[others])          # untouched tokens keep gates


def test_reroute_fills_the_second_expert():
    """k = 1, E = 2, C = T/2, every token prefers expert 0: the second half of the tokens
    is rerouted to expert 1, so slot order equals token order."""
    T = 10
    z = np.tile([1.0, 0.0], (T, 1))
    d = O.dispatch_padded(O.top_k(z, 1), z, 2, T // 2, O.OVERFLOW_REROUTE)
    assert d["route_row"][:, 0].tolist() == list(range(T))
    assert d["row_token"].tolist() == list(range(T))
    assert d["rerouted"][:, 0].tolist() == [False] * 5 + [True] * 5
    drop = O.dispatch_padded(O.top_k(z, 1), z, 2, T // 2)
    assert drop["route_row"][:, 0].tolist() == list(range(5)) + [-1] * 5


def test_reroute_invariants_brute_force():
    rng = np.random.default_rng(7)
    for trial in range(40):
        T, E, k = int(rng.integers(1, 40)), int(rng.integers(2, 8)), 0
        k = int(rng.integers(1, E + 1))
        z = np.round(rng.normal(size=(T, E)), 1)
        ids = O.top_k(z, k)
        C = int(rng.integers(0, max(1, T * k // E) + 2))
        drop = O.dispatch_padded(ids, z, E, C)
        rr = O.dispatch_padded(ids, z, E, C, O.OVERFLOW_REROUTE)
        ragged = O.dispatch(ids, E, C)
        # phase 1 equals the drop policy, which equals the ragged dispatch's kept set
        assert np.array_equal(drop["route_row"] >= 0, ragged["route_row"] >= 0)
        assert np.array_equal(rr["route_row"][drop["route_row"] >= 0],
                              drop["route_row"][drop["route_row"] >= 0])
        assert (rr["counts"] <= C).all() and int(rr["counts"].sum()) == int((rr["route_row"] >= 0).sum())
        for t in range(T):
            assert len(set(rr["final_ids"][t].tolist())) == k      # experts stay distinct
            held = set(rr["final_ids"][t].tolist())
            rank = sorted(range(E), key=lambda e: (-z[t, e], e))
            for j in range(k):
                if rr["route_row"][t, j] < 0:   # dropped: every expert it could take is full
                    assert all(rr["counts"][e] == C for e in range(E) if e not in held)
                if rr["rerouted"][t, j]:        # better-ranked candidates are full
                    tgt = int(rr["final_ids"][t, j])
                    for e in rank[:rank.index(tgt)]:
                        assert e in held or rr["counts"][e] == C
        for r, t in enumerate(rr["row_token"]):
            if t >= 0:
                e, s = divmod(r, C)
                assert s < rr["counts"][e] and t in np.where(rr["route_row"] == r)[0]
        # capacity large enough: no overflow, both policies equal the dropless order
        big = O.dispatch_padded(ids, z, E, T * k, O.OVERFLOW_REROUTE)
        full = O.dispatch(ids, E, None)
        assert not big["rerouted"].any()
        for e in range(E):
            toks = full["row_token"][full["offsets"][e]:full["offsets"][e + 1]].tolist()
            assert big["row_token"][e * T * k:e * T * k + len(toks)].tolist() == toks


def test_padded_layer_equals_ragged_layer():
    """The buffer layout changes no output; with room for every route, rerouting changes
    nothing either (dropless)."""
    rng = np.random.default_rng(11)
    T, d, E, k, F = 24, 8, 4, 2, 6
    p = {"w_router": rng.normal(size=(E, d)), "logit_bias": None,
         "w_gate": rng.normal(size=(E, F, d)), "w_up": rng.normal(size=(E, F, d)),
         "w_down": rng.normal(size=(E, d, F))}
    x = rng.normal(size=(T, d))
    for C in (3, 7, 12):
        y_r, _ = O.moe_layer(x, p, k, O.GATE_SOFTMAX_TOPK_RENORM, C)
        y_p, info = O.moe_layer(x, p, k, O.GATE_SOFTMAX_TOPK_RENORM, C, layout="padded")
        assert np.array_equal(y_r, y_p)
    y_free, _ = O.moe_layer(x, p, k, O.GATE_TOPK_SOFTMAX, None)
    y_rr, info = O.moe_layer(x, p, k, O.GATE_TOPK_SOFTMAX, T * k, layout="padded",
                             overflow=O.OVERFLOW_REROUTE)
    assert np.array_equal(y_free, y_rr) and not info["rerouted"].any()
    # tight capacity: rerouted tokens mix their final experts with recomputed gates
    for C in range(6, 16):
        y_t, info = O.moe_layer(x, p, k, O.GATE_SOFTMAX_TOPK, C, layout="padded",
                                overflow=O.OVERFLOW_REROUTE)
        if info["rerouted"].any():
            break
    t = int(np.where(info["rerouted"].any(axis=1))[0][0])
    sm = O.softmax(O.router_logits(x, p["w_router"])[t])
    want = sum(sm[e] * O.swiglu_expert(x[t:t + 1], p["w_gate"][e], p["w_up"][e], p["w_down"][e])[0]
               for j, e in enumerate(info["final_ids"][t]) if info["route_row"][t, j] >= 0)
    assert np.allclose(y_t[t], want, rtol=1e-12, atol=1e-12)
