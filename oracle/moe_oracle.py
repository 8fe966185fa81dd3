"""Plain fp64 CPU oracle for the MoE layer forward: route -> pack -> compute -> combine.

TEST INFRASTRUCTURE ONLY.  This module is the independent reference that the CUDA
path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import it.  The product path (the CUDA
library ``libmoe.so`` and its Python binding) never calls it and has no CPU fallback.
It shares no code with the CUDA path: no kernels, headers, tables or helpers.

Everything is float64 numpy.  Inputs stored as bf16 or fp32 convert exactly to float64.
A library matmul (numpy ``@``) is used as a single step where the pages apply a linear
layer; there is no blocking, fusion or reordering beyond what the pages state.

Sources (web pages, cited by title and section):
  [MoE-271K]  "271,104 Routes: What I Missed About Mixture-of-Experts"
  [MoE-L]     "Mixture of Experts: Routing, Dispatch, and Load Balancing"
  [MoE-VIS]   "MoE Inference Visualized - How Expert Routing Actually Works Inside a Real Model"
  [MoE-S19]   "Mixture-of-Experts: routing and capacity" (Session 19 slides)
  [MoE-AEV]   "Mixture-of-experts routing" (AI Engineering Visualised)

Readings taken where the pages are silent or disagree:
  * Three gate modes are kept apart because the pages place the softmax in two places
    (all experts, or only the selected k) and renormalise in one of them.
  * Top-k ranks the logits (softmax is monotone); equal logits go to the lower index.
  * Capacity C = ceil(phi*T*k/E) in exact integer arithmetic; one capacity group is
    the whole call; overflow drops routes by arrival order = token index; a dropped
    route contributes zero and the surviving gates are not renormalised.
  * The shared expert has gate 1, is never dropped, and sits outside renormalisation.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
against the pages' worked examples, closed forms, brute force or an independent
dense formulation.  No function here is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

# Gate modes, named after where the softmax sits.
GATE_SOFTMAX_TOPK = "softmax_topk"                 # softmax over all E, keep p of the top-k
GATE_SOFTMAX_TOPK_RENORM = "softmax_topk_renorm"   # ... then divide by their sum
GATE_TOPK_SOFTMAX = "topk_softmax"                 # top-k of the logits, softmax over those k
GATE_MODES = (GATE_SOFTMAX_TOPK, GATE_SOFTMAX_TOPK_RENORM, GATE_TOPK_SOFTMAX)


def as_f64(a) -> np.ndarray:
    """Exact conversion of a stored array (numpy or torch CPU tensor) to float64."""
    if hasattr(a, "detach"):  # a torch tensor: bf16 -> f64 is exact
        import torch  # local import: the oracle itself needs only numpy
        return a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------------
# Route
# ----------------------------------------------------------------------------------

def router_logits(x, w_router, logit_bias=None) -> np.ndarray:
    """z[t, e] = sum_i x[t, i] * W_r[e, i] + bias[e], in float64.

    [MoE-L] section 1, "What the router actually does": the router is a linear
    projection from d to N expert scores; nn.Linear stores its weight as [N, d].
    [MoE-VIS] "The Router": one row of the [4, 768] weight per expert, dotted with
    the token state.  ``logit_bias`` is the additive per-expert term (the ``b_router``
    of [MoE-L] section 1); the workloads use it as a fixed skew.
    """
    x = as_f64(x)
    w = as_f64(w_router)
    z = x @ w.T
    if logit_bias is not None:
        z = z + as_f64(logit_bias)[None, :]
    return z


def softmax(v) -> np.ndarray:
    """Softmax along the last axis: exp(v - max) / sum exp(v - max).

    [MoE-S19] "Router" and "Worked case": logits [2.1, 1.8, 0.2] give about
    [0.529, 0.392, 0.079].  Subtracting the max does not change the value.
    """
    v = np.asarray(v, dtype=np.float64)
    m = np.max(v, axis=-1, keepdims=True)
    ex = np.exp(v - m)
    return ex / np.sum(ex, axis=-1, keepdims=True)


def top_k(z, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, largest first; ties go to the lower index.

    [MoE-271K] section 2 ("logits.topk(k)") and [MoE-L] section 3 (topk of the
    probabilities; softmax is monotone so the ranking is the same).  torch leaves
    the order of equal values open; the reading here is lowest index first.
    """
    z = np.asarray(z, dtype=np.float64)
    T, E = z.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        # sort key: larger logit first, then smaller expert index
        order = sorted(range(E), key=lambda e: (-z[t, e], e))
        ids[t] = order[:k]
    return ids


def gates(z, ids, mode: str) -> np.ndarray:
    """Gate weight of each selected expert, per gate mode.

    softmax_topk        [MoE-VIS] "The Router" / "Expert Execution": softmax over all
                        experts, the chosen expert's probability is its router weight.
    softmax_topk_renorm [MoE-L] section 3 (weighted sum divided by the total selected
                        weight) and [MoE-S19] "Top-k and mixture" (0.529, 0.392 become
                        0.574, 0.426 after dividing by 0.921).
    topk_softmax        [MoE-271K] sections 2 and 4 (softmax of the top-k logits) and
                        [MoE-AEV] "The gate": g_i = exp(r_i) / sum over top-k exp(r_j).
    """
    z = np.asarray(z, dtype=np.float64)
    ids = np.asarray(ids)
    T, k = ids.shape
    g = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        sel = z[t, ids[t]]
        if mode == GATE_SOFTMAX_TOPK:
            g[t] = softmax(z[t])[ids[t]]
        elif mode == GATE_SOFTMAX_TOPK_RENORM:
            # p_i / sum_sel p_j with p = softmax over all E.  The full softmax's normaliser
            # cancels in the ratio, so it is evaluated as exp(z_i - c) / sum_sel exp(z_j - c)
            # with c the largest selected logit: the same value, finite even when every
            # selected p underflows (a rerouted token may no longer hold its top expert).
            e = np.exp(sel - np.max(sel))
            g[t] = e / np.sum(e)
        elif mode == GATE_TOPK_SOFTMAX:
            g[t] = softmax(sel)
        else:
            raise ValueError(f"unknown gate mode {mode!r}")
    return g


def route(x, w_router, logit_bias, k: int, mode: str):
    """Router step: logits, top-k ids and gates.  Returns (ids, gates, logits)."""
    z = router_logits(x, w_router, logit_bias)
    ids = top_k(z, k)
    return ids, gates(z, ids, mode), z


def topk_margin(z, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest logit of each token (inf when k == E).

    Tokens whose gap is tiny can legitimately flip between two correct top-k sets
    under different rounding; parity tests exclude them from the id comparison.
    """
    z = np.asarray(z, dtype=np.float64)
    T, E = z.shape
    if k >= E:
        return np.full(T, np.inf)
    s = -np.sort(-z, axis=1)
    return s[:, k - 1] - s[:, k]


# ----------------------------------------------------------------------------------
# Pack: capacity, arrival-order positions, grouping by expert
# ----------------------------------------------------------------------------------

def capacity(T: int, k: int, E: int, phi_num: int, phi_den: int) -> int:
    """C = ceil(phi * T * k / E) with phi = phi_num / phi_den, in exact integer arithmetic.

    [MoE-AEV] "Capacity" and [MoE-S19] "Capacity": C = ceil(T*k/E * f); the worked
    case gives ceil(8*2/4 * 1.25) = 5.
    """
    if min(T, k, E, phi_num, phi_den) < 0 or E == 0 or phi_den == 0:
        raise ValueError("bad capacity arguments")
    num = phi_num * T * k
    den = phi_den * E
    return -(-num // den)


def dispatch(ids, E: int, C: int | None):
    """Arrival-order positions, capacity mask and the expert-major packed order.

    Walk the routes in arrival order (token t = 0..T-1, then slot j = 0..k-1), count
    the routes each expert has received so far; the route's position in its expert
    batch is that count.  With a capacity C the route is kept iff its position < C
    ([MoE-S19] "Worked case": the 6th arrival at E1 with C = 5 is dropped; instructor
    notes: arrival order decides who is dropped).  C = None means dropless
    ([MoE-AEV] "Capacity": dropless variable-size grouped matmuls).

    Packed order groups kept routes by expert, tokens ascending within an expert; this
    is the stable argsort of the flattened expert ids of [MoE-271K] section 3, and the
    expert segment boundaries are the exclusive prefix sum of the kept counts
    (bincount + cumsum in the same section).

    Returns a dict:
      demand[E]      routes asking for each expert (before capacity)
      kept[E]        routes each expert accepts
      pos[T,k]       arrival position of each route in its expert
      route_row[T,k] row of the route in the packed buffer, -1 if dropped
      row_token[R]   token of each packed row (R = total kept)
      offsets[E+1]   segment starts; offsets[E] = R
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    count = np.zeros(E, dtype=np.int64)
    pos = np.zeros((T, k), dtype=np.int64)
    keep = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            if not 0 <= e < E:
                raise ValueError(f"expert id {e} out of range")
            pos[t, j] = count[e]
            count[e] += 1
            keep[t, j] = (C is None) or (pos[t, j] < C)
    demand = count.copy()
    kept = np.array([min(int(demand[e]), C) if C is not None else int(demand[e])
                     for e in range(E)], dtype=np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + kept[e]
    R = int(offsets[E])
    route_row = np.full((T, k), -1, dtype=np.int64)
    row_token = np.full(R, -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                e = int(ids[t, j])
                r = int(offsets[e] + pos[t, j])
                route_row[t, j] = r
                row_token[r] = t
    return dict(demand=demand, kept=kept, pos=pos, route_row=route_row,
                row_token=row_token, offsets=offsets)


OVERFLOW_DROP = "drop"
OVERFLOW_REROUTE = "reroute"


def dispatch_padded(ids, z, E: int, C: int, overflow: str = OVERFLOW_DROP):
    """The padded dispatch buffer [E, C, d] and its overflow policy.

    [MoE-S19] "Capacity" / "Visual support": capacity is a tensor dimension; expert e
    owns slots e*C .. e*C + C - 1, filled in arrival order, empty slots stay padding
    (the worked case: 16 assignments, 20 slots, 15 filled, 1 dropped).
    [MoE-S19] "Overflow policies": drop (the route is lost) or reroute (the overflowing
    route is handled by the next-best expert by score, the router decision overridden).

    Readings (the pages give no algorithm for reroute):
      * Phase 1 is the drop policy's arrival-order pass, unchanged.
      * Phase 2 takes the overflowed routes in arrival order (t, then j).  Each goes to
        the expert ranked best by the token's logits (descending, ties to the lower
        index) among those the token does not already hold and that still have a free
        slot; its slot is the next free one.  If there is none it is dropped.
      * A token's gates are then the gate mode applied to its final experts (slot j's
        reroute target, or its original expert, dropped or not); tokens without a
        rerouted route keep their gates.  ``reroute_gates`` does that step.

    Returns a dict:
      demand[E]       routes asking for each expert before capacity (router's choice)
      counts[E]       filled slots per expert after the policy
      final_ids[T,k]  expert that handles each route (the original when not rerouted)
      rerouted[T,k]   True where phase 2 moved the route
      route_row[T,k]  e*C + slot of the route, -1 if dropped
      row_token[E*C]  token in each slot, -1 for padding
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    if overflow not in (OVERFLOW_DROP, OVERFLOW_REROUTE):
        raise ValueError(f"unknown overflow policy {overflow!r}")
    count = np.zeros(E, dtype=np.int64)
    demand = np.zeros(E, dtype=np.int64)
    slot = np.full((T, k), -1, dtype=np.int64)
    final = ids.astype(np.int64).copy()
    rerouted = np.zeros((T, k), dtype=bool)
    overflowed = []
    for t in range(T):                      # phase 1: arrival order
        for j in range(k):
            e = int(ids[t, j])
            if not 0 <= e < E:
                raise ValueError(f"expert id {e} out of range")
            demand[e] += 1
            if count[e] < C:
                slot[t, j] = count[e]
                count[e] += 1
            else:
                overflowed.append((t, j))
    if overflow == OVERFLOW_REROUTE:        # phase 2: overflowed routes, arrival order
        zz = np.asarray(z, dtype=np.float64)
        for t, j in overflowed:
            held = set(int(e) for e in final[t])
            order = sorted(range(E), key=lambda e: (-zz[t, e], e))
            for e in order:
                if e not in held and count[e] < C:
                    final[t, j] = e
                    slot[t, j] = count[e]
                    count[e] += 1
                    rerouted[t, j] = True
                    break
    route_row = np.where(slot >= 0, final * C + slot, -1)
    row_token = np.full(E * C, -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if route_row[t, j] >= 0:
                row_token[route_row[t, j]] = t
    return dict(demand=demand, counts=count, final_ids=final, rerouted=rerouted,
                route_row=route_row, row_token=row_token)


def reroute_gates(z, final_ids, g, rerouted, mode: str) -> np.ndarray:
    """Gates after rerouting: the gate mode over each rerouted token's final experts."""
    g = np.array(g, dtype=np.float64, copy=True)
    for t in np.where(np.asarray(rerouted).any(axis=1))[0]:
        g[t] = gates(np.asarray(z)[t:t + 1], np.asarray(final_ids)[t:t + 1], mode)[0]
    return g


# ----------------------------------------------------------------------------------
# Compute: SwiGLU expert
# ----------------------------------------------------------------------------------

def silu(a):
    """SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a))."""
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def swiglu_expert(X, w_gate, w_up, w_down) -> np.ndarray:
    """down_proj(SiLU(gate_proj(X)) * up_proj(X)) on the rows of X.

    [MoE-VIS] "Expert Execution": each expert is the dense SwiGLU MLP.  Weights are in
    nn.Linear storage: w_gate, w_up [F, d]; w_down [d, F].  Rows are independent.
    """
    X = as_f64(X)
    g = X @ as_f64(w_gate).T
    u = X @ as_f64(w_up).T
    h = silu(g) * u
    return h @ as_f64(w_down).T


# ----------------------------------------------------------------------------------
# Whole layer
# ----------------------------------------------------------------------------------

def moe_layer(x, p: dict, k: int, mode: str, C: int | None = None,
              add_residual: bool = False, tokens=None, routing=None,
              layout: str = "ragged", overflow: str = OVERFLOW_DROP):
    """One MoE layer forward, the per-token loop of the pages.

    Steps ([MoE-271K] section 3 data path; [MoE-VIS] "Expert Execution"):
      1. route every token (logits, top-k, gates);
      2. capacity pass over all tokens in arrival order (drops depend on all tokens);
      3. gather the kept rows of each expert and run its SwiGLU (only the rows of the
         requested ``tokens`` are computed when a subset is given);
      4. per token, sum g * expert output over slots j = 0..k-1, add the shared expert
         (gate 1, [MoE-S19] "Top-k and mixture") and the residual x ([MoE-L] section 2
         step 9).

    ``p`` holds w_router [E,d], logit_bias [E] or None, w_gate/w_up [E,F,d],
    w_down [E,d,F] and optional shared_gate/shared_up [F,d], shared_down [d,F].
    ``routing`` = (ids, gates) or (ids, gates, logits) overrides step 1 (used to run
    the later steps on a given routing; the reroute policy needs the logits).
    ``layout`` "padded" uses the [E, C, d] buffer of ``dispatch_padded`` (C required),
    with ``overflow`` "drop" or "reroute".  Returns (y [len(tokens), d], info dict).
    """
    x64 = as_f64(x)
    T, d = x64.shape
    E = len(p["w_gate"])
    if routing is None:
        ids, g, z = route(x64, p["w_router"], p.get("logit_bias"), k, mode)
    else:
        ids, g = np.asarray(routing[0]), as_f64(routing[1])
        z = as_f64(routing[2]) if len(routing) > 2 else None
    if layout == "padded":
        if C is None:
            raise ValueError("the padded layout needs a capacity")
        disp = dispatch_padded(ids, z, E, C, overflow)
        g = reroute_gates(z, disp["final_ids"], g, disp["rerouted"], mode)
        disp["offsets"] = np.array([e * C for e in range(E)] + [E * C], dtype=np.int64)
        seg = [(e * C, e * C + int(disp["counts"][e])) for e in range(E)]
    elif layout == "ragged":
        if overflow != OVERFLOW_DROP:
            raise ValueError("the reroute policy uses the padded layout")
        disp = dispatch(ids, E, C)
        seg = [(int(disp["offsets"][e]), int(disp["offsets"][e + 1])) for e in range(E)]
    else:
        raise ValueError(f"unknown layout {layout!r}")
    route_row = disp["route_row"]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    want = np.zeros(T, dtype=bool)
    want[tokens] = True

    # 3. per expert: gather its kept rows (in packed order) that belong to wanted tokens
    out_rows = {}
    for e in range(E):
        lo, hi = seg[e]
        rows = [r for r in range(lo, hi) if want[disp["row_token"][r]]]
        if not rows:
            continue
        toks = disp["row_token"][rows]
        o = swiglu_expert(x64[toks], p["w_gate"][e], p["w_up"][e], p["w_down"][e])
        for r, orow in zip(rows, o):
            out_rows[r] = orow

    shared = None
    if p.get("shared_gate") is not None:
        shared = swiglu_expert(x64[tokens], p["shared_gate"], p["shared_up"], p["shared_down"])

    # 4. per-token combine in slot order
    y = np.zeros((len(tokens), d), dtype=np.float64)
    for i, t in enumerate(tokens):
        acc = np.zeros(d, dtype=np.float64)
        for j in range(k):
            r = int(route_row[t, j])
            if r >= 0:
                acc = acc + g[t, j] * out_rows[r]
        if shared is not None:
            acc = acc + shared[i]
        if add_residual:
            acc = acc + x64[t]
        y[i] = acc
    info = dict(ids=ids, gates=g, logits=z, **disp)
    return y, info


def round_to_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even), as float64.

    bfloat16 keeps 8 significant bits (1 implicit + 7 stored) and float32's exponent
    range.  Writing v = m * 2**e with 0.5 <= |m| < 1, the bf16 value is
    rint(m * 2**8) * 2**(e - 8), where rint rounds half to even.  Used only to model
    the bf16 storage of activations between chained layers.
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    r = np.ldexp(np.rint(m * 256.0), e - 8)
    r = np.where(np.abs(r) > 3.3895313892515355e38, np.copysign(np.inf, v), r)
    return r


def moe_stack(x0, layers: list, k: int, mode: str, C: int | None = None,
              bf16_activations: bool = True):
    """Layers chained by the residual: x_{l+1} = x_l + MoE_l(x_l).

    [MoE-271K] section 4 (Granite: 24 MoE layers, 32 experts, top-8) and [MoE-L]
    section 2 step 9 (residual addition).  With bf16 activations each layer's output is
    stored as bf16 before it feeds the next layer.  Returns (x_L, per-layer infos).
    """
    x = as_f64(x0)
    infos = []
    for p in layers:
        y, info = moe_layer(x, p, k, mode, C, add_residual=True)
        info["x_in"] = x
        x = round_to_bf16(y) if bf16_activations else y
        infos.append(info)
    return x, infos


# ----------------------------------------------------------------------------------
# Routing statistics
# ----------------------------------------------------------------------------------

def imbalance(demand) -> float:
    """I = max_e D_e / mean_e D_e on pre-capacity demand ([MoE-AEV] "Load imbalance")."""
    D = np.asarray(demand, dtype=np.float64)
    return float(np.max(D) / np.mean(D))


def drop_count(demand, C: int | None) -> int:
    """Routes dropped by capacity: sum_e max(0, D_e - C)."""
    if C is None:
        return 0
    return int(sum(max(0, int(D) - C) for D in demand))


def routing_stats(x, w_router, logit_bias, k: int, C: int | None, alpha: float = 1e-2,
                  ids=None, overflow: str = OVERFLOW_DROP):
    """Routing statistics of one layer call, in float64.

    f_e   fraction of routes dispatched to expert e before capacity (demand_e / (T k));
          [MoE-L] section 4 defines f_i as the fraction dispatched to expert i for top-1;
          with top-k the routes are counted, so that sum_e f_e = 1 as in the top-1 case.
    P_e   mean over tokens of the full softmax probability of expert e ([MoE-L] section 4,
          "the mean routing probability").
    aux   alpha * E * sum_e f_e P_e ([MoE-L] section 4; alpha = 1e-2 as reported there).
    I     max_e demand_e / mean_e demand_e on pre-capacity demand ([MoE-AEV] Load imbalance).
    drop  dropped routes / (T k); padding: empty slots / (E C) of the capacity buffer
          ([MoE-S19] Worked case: 20 slots, 15 used, 25% padding); 0 when dropless or
          C = 0 (no slots).
    With ``overflow`` "reroute" (padded buffer, ``dispatch_padded``) kept counts the
    routes placed after rerouting; f stays the router's pre-capacity choice.
    Returns a dict with those entries and kept (the number of kept routes).
    """
    z = router_logits(x, w_router, logit_bias)
    T, E = z.shape
    if ids is None:
        ids = top_k(z, k)
    if overflow == OVERFLOW_REROUTE and C is not None:
        d = dispatch_padded(ids, z, E, C, overflow)
        kept = int(d["counts"].sum())
    else:
        d = dispatch(ids, E, C)
        kept = int(d["kept"].sum())
    demand = d["demand"].astype(np.float64)
    f = demand / (T * k)
    P = softmax(z).mean(axis=0)
    return dict(f=f, P=P, aux=alpha * E * float(np.sum(f * P)), imbalance=imbalance(demand),
                drop_rate=(T * k - kept) / (T * k),
                padding_rate=(0.0 if not C else (E * C - kept) / (E * C)), kept=kept)
