"""The expert-parallel exchange (experts sharded over ranks, two all-to-alls) on CPU ranks:
gloo, world size 2, rendezvous on 127.0.0.1.

Each rank routes and packs its own tokens over all E experts with the oracle, exchanges
the packed rows with ``expert_parallel``, runs the oracle's SwiGLU expert on its local
experts' rows only, returns the results and combines.  The output of every rank must equal
the oracle's single-process layer on that rank's tokens with all experts ("271,104
Routes", section 3, When the experts live on different GPUs: the result is the same as on
one GPU; only where the experts run changes).  The plan's counts, the order of the received
rows and a bit-exact round trip of bf16 rows are checked too.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O
from routing_dispatch_expert_gemm_b200 import expert_parallel as EP

E, d, F, k = 8, 32, 16, 2
TOKENS = (37, 50)  # per rank: the ranks' batches differ


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _params(shared):
    g = np.random.default_rng(7)
    p = dict(w_router=g.standard_normal((E, d)), logit_bias=g.standard_normal(E) * 0.5,
             w_gate=g.standard_normal((E, F, d)) / np.sqrt(d),
             w_up=g.standard_normal((E, F, d)) / np.sqrt(d),
             w_down=g.standard_normal((E, d, F)) / np.sqrt(F))
    if shared:
        p.update(shared_gate=g.standard_normal((F, d)) / np.sqrt(d),
                 shared_up=g.standard_normal((F, d)) / np.sqrt(d),
                 shared_down=g.standard_normal((d, F)) / np.sqrt(F))
    return p


def _ep_layer(x, p, C, shared, group=None):
    """The layer under expert parallelism, oracle arithmetic at every compute step."""
    W, r = dist.get_world_size(), dist.get_rank()
    mine = EP.experts_of(r, W, E)
    ids, g, _ = O.route(x, p["w_router"], p["logit_bias"], k, "softmax_topk")
    disp = O.dispatch(ids, E, C)
    x_packed = torch.from_numpy(x[disp["row_token"]])
    counts = torch.from_numpy(np.diff(disp["offsets"]))
    plan = EP.plan_exchange(counts, group)
    x_local = EP.exchange_rows(x_packed, plan, group).numpy()
    y_local = np.zeros_like(x_local)
    for i, e in enumerate(mine):  # only this rank's experts' weights are used
        lo, hi = int(plan.local_offsets[i]), int(plan.local_offsets[i + 1])
        if hi > lo:
            y_local[lo:hi] = O.swiglu_expert(x_local[lo:hi], p["w_gate"][e], p["w_up"][e],
                                             p["w_down"][e])
    y_packed = EP.return_rows(torch.from_numpy(y_local), plan, group).numpy()
    sh = (O.swiglu_expert(x, p["shared_gate"], p["shared_up"], p["shared_down"])
          if shared else None)
    y = np.zeros_like(x)
    for t in range(x.shape[0]):
        acc = np.zeros(d)
        for j in range(k):
            row = int(disp["route_row"][t, j])
            if row >= 0:
                acc = acc + g[t, j] * y_packed[row]
        if sh is not None:
            acc = acc + sh[t]
        y[t] = acc + x[t]
    return y, plan, disp


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = np.random.default_rng(100 + rank).standard_normal((TOKENS[rank], d))
        for case, (C, shared) in enumerate([(None, False), (6, True), (1, False)]):
            p = _params(shared)
            y, plan, disp = _ep_layer(x, p, C, shared)
            y_ref, _ = O.moe_layer(x, p, k, "softmax_topk", C=C, add_residual=True)
            out[(rank, case, "err")] = float(np.max(np.abs(y - y_ref)))
            out[(rank, case, "scale")] = float(np.max(np.abs(y_ref)))
            # plan: what is sent is every kept route, by destination; perm is a permutation
            out[(rank, case, "sent")] = (plan.rows_sent, int(disp["offsets"][E]))
            out[(rank, case, "perm")] = bool(torch.equal(torch.sort(plan.perm).values,
                                                         torch.arange(plan.rows_received)))
            kept = torch.from_numpy(np.diff(disp["offsets"])).reshape(world, E // world)
            gathered = [torch.zeros_like(kept) for _ in range(world)]
            dist.all_gather(gathered, kept)
            # rows from source s for local expert e = what s kept for global expert e
            want = torch.stack([gk[rank] for gk in gathered])
            out[(rank, case, "recv")] = bool(torch.equal(plan.recv_counts, want))
        # received rows are expert-major, source-major within an expert; a bf16 round
        # trip through both exchanges is bit-exact
        rows = torch.from_numpy(np.random.default_rng(rank).standard_normal((30, 16)))
        rows = rows.to(torch.bfloat16)
        counts = torch.tensor([3, 0, 5, 2, 4, 6, 1, 9] if rank == 0 else [1, 2, 0, 7, 3, 3, 8, 6])
        plan = EP.plan_exchange(counts)
        local = EP.exchange_rows(rows, plan)
        back = EP.return_rows(local, plan)
        out[(rank, "bf16")] = bool(torch.equal(back.view(torch.int16),
                                               rows[:plan.rows_sent].view(torch.int16)))
        allrows = [torch.zeros(30, 16, dtype=torch.bfloat16) for _ in range(world)]
        dist.all_gather(allrows, rows)
        allcounts = [torch.zeros_like(counts) for _ in range(world)]
        dist.all_gather(allcounts, counts)
        expect = []
        for i, e in enumerate(EP.experts_of(rank, world, E)):
            for s in range(world):
                lo = int(allcounts[s][:e].sum())
                expect.append(allrows[s][lo:lo + int(allcounts[s][e])])
        out[(rank, "order")] = bool(torch.equal(local.view(torch.int16),
                                                torch.cat(expect).view(torch.int16)))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_exchange_gloo_world2():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        for case in range(3):
            assert out[(rank, case, "err")] <= 1e-12 * max(1.0, out[(rank, case, "scale")])
            sent, kept = out[(rank, case, "sent")]
            assert sent == kept
            assert out[(rank, case, "perm")] and out[(rank, case, "recv")]
        assert out[(rank, "bf16")] and out[(rank, "order")]


def test_experts_of_blocks():
    assert list(EP.experts_of(0, 2, 8)) == [0, 1, 2, 3]
    assert list(EP.experts_of(3, 4, 8)) == [6, 7]
    try:
        EP.experts_of(0, 3, 8)
    except ValueError:
        pass
    else:
        raise AssertionError("8 experts do not divide over 3 ranks")
