"""Seeded synthetic workloads for the MoE layer forward.

This module only draws inputs; it holds none of the layer's arithmetic.  The same tensors
feed the CUDA path and the fp64 oracle.  Recipe (fixed draw order, fp32 draws rounded to
the storage type):  x, then per layer: router weight W_r [E, d], logit bias [E] (when
drawn), then per expert W_gate [F, d], W_up [F, d], W_down [d, F], then the shared expert.

Scales ("std" = standard deviation):
  tiny fp32      x ~ N(0,1); router and experts N(0, 1/d) as a variance (std d^-1/2)
  Granite-shaped x ~ N(0,1); all weights std 0.02; 24 layers chained by the residual
  Switch-shaped  x ~ N(0,1); weights std 0.02; logit bias [+1, 0, 0, -1]
  Mixtral-shaped x ~ N(0,1); weights std 0.02; logit bias -1.1 ln(e+1) (Zipf s = 1.1)
  64+1 shared    x ~ N(0,1); router std d^-1/2 so logits ~ N(0,1); bias ~ N(0, 0.5^2);
                 experts std 0.02
No dataset is involved: N(0,1) token states stand in for real prompts.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    d_ff: int
    dtype: str = "bf16"                # storage / arithmetic type of activations and weights
    gate_mode: str = "topk_softmax"
    phi: tuple | None = None           # capacity factor (num, den); None = dropless
    has_shared: bool = False
    add_residual: bool = False
    layers: int = 1
    router_std: float | None = 0.02    # None: d ** -0.5
    expert_std: float | None = 0.02    # None: d ** -0.5
    layout: str = "ragged"             # ragged | padded ([E, C, d] buffer; needs phi)
    overflow: str = "drop"             # drop | reroute (padded only)
    bias: str = "none"                 # none | switch | zipf | normal

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def _w(name, **kw):
    return Workload(name=name, **kw)


WORKLOADS = {
    "tiny_fp32": _w("tiny_fp32", T=64, d=64, E=4, k=2, d_ff=128, dtype="f32",
                    gate_mode="softmax_topk_renorm", router_std=None, expert_std=None),
    "granite24": _w("granite24", T=1412, d=1024, E=32, k=8, d_ff=512, gate_mode="topk_softmax",
                    add_residual=True, layers=24),
    "switch_dropless": _w("switch_dropless", T=4096, d=768, E=4, k=1, d_ff=2432,
                          gate_mode="softmax_topk", bias="switch"),
    "switch_phi050": _w("switch_phi050", T=4096, d=768, E=4, k=1, d_ff=2432,
                        gate_mode="softmax_topk", bias="switch", phi=(1, 2)),
    "switch_phi100": _w("switch_phi100", T=4096, d=768, E=4, k=1, d_ff=2432,
                        gate_mode="softmax_topk", bias="switch", phi=(1, 1)),
    "switch_phi125": _w("switch_phi125", T=4096, d=768, E=4, k=1, d_ff=2432,
                        gate_mode="softmax_topk", bias="switch", phi=(5, 4)),
    "mixtral_prefill": _w("mixtral_prefill", T=8192, d=4096, E=8, k=2, d_ff=14336,
                          gate_mode="topk_softmax", bias="zipf"),
    "mixtral_decode": _w("mixtral_decode", T=16, d=4096, E=8, k=2, d_ff=14336,
                         gate_mode="topk_softmax", bias="zipf"),
}
for _T in (1, 16, 256, 4096):
    for _phi, _tag in ((None, "dropless"), ((1, 1), "phi1"), ((2, 1), "phi2")):
        WORKLOADS[f"shared64_T{_T}_{_tag}"] = _w(
            f"shared64_T{_T}_{_tag}", T=_T, d=4096, E=64, k=2, d_ff=32768,
            gate_mode="softmax_topk_renorm", phi=_phi, has_shared=True, router_std=None,
            bias="normal")


# A scaled-down stand-in of the 64+1 layer for profiler captures (16 routed experts of
# d_ff = 8192 plus the shared one, 3.5 GB of weights; T = 1024 keeps T k / E = 128 rows per
# expert, the 64+1 layer's segment size at T = 4096).  Not a workload of the pages.
WORKLOADS["shared16_T1024_F8192"] = _w(
    "shared16_T1024_F8192", T=1024, d=4096, E=16, k=2, d_ff=8192,
    gate_mode="softmax_topk_renorm", has_shared=True, router_std=None, bias="normal")

# The Switch-shaped and 64+1 layers with capacity through the padded [E, C, d] buffer and
# the reroute overflow policy.
WORKLOADS["switch_phi125_reroute"] = WORKLOADS["switch_phi125"].with_(
    name="switch_phi125_reroute", layout="padded", overflow="reroute")
WORKLOADS["shared64_T4096_phi1_reroute"] = WORKLOADS["shared64_T4096_phi1"].with_(
    name="shared64_T4096_phi1_reroute", layout="padded", overflow="reroute")
# The same routing with d_ff = 1024 (x and the router are drawn before the experts, so the
# overflow and the reroute work are identical): a stand-in small enough for profiler
# captures of the reroute kernels.  Not a workload of the pages.
WORKLOADS["shared64_T4096_phi1_reroute_F1024"] = WORKLOADS["shared64_T4096_phi1_reroute"].with_(
    name="shared64_T4096_phi1_reroute_F1024", d_ff=1024)


def _randn(shape, gen, device, std, dtype):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(dtype)


def _bias(wl: Workload, gen, device):
    if wl.bias == "none":
        return None
    if wl.bias == "switch":
        return torch.tensor([1.0, 0.0, 0.0, -1.0], device=device)
    if wl.bias == "zipf":
        return torch.tensor([-1.1 * math.log(e + 1) for e in range(wl.E)], device=device)
    if wl.bias == "normal":
        return torch.randn(wl.E, generator=gen, device=device, dtype=torch.float32) * 0.5
    raise ValueError(wl.bias)


def make_layer(wl: Workload, gen, device, experts: bool = True) -> dict:
    """One layer's parameters (router, bias, stacked experts, optional shared expert).

    ``experts=False`` stops after the router and bias; the draws made are the same prefix
    of the stream as a full layer, so the router is identical either way."""
    dt = wl.torch_dtype
    rs = wl.router_std if wl.router_std is not None else wl.d ** -0.5
    es = wl.expert_std if wl.expert_std is not None else wl.d ** -0.5
    p = {"w_router": _randn((wl.E, wl.d), gen, device, rs, dt), "logit_bias": _bias(wl, gen, device)}
    if not experts:
        return p
    wg = torch.empty((wl.E, wl.d_ff, wl.d), dtype=dt, device=device)
    wu = torch.empty((wl.E, wl.d_ff, wl.d), dtype=dt, device=device)
    wd = torch.empty((wl.E, wl.d, wl.d_ff), dtype=dt, device=device)
    for e in range(wl.E):  # one expert at a time keeps the fp32 temporaries small
        wg[e] = _randn((wl.d_ff, wl.d), gen, device, es, dt)
        wu[e] = _randn((wl.d_ff, wl.d), gen, device, es, dt)
        wd[e] = _randn((wl.d, wl.d_ff), gen, device, es, dt)
    p.update(w_gate=wg, w_up=wu, w_down=wd)
    if wl.has_shared:
        p.update(shared_gate=_randn((wl.d_ff, wl.d), gen, device, es, dt),
                 shared_up=_randn((wl.d_ff, wl.d), gen, device, es, dt),
                 shared_down=_randn((wl.d, wl.d_ff), gen, device, es, dt))
    else:
        p.update(shared_gate=None, shared_up=None, shared_down=None)
    return p


def make_inputs(wl: Workload, seed: int = 0, device="cpu", layers: int | None = None,
                experts: bool = True):
    """Returns (x [T, d], [layer params ...]) drawn in the fixed order from one generator."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = _randn((wl.T, wl.d), gen, device, 1.0, wl.torch_dtype)
    n = wl.layers if layers is None else layers
    if not experts:
        return x, [make_layer(wl, gen, device, experts=False)]
    return x, [make_layer(wl, gen, device) for _ in range(n)]


def random_ids(T: int, E: int, k: int, seed: int = 0, skew: float = 1.0) -> torch.Tensor:
    """Distinct expert ids per token drawn with a Zipf-like preference (skew >= 0)."""
    gen = torch.Generator().manual_seed(seed)
    w = torch.tensor([(e + 1.0) ** -skew for e in range(E)])
    ids = torch.stack([torch.multinomial(w, k, replacement=False, generator=gen) for _ in range(T)])
    return ids.to(torch.int32)


def integer_router(wl: Workload, seed: int = 0, device="cpu", bias=None):
    """Token states and router weights with small integer values (|x| <= 3, |w| <= 2) and an
    optional integer logit bias.  Every product and partial sum of the logit contraction is
    an integer below 2**24, so fp32 accumulation in any order gives the exact logits: the
    GPU and an fp64 reference then rank experts identically, exact ties included.  Used to
    test the reroute policy, whose cascade depends on the full ranking of each token.
    Returns (x [T, d], w_router [E, d], logit_bias [E] fp32 or None)."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    dt = wl.torch_dtype
    x = torch.randint(-3, 4, (wl.T, wl.d), generator=gen).to(dt).to(device)
    w = torch.randint(-2, 3, (wl.E, wl.d), generator=gen).to(dt).to(device)
    b = None if bias is None else torch.tensor([float(v) for v in bias], device=device)
    return x, w, b
