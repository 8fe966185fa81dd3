"""ep_forward (the expert-parallel layer composed from the library's route, dispatch, expert
FFN and combine entry points around the exchange) on one GPU: NCCL with world size 1.
Its exchange is then the identity, so the output must equal moe_forward bit for bit: each
output row sees the same arithmetic, only the entry points and the segment table handed to
the grouped GEMMs differ.  The exchange with two or more ranks is covered on gloo CPU ranks
(test_expert_parallel_cpu.py)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from routing_dispatch_expert_gemm_b200 import expert_parallel as EP
from routing_dispatch_expert_gemm_b200 import inputs as I
from routing_dispatch_expert_gemm_b200 import native as N

from harness import config_for, forward_gpu

pytestmark = pytest.mark.gpu
W = I.WORKLOADS


@pytest.fixture(scope="module")
def nccl_world1():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from routing_dispatch_expert_gemm_b200 import build
    build.build()
    N.lib()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("wl", [W["granite24"].with_(T=300, layers=1),
                                W["switch_phi125"].with_(T=512)],
                         ids=["granite_T300", "switch_phi125"])
def test_ep_forward_world1_equals_moe_forward(nccl_world1, wl):
    x, (p,) = I.make_inputs(wl, seed=11, device="cuda", layers=1)
    cfg = config_for(wl)
    ref = forward_gpu(cfg, x, p)
    assert ref["status"] == 0
    y = EP.ep_forward(cfg, x, p["w_router"], p["logit_bias"], p["w_gate"], p["w_up"],
                      p["w_down"])
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref["y"].view(torch.int16))


def test_ep_forward_rejects_unsupported_layouts(nccl_world1):
    wl = W["switch_phi125_reroute"].with_(T=64)
    cfg = config_for(wl)
    x = torch.zeros((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        EP.ep_forward(cfg, x, None, None, None, None, None)
