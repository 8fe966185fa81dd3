"""moe_dispatch_noalloc: the pack step for callers that cannot allocate device memory.

Some callers cannot give the library a workspace: a plugin that is handed only its
input and output buffers by a framework owning all device memory, a runtime whose memory
budget is fixed before start-up, or a hot path that must not call an allocator.  This
entry point keeps its scratch (the per-tile expert histogram) in a fixed array inside the
library.  The test calls it through the C ABI twice in a row, on different routings, and
checks that every output equals what moe_dispatch (with a workspace) produces: the pack
step is integer and byte work, so the comparison is exact.  It runs last (file name) and
also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

from routing_dispatch_expert_gemm_b200 import inputs as I
from routing_dispatch_expert_gemm_b200 import native as N

pytestmark = pytest.mark.gpu


def _outputs(cfg, d, dev):
    rmax = N.moe_max_rows(cfg)
    return dict(x_packed=torch.zeros((rmax, d), dtype=torch.bfloat16, device=dev),
                row_token=torch.full((rmax,), -7, dtype=torch.int32, device=dev),
                route_row=torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev),
                offsets=torch.empty(N.offsets_len(cfg), dtype=torch.int32, device=dev),
                demand=torch.empty(cfg.E, dtype=torch.int32, device=dev))


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from routing_dispatch_expert_gemm_b200 import build
    build.build()
    lib = N.lib()
    dev = torch.device("cuda")
    d = 256
    cases = [(1412, 32, 8, 1.0, -1), (4096, 64, 2, 1.3, 128)]   # two calls in a row
    for T, E, k, skew, cap in cases:
        cfg = N.make_config(T, d, E, k, 512, capacity=cap)
        ids = I.random_ids(T, E, k, seed=T, skew=skew).to(dev)
        x = torch.randn((T, d), generator=torch.Generator().manual_seed(E)).to(torch.bfloat16).to(dev)
        ref = _outputs(cfg, d, dev)
        ws = N.workspace(cfg)
        N.moe_dispatch(cfg, x, ids, None, ref["x_packed"], ref["row_token"], ref["route_row"],
                       ref["offsets"], ref["demand"], ws)
        assert N.moe_get_device_status(ws) == 0
        out = _outputs(cfg, d, dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        code = lib.moe_dispatch_noalloc(ctypes.byref(cfg), x.data_ptr(), ids.data_ptr(),
                                        out["x_packed"].data_ptr(), out["row_token"].data_ptr(),
                                        out["route_row"].data_ptr(), out["offsets"].data_ptr(),
                                        out["demand"].data_ptr(), status.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
        assert code == 0, N.moe_status_string(code)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        R = int(ref["offsets"][E])
        for key in ("route_row", "offsets", "demand"):
            assert torch.equal(out[key], ref[key]), key
        assert torch.equal(out["row_token"][:R], ref["row_token"][:R])
        assert torch.equal(out["x_packed"][:R].view(torch.int16), ref["x_packed"][:R].view(torch.int16))
    # the padded [E, C, d] buffer (drop policy): the same comparison over every slot
    T, E, k, C = 1000, 16, 4, 200
    cfg = N.make_config(T, d, E, k, 512, capacity=C, layout="padded")
    ids = I.random_ids(T, E, k, seed=5, skew=1.5).to(dev)
    x = torch.randn((T, d), generator=torch.Generator().manual_seed(9)).to(torch.bfloat16).to(dev)
    ref = _outputs(cfg, d, dev)
    N.moe_dispatch(cfg, x, ids, None, ref["x_packed"], ref["row_token"], ref["route_row"],
                   ref["offsets"], ref["demand"], N.workspace(cfg))
    out = _outputs(cfg, d, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    N.moe_dispatch_noalloc(cfg, x, ids, out["x_packed"], out["row_token"], out["route_row"],
                           out["offsets"], out["demand"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for key in ("route_row", "offsets", "demand", "row_token"):
        assert torch.equal(out[key], ref[key]), key
    filled = ref["row_token"] >= 0
    assert int(filled.sum()) == int(ref["offsets"][E + 2:].sum())
    assert torch.equal(out["x_packed"][filled].view(torch.int16), ref["x_packed"][filled].view(torch.int16))
    # beyond the fixed array: rejected before any launch
    big = N.make_config(1 << 20, 128, 256, 2, 128)
    assert lib.moe_dispatch_noalloc(ctypes.byref(big), 1, 1, 1, 1, 1, 1, 1, None, None) == 2
