"""moe_dispatch_noalloc: the pack step for callers that cannot allocate device memory.

Some callers cannot give the library a workspace: a plugin that is handed only its
input and output buffers by a framework owning all device memory, a runtime whose memory
budget is fixed before start-up, or a hot path that must not call an allocator.  This
entry point keeps its scratch (the per-tile expert histogram) in a fixed array inside the
library.  The test calls it through the C ABI twice in a row, on different routings, and
checks every output against the fp64 oracle's dispatch on the same ids and against what
moe_dispatch (with a workspace) produces: the pack step is integer and byte work, so the
comparisons are exact.  A repeat call must leave the device's free memory and torch's
allocator unchanged.  It runs last (file name) and also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
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


def _call(lib, cfg, x, ids, out, status):
    return lib.moe_dispatch_noalloc(ctypes.byref(cfg), x.data_ptr(), ids.data_ptr(),
                                    out["x_packed"].data_ptr(), out["row_token"].data_ptr(),
                                    out["route_row"].data_ptr(), out["offsets"].data_ptr(),
                                    out["demand"].data_ptr(), status.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)


def test_noalloc_dispatch_matches_oracle_and_workspace_dispatch_twice():
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
        ids_h = I.random_ids(T, E, k, seed=T, skew=skew)
        ids = ids_h.to(dev)
        x_h = torch.randn((T, d), generator=torch.Generator().manual_seed(E)).to(torch.bfloat16)
        x = x_h.to(dev)
        out = _outputs(cfg, d, dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        code = _call(lib, cfg, x, ids, out, status)
        assert code == 0, N.moe_status_string(code)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # against the oracle: positions, drops, offsets, demand, packed order and bytes
        ref = O.dispatch(ids_h.numpy(), E, None if cap < 0 else cap)
        R = int(ref["offsets"][E])
        assert out["demand"].cpu().numpy().tolist() == ref["demand"].tolist()
        assert out["offsets"].cpu().numpy()[:E + 1].tolist() == ref["offsets"].tolist()
        assert int(out["offsets"][E + 1]) == R
        assert out["route_row"].cpu().numpy().tolist() == ref["route_row"].tolist()
        assert out["row_token"].cpu().numpy()[:R].tolist() == ref["row_token"].tolist()
        assert torch.equal(out["x_packed"][:R].cpu().view(torch.int16),
                           x_h.view(torch.int16)[torch.from_numpy(ref["row_token"])])
        # against the workspace entry point
        wref = _outputs(cfg, d, dev)
        ws = N.workspace(cfg)
        N.moe_dispatch(cfg, x, ids, None, wref["x_packed"], wref["row_token"], wref["route_row"],
                       wref["offsets"], wref["demand"], ws)
        assert N.moe_get_device_status(ws) == 0
        for key in ("route_row", "offsets", "demand"):
            assert torch.equal(out[key], wref[key]), key
        assert torch.equal(out["row_token"][:R], wref["row_token"][:R])
        assert torch.equal(out["x_packed"][:R].view(torch.int16), wref["x_packed"][:R].view(torch.int16))

    # a repeat call allocates nothing: device free memory and torch's allocator unchanged
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    code = _call(lib, cfg, x, ids, out, status)
    torch.cuda.synchronize()
    assert code == 0
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"

    # the padded [E, C, d] buffer (drop policy): every slot against the oracle
    T, E, k, C = 1000, 16, 4, 200
    cfg = N.make_config(T, d, E, k, 512, capacity=C, layout="padded")
    ids_h = I.random_ids(T, E, k, seed=5, skew=1.5)
    ids = ids_h.to(dev)
    x_h = torch.randn((T, d), generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    x = x_h.to(dev)
    out = _outputs(cfg, d, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    N.moe_dispatch_noalloc(cfg, x, ids, out["x_packed"], out["row_token"], out["route_row"],
                           out["offsets"], out["demand"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.dispatch_padded(ids_h.numpy(), None, E, C)
    assert out["route_row"].cpu().numpy().tolist() == ref["route_row"].tolist()
    assert out["row_token"].cpu().numpy().tolist() == ref["row_token"].tolist()
    assert out["demand"].cpu().numpy().tolist() == ref["demand"].tolist()
    offs = out["offsets"].cpu().numpy()
    assert offs[:E + 1].tolist() == [e * C for e in range(E + 1)]
    assert offs[E + 2:].tolist() == ref["counts"].tolist()
    filled = np.where(ref["row_token"] >= 0)[0]
    assert torch.equal(out["x_packed"][torch.from_numpy(filled).to(dev)].cpu().view(torch.int16),
                       x_h.view(torch.int16)[torch.from_numpy(ref["row_token"][filled])])
    # beyond the fixed array: rejected before any launch
    big = N.make_config(1 << 20, 128, 256, 2, 128)
    assert lib.moe_dispatch_noalloc(ctypes.byref(big), 1, 1, 1, 1, 1, 1, 1, None, None) == 2
