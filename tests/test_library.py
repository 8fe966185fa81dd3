"""CPU checks of the C-ABI library: it builds, loads, exports every symbol that
include/moe.h declares, and its host-side logic (validation, capacity, sizes) is right.
No call here launches work on a GPU: every call either is pure host arithmetic or fails
validation before any CUDA call."""
import ctypes
import os
import re

import pytest

from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def native():
    from routing_dispatch_expert_gemm_b200 import build, native
    build.build()
    native.lib()
    return native


def header_functions():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(native):
    declared = header_functions()
    assert len(declared) >= 12
    assert sorted(native.EXPORTS) == declared
    lib = ctypes.CDLL(native.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert native.moe_abi_version() == native.ABI_VERSION == 5


def test_library_is_sm100a_build(native):
    from routing_dispatch_expert_gemm_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.ARCH


def test_capacity_matches_oracle(native):
    for T in (1, 7, 8, 16, 256, 1412, 4096, 8192):
        for k in (1, 2, 8):
            for E in (1, 4, 8, 32, 64):
                for num, den in ((1, 2), (1, 1), (5, 4), (3, 2), (2, 1)):
                    assert native.moe_capacity(T, k, E, num, den) == O.capacity(T, k, E, num, den)
    assert native.moe_capacity(8, 2, 4, 5, 4) == 5
    assert native.moe_capacity(8, 2, 0, 1, 1) == -1
    assert native.moe_capacity(8, 2, 4, 1, 0) == -1


def test_validation_and_sizes(native):
    cfg = native.make_config(64, 64, 4, 2, 128, dtype="f32", gate_mode="softmax_topk_renorm")
    assert native.moe_max_rows(cfg) == 128
    ws = native.moe_workspace_bytes(cfg)
    assert ws > 256 and ws % 256 == 0
    capped = native.make_config(4096, 768, 4, 1, 2432, capacity=512, gate_mode="softmax_topk")
    assert native.moe_max_rows(capped) == 2048
    zero = native.make_config(16, 128, 4, 1, 128, capacity=0)
    assert native.moe_max_rows(zero) == 1
    shared = native.make_config(16, 4096, 64, 2, 32768, has_shared=True,
                                gate_mode="softmax_topk_renorm")
    assert native.moe_workspace_bytes(shared) > native.moe_workspace_bytes(
        native.make_config(16, 4096, 64, 2, 32768, gate_mode="softmax_topk_renorm"))
    bad = [native.make_config(0, 64, 4, 2, 128),                  # T < 1
           native.make_config(8, 64, 4, 5, 128),                  # k > E
           native.make_config(8, 64, 4, 2, 128, gate_mode="topk_softmax")]
    bad[2].gate_mode = 7
    for c in bad:
        assert native.moe_workspace_bytes(c) == 0
    unsupported = [native.make_config(8, 96, 4, 2, 128),          # bf16 needs d % 128
                   native.make_config(8, 128, 300, 2, 128),       # E > 256
                   native.make_config(8, 64, 4, 2, 130, dtype="f32")]
    for c in unsupported:
        assert native.moe_workspace_bytes(c) == 0


def test_errors_return_before_any_launch(native):
    lib = native.lib()
    cfg = native.make_config(8, 128, 4, 2, 128)
    fake = 1 << 20  # never dereferenced: validation fails first
    # k > E: invalid config
    badk = native.make_config(8, 128, 4, 5, 128)
    assert lib.moe_route(ctypes.byref(badk), fake, fake, None, fake, fake, 256 * 4096, None) == 1
    # unaligned / missing workspace
    assert lib.moe_route(ctypes.byref(cfg), fake, fake, None, fake, fake, 12345, None) == 3
    assert lib.moe_route(ctypes.byref(cfg), fake, fake, None, fake, fake, None, None) == 3
    # null required pointers
    assert lib.moe_route(ctypes.byref(cfg), None, fake, None, fake, fake, 4096, None) == 1
    assert lib.moe_dispatch(ctypes.byref(cfg), fake, None, None, fake, fake, fake, fake, fake,
                            4096, None) == 1
    # the reroute policy rewrites the gates: they are required
    rr = native.make_config(8, 128, 4, 2, 128, capacity=4, layout="padded", overflow="reroute")
    assert lib.moe_dispatch(ctypes.byref(rr), fake, fake, None, fake, fake, fake, fake, fake,
                            4096, None) == 1
    assert lib.moe_combine(ctypes.byref(cfg), fake, fake, fake, None, None, None, None) == 1
    res = native.make_config(8, 128, 4, 2, 128, add_residual=True)
    assert lib.moe_combine(ctypes.byref(res), fake, fake, fake, fake, None, fake, None) == 1
    sh = native.make_config(8, 128, 4, 2, 128, has_shared=True)
    assert lib.moe_expert_ffn(ctypes.byref(sh), fake, fake, fake, fake, fake, fake, None, None,
                              None, fake, fake, 4096, None) == 1
    assert lib.moe_forward(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, None, None,
                           None, None, None, None, None, None, 4096, None) == 1
    # moe_forward_profiled takes 6 or 7 events, none of them NULL
    evs = (ctypes.c_void_p * 8)(*([fake] * 8))
    prof = lambda events, n: lib.moe_forward_profiled(
        ctypes.byref(cfg), fake, fake, None, fake, fake, fake, None, None, None, fake, None,
        None, None, None, events, n, 4096, None)
    for n in (0, 5, 8):
        assert prof(evs, n) == 1
    assert prof(None, 6) == 1
    holed = (ctypes.c_void_p * 7)(*([fake] * 6 + [None]))
    assert prof(holed, 7) == 1
    assert lib.moe_debug_bounded_wait(4096, 10, None) == 1
    assert native.moe_status_string(6).startswith("a bounded")


def test_routing_stats_arguments(native):
    lib = native.lib()
    fake = 1 << 20  # never dereferenced: validation fails first
    off = native.make_config(8, 128, 4, 2, 128)
    on = native.make_config(8, 128, 4, 2, 128, stats=True)
    # the statistics need the router's per-tile sums: cfg.stats = 0 is rejected
    assert lib.moe_routing_stats(ctypes.byref(off), fake, fake, 0.01, None, None, fake, 4096,
                                 None) == 1
    assert lib.moe_routing_stats(ctypes.byref(on), fake, fake, 0.01, None, None, None, 4096,
                                 None) == 1                              # summary required
    assert lib.moe_routing_stats(ctypes.byref(on), fake, fake, float("nan"), None, None, fake,
                                 4096, None) == 1
    assert lib.moe_routing_stats(ctypes.byref(on), fake, fake, 0.01, None, None, fake, 12345,
                                 None) == 3                              # misaligned workspace
    bad = native.make_config(8, 128, 4, 2, 128)
    bad.stats = 2
    assert native.moe_workspace_bytes(bad) == 0
    # the statistics scratch is only laid out when asked for
    big = dict(T=4096, d=4096, E=64, k=2, d_ff=1024)
    assert (native.moe_workspace_bytes(native.make_config(**big, stats=True))
            > native.moe_workspace_bytes(native.make_config(**big)))
    assert ctypes.sizeof(native.MoeRoutingSummary) == 32


def test_layout_and_overflow_validation(native):
    # the padded buffer is sized by the capacity; reroute needs the padded buffer
    assert native.moe_workspace_bytes(native.make_config(8, 128, 4, 2, 128, layout="padded")) == 0
    assert native.moe_workspace_bytes(native.make_config(
        8, 128, 4, 2, 128, capacity=4, overflow="reroute")) == 0
    bad = native.make_config(8, 128, 4, 2, 128, capacity=4)
    bad.layout = 2
    assert native.moe_workspace_bytes(bad) == 0
    pad = native.make_config(1000, 128, 8, 2, 256, capacity=300, layout="padded")
    assert native.moe_max_rows(pad) == 8 * 300                 # E*C even above T*k
    rag = native.make_config(1000, 128, 8, 2, 256, capacity=300)
    assert native.moe_max_rows(rag) == 2000
    assert native.offsets_len(pad) == 2 * 8 + 2 and native.offsets_len(rag) == 8 + 2
    rr = native.make_config(1000, 128, 8, 2, 256, capacity=300, layout="padded",
                            overflow="reroute")
    assert native.moe_workspace_bytes(rr) > native.moe_workspace_bytes(pad)
    lib = native.lib()
    fake = 1 << 20
    # no workspace for the router's logits: reroute is unsupported without allocation
    assert lib.moe_dispatch_noalloc(ctypes.byref(rr), fake, fake, fake, fake, fake, fake,
                                    fake, None, None) == 2
    assert lib.moe_dispatch_noalloc(ctypes.byref(native.make_config(
        8, 128, 4, 2, 128, layout="padded")), fake, fake, fake, fake, fake, fake, fake, None,
        None) == 1


def test_config_sweep_validation_and_sizes(native):
    """Random configs: valid ones get a 256-byte-aligned workspace and the documented row
    bound; each optional feature only adds scratch; invalid combinations are rejected."""
    import random
    rng = random.Random(0)
    for _ in range(400):
        E = rng.choice([1, 2, 4, 8, 32, 64, 200, 256])
        k = rng.randint(1, min(E, 32))
        T = rng.choice([1, 7, 128, 129, 1000, 4096])
        dtype = rng.choice(["bf16", "f32"])
        d = rng.choice([128, 256, 1024]) if dtype == "bf16" else rng.choice([4, 64, 100])
        F = rng.choice([128, 512]) if dtype == "bf16" else rng.choice([4, 128])
        cap = rng.choice([-1, 0, 1, 17, T * k])
        layout = rng.choice(["ragged", "padded"])
        overflow = rng.choice(["drop", "reroute"])
        cfg = native.make_config(T, d, E, k, F, dtype=dtype, capacity=cap, layout=layout,
                                 overflow=overflow, has_shared=rng.random() < 0.3,
                                 add_residual=rng.random() < 0.5, stats=rng.random() < 0.5)
        ws = native.moe_workspace_bytes(cfg)
        if layout == "padded" and cap < 0:
            assert ws == 0                       # the padded buffer needs C
            continue
        if overflow == "reroute" and layout != "padded":
            assert ws == 0                       # reroute fills the padded buffer's slots
            continue
        assert ws > 0 and ws % 256 == 0, (cfg, ws)
        rows = native.moe_max_rows(cfg)
        if layout == "padded":
            assert rows == max(E * cap, 1)
        else:
            assert rows == max(min(T * k, E * cap) if cap >= 0 else T * k, 1)
        base = native.make_config(T, d, E, k, F, dtype=dtype, capacity=cap, layout=layout)
        assert native.moe_workspace_bytes(base) <= ws


def test_ffn_tile_shape_choice(native):
    """Automatic tile shape: row tiles over SM pairs when the routed experts average at least
    512 rows (Mixtral- and Switch-shaped layers), else row tiles (the 64+1 layer, decode, the
    Granite-shaped layer); column tiles when asked for or when a fused step is requested;
    bad values and row tiles with fusion rejected."""
    mk = native.make_config
    assert native.moe_ffn_tile_shape(mk(4096, 4096, 64, 2, 32768, has_shared=True)) == "rows"
    assert native.moe_ffn_tile_shape(mk(16, 4096, 8, 2, 14336)) == "rows"
    assert native.moe_ffn_tile_shape(mk(1412, 1024, 32, 8, 512)) == "rows"
    assert native.moe_ffn_tile_shape(mk(8192, 4096, 8, 2, 14336)) == "row_pairs"
    assert native.moe_ffn_tile_shape(mk(4096, 768, 4, 1, 2432)) == "row_pairs"
    assert native.moe_ffn_tile_shape(mk(4096, 768, 4, 1, 2432, capacity=512)) == "row_pairs"
    assert native.moe_ffn_tile_shape(mk(4096, 768, 4, 1, 2432, capacity=511)) == "rows"
    assert native.moe_ffn_tile_shape(mk(2048, 640, 4, 1, 2432)) == "rows"  # d % 256
    assert native.moe_ffn_tile_shape(mk(8192, 4096, 8, 2, 14336, tiles="rows")) == "rows"
    assert native.moe_ffn_tile_shape(mk(16, 4096, 8, 2, 14336, tiles="row_pairs")) == "row_pairs"
    assert native.moe_ffn_tile_shape(mk(16, 640, 8, 2, 1024, tiles="row_pairs")) == "rows"
    assert native.moe_workspace_bytes(mk(8192, 4096, 8, 2, 14336, tiles="row_pairs",
                                         fuse="gather")) == 0
    assert native.moe_ffn_tile_shape(mk(8192, 4096, 8, 2, 14336, tiles="columns")) == "columns"
    assert native.moe_ffn_tile_shape(mk(16, 4096, 8, 2, 14336, tiles="rows")) == "rows"
    assert native.moe_ffn_tile_shape(mk(16, 4096, 8, 2, 14336, tiles="pairs")) == "pairs"
    assert native.moe_ffn_tile_shape(mk(16, 768, 4, 1, 2432, tiles="pairs")) == "rows"  # d % 256
    for fuse in ("gather", "combine", "gather+combine"):
        assert native.moe_ffn_tile_shape(mk(1412, 1024, 32, 8, 512, fuse=fuse)) == "columns"
        assert native.moe_workspace_bytes(mk(1412, 1024, 32, 8, 512, fuse=fuse, tiles="rows")) == 0
        assert native.moe_workspace_bytes(mk(64, 64, 4, 2, 128, dtype="f32", fuse=fuse)) == 0
    assert native.moe_workspace_bytes(mk(1412, 1024, 32, 8, 512, fuse="combine")) > \
        native.moe_workspace_bytes(mk(1412, 1024, 32, 8, 512))
    # the shared expert's segment on SM pairs next to row tiles: 4 FFN launches instead of 2
    assert native.moe_ffn_launches(mk(4096, 4096, 64, 2, 32768, has_shared=True)) == 4
    assert native.moe_ffn_launches(mk(1024, 512, 16, 2, 1024, has_shared=True)) == 4
    assert native.moe_ffn_launches(mk(511, 4096, 64, 2, 32768, has_shared=True)) == 2
    assert native.moe_ffn_launches(mk(4096, 4096, 64, 2, 32768, has_shared=True,
                                      tiles="rows")) == 2
    assert native.moe_ffn_launches(mk(8192, 4096, 8, 2, 14336)) == 2
    assert native.moe_ffn_launches(mk(64, 64, 4, 2, 128, dtype="f32", has_shared=True)) == 2
    bad = mk(16, 4096, 8, 2, 14336)
    bad.tiles = 5
    assert native.lib().moe_ffn_tile_shape(ctypes.byref(bad)) == 0
    assert native.lib().moe_ffn_launches(ctypes.byref(bad)) == 0
    assert native.moe_workspace_bytes(bad) == 0
