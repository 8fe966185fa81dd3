"""Host-side accounting of bench.py (no GPU): the algorithmic bytes / FLOPs model behind
every roofline fraction, and the lookup of ncu traffic figures by source fingerprint."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from routing_dispatch_expert_gemm_b200 import inputs as I  # noqa: E402


def test_granite_layer_costs():
    """Granite-shaped layer, dropless, all 32 experts touched: R = T k = 11,296 rows."""
    wl = I.WORKLOADS["granite24"]
    T, d, E, k, F = 1412, 1024, 32, 8, 512
    R = T * k
    c = bench.kernel_costs(wl, R, E)
    esz = 2
    assert c["gemm_gate_up"]["flops"] == 4.0 * R * d * F == pytest.approx(23.69e9, rel=1e-3)
    assert c["gemm_gate_up"]["bytes"] == E * 2 * F * d * esz + R * d * esz + R * F * esz
    assert c["gemm_gate_up"]["bytes"] == pytest.approx(101.8e6, rel=1e-3)
    assert c["gemm_down"]["flops"] == 2.0 * R * d * F
    assert c["gemm_down"]["bytes"] == pytest.approx(68.2e6, rel=1e-3)
    assert c["route"]["flops"] == 2.0 * T * d * E
    # the route count of the 24-layer stack
    assert R * 24 == 271104
    # combine: the kept rows, x for the output and the residual, and the route table
    assert c["combine"]["bytes"] == R * d * esz + T * d * esz * 2 + T * k * 8


def test_shared_expert_counts_as_an_extra_weight_set():
    wl = I.WORKLOADS["shared64_T16_dropless"]
    c0 = bench.kernel_costs(wl, 32, 20)
    # 20 touched routed experts + the shared one stream their weights; rows R + T
    assert c0["gemm_gate_up"]["bytes"] == (21 * 2 * wl.d_ff * wl.d + 48 * wl.d + 48 * wl.d_ff) * 2
    assert c0["gemm_down"]["flops"] == 2.0 * 48 * wl.d * wl.d_ff


def test_traffic_lookup_requires_matching_sources(tmp_path, monkeypatch):
    """A traffic figure counts only while the kernel's source is the one it was measured on."""
    sha = bench.source_sha("gemm_gate_up")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "x.md").write_text(
        f"traffic_bytes_per_launch gemm_gate_up@granite24 = 123456 sources {sha}\n"
        f"traffic_bytes_per_launch gemm_down@granite24 = 654321 sources 000000000000\n")
    src = os.path.join(ROOT, "routing_dispatch_expert_gemm_b200")
    os.symlink(src, tmp_path / "routing_dispatch_expert_gemm_b200")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("gemm_gate_up", "granite24") == 123456.0
    assert bench.traffic_from_profiles("gemm_down", "granite24") is None   # stale sources
    assert bench.traffic_from_profiles("gemm_gate_up", "mixtral_prefill") is None


def test_committed_granite_traffic_is_current_or_absent():
    """The committed profile either matches the current GEMM source or is ignored (never
    reported against a kernel it was not measured on)."""
    t = bench.traffic_from_profiles("gemm_gate_up", "granite24")
    assert t is None or 50e6 < t < 120e6


def test_default_workload_is_the_largest_single_gpu_configuration():
    """With no flags the headline is the 64+1 layer at T=4096 (the largest configuration that
    fits one GPU), and the other configurations follow under 'workloads'."""
    a = bench.parse_args([])
    wl = I.WORKLOADS[a.workload]
    assert (wl.T, wl.d, wl.E, wl.k, wl.d_ff, wl.has_shared) == (4096, 4096, 64, 2, 32768, True)
    sizes = {n: w.T * w.d * w.d_ff * (w.E + int(w.has_shared)) for n, w in I.WORKLOADS.items()}
    assert sizes[a.workload] == max(sizes.values())
    assert a.workload not in a.also
    for name in ("granite24", "mixtral_prefill", "mixtral_decode", "shared64_T16_dropless"):
        assert name in a.also
    assert a.warmup >= 3
    assert bench.parse_args(["--also", "none"]).also == []
    assert bench.parse_args(["--workload", "granite24", "--also", "granite24,mixtral_decode"]).also \
        == ["mixtral_decode"]


def test_oracle_sample_is_bounded_for_large_layers():
    """The CPU baseline computes every token of small layers and a few tokens of the layers
    whose experts are large (each touched expert costs 3 d F fp64 values)."""
    assert bench.oracle_tokens(I.WORKLOADS["tiny_fp32"]) is None
    assert bench.oracle_tokens(I.WORKLOADS["granite24"]) is None
    assert bench.oracle_tokens(I.WORKLOADS["mixtral_prefill"]) == 32
    assert bench.oracle_tokens(I.WORKLOADS["shared64_T4096_dropless"]) == 4
