"""Host-side logic of bench.py (no GPU): algorithmic bytes, the roofline bound
and the rule that ties a measured DRAM traffic figure to the kernel sources."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


SHAPE_7B = dict(B=8, NH=8, T=8192, DK=256, DV=512, L=256)
PEAKS = {"hbm_gbs": 6550.4, "bf16_tflops": 1646.3, "bf16_tflops_sustained": 1387.9,
         "sm_max_mhz": 1965.0}


def test_unfused_bytes_exceed_fused_by_the_state_round_trip_and_the_kv_reread(bench):
    s = SHAPE_7B
    args = (s["B"], s["NH"], s["T"], s["DK"], s["DV"], s["L"], 2)
    fused = bench.kernel_bytes("tc_fused", *args)
    g2 = bench.kernel_bytes("tc_states", *args)
    g3 = bench.kernel_bytes("tc_parallel", *args)
    BH, NC = s["B"] * s["NH"], s["T"] // s["L"]
    state_copy = BH * NC * (s["DK"] * s["DV"] * 2 + s["DK"] * 4)
    kv = BH * s["T"] * (s["DK"] + s["DV"]) * 2
    # G2 writes the states once and G3 reads them once; G2 reads K and V again.
    extra = (g2 + g3) - fused
    assert extra == pytest.approx(2 * state_copy + kv, rel=0.02)
    # The fused minimum is the pages' workload size: about 1.65 GB at this shape.
    assert 1.6e9 < fused < 1.7e9


def test_roofline_bound_follows_intensity(bench):
    s = SHAPE_7B
    shape = (s["B"], s["NH"], s["T"], s["DK"], s["DV"], s["L"], 2)
    fph = bench.flops_per_head(s["T"], s["DK"], s["DV"], s["L"])
    BH = s["B"] * s["NH"]
    g3_flops = BH * (fph["inter"] + fph["intra"])
    roof = bench.roofline("tc_parallel", 0.5, g3_flops, shape, PEAKS, "measured", False,
                          "not-a-profiled-workload")
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["intensity_flop_per_byte"] < roof["ridge_flop_per_byte"]
    assert roof["achieved"] == pytest.approx(roof["algorithmic_bytes"] / 0.5e-3 / 1e9)
    assert roof["traffic"] is None
    # A kernel whose intensity is above the ridge is reported against the tensor peak.
    big = bench.roofline("tc_parallel", 0.5, 1e3 * roof["algorithmic_bytes"], shape, PEAKS,
                         "measured", False, "x")
    assert big["bound"] == "tensor" and big["peak"] == PEAKS["bf16_tflops"]
    simt = bench.roofline("simt_parallel", 1.0, g3_flops, shape, PEAKS, "measured", False, "x")
    assert simt["bound"] == "alu"


def test_measured_traffic_is_dropped_when_the_sources_change(bench, monkeypatch):
    files = ["tc_parallel_wide.cu", "tc_ptx.cuh"]
    entry = {"bytes": 1.0e9, "sources": files,
             "sha1": bench.sources_sha1(files)}
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("tc_parallel", "probe"), entry)
    assert bench.measured_traffic("tc_parallel", "probe") == 1.0e9
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("tc_parallel", "probe"),
                        dict(entry, sha1="0" * 40))
    assert bench.measured_traffic("tc_parallel", "probe") is None
    assert bench.measured_traffic("tc_parallel", "no-such-workload") is None


def test_recorded_traffic_entries_name_existing_sources(bench):
    for (fam, workload), e in bench.MEASURED_TRAFFIC.items():
        for f in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "mlstm_chunkwise_b200", "csrc", f)), f
        assert len(e["sha1"]) == 40 and e["bytes"] > 0


def test_roofline_uses_the_methods_bytes(bench):
    """At the 7B shape the output kernel's method bytes are Q, K, V read and H
    written (1.617 GB); its own bytes add the bf16 chunk states, n and gates."""
    s = SHAPE_7B
    mb = bench.method_bytes("tc_parallel", s["B"], s["NH"], s["T"], s["DK"], s["DV"], 2, False)
    BH = s["B"] * s["NH"]
    assert mb == BH * s["T"] * (2 * s["DK"] + 2 * s["DV"]) * 2
    kb = bench.kernel_bytes("tc_parallel", s["B"], s["NH"], s["T"], s["DK"], s["DV"], s["L"], 2)
    assert kb > mb
    peaks = {"hbm_gbs": 6550.4, "bf16_tflops": 1646.3, "bf16_tflops_sustained": 1387.9}
    fph = bench.flops_per_head(s["T"], s["DK"], s["DV"], s["L"])
    flops = BH * (fph["inter"] + fph["intra"])
    roof = bench.roofline("tc_parallel", 0.5, flops,
                          (s["B"], s["NH"], s["T"], s["DK"], s["DV"], s["L"], 2), peaks,
                          "measured", False, "none")
    assert roof["bound"] == "hbm"
    assert abs(roof["frac"] - mb / 0.5e-3 / 1e9 / 6550.4) < 1e-12
    assert roof["frac_hbm_kernel_bytes"] > roof["frac"]
    assert abs(roof["frac_tensor"] - flops / 0.5e-3 / 1e12 / 1646.3) < 1e-12


def test_chunk_state_bytes_by_path(bench):
    s = SHAPE_7B
    args = (s["B"], s["NH"], s["T"], s["DK"], s["DV"], s["L"])
    BH, NC = s["B"] * s["NH"], s["T"] // s["L"]
    assert bench.chunk_state_bytes_written({"gates", "tc_fused"}, *args) == 0
    tc = bench.chunk_state_bytes_written({"gates", "tc_states", "tc_parallel"}, *args)
    simt = bench.chunk_state_bytes_written({"gates", "simt_states", "simt_parallel"}, *args)
    assert tc == BH * NC * (s["DK"] * s["DV"] * 2 + s["DK"] * 4)
    assert simt > tc  # fp32 states on the SIMT path
