"""bench.py's host-side bookkeeping, on the CPU: rooflines, the traffic record
and the workload description.  The GPU timing itself is covered by running
bench.py on a B200."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from structured_attention_video_b200 import synth  # noqa: E402

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
         "sm_max_mhz": 1965.0}


def test_lstep_roofline_uses_the_algorithmic_flops_and_the_burst_peak():
    """The timed region is short and runs at boost clock: the burst GEMM figure is
    the peak; the sustained (power-capped) figure is only a side field."""
    wl = synth.WORKLOADS["720p"]
    flops = 4.0 * wl.N * wl.b1 * wl.d * wl.B * wl.H
    r = bench.kernel_roofline("tc_lstep_kernel", 1.0, wl, PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(flops / 1e-3 / 1e12)
    assert r["peak"] == 1600.0
    assert r["frac"] == pytest.approx(r["achieved"] / 1600.0)
    assert r["frac_of_sustained"] == pytest.approx(r["achieved"] / 1400.0)
    assert "burst" in r["peak_source"]


def test_clock_scaling_lowers_the_peak_to_the_run_clock():
    wl = synth.WORKLOADS["720p"]
    r = bench.kernel_roofline("tc_lstep_kernel", 1.0, wl, PEAKS, "measured")
    bench.clock_scaled(r, {"sm_mhz": 1965.0 / 2}, PEAKS)
    assert r["frac_at_run_clock"] == pytest.approx(2 * r["frac"])
    r2 = bench.kernel_roofline("tc_lstep_kernel", 1.0, wl, PEAKS, "measured")
    bench.clock_scaled(r2, {"sm_mhz": 1965.0}, PEAKS)
    assert r2["frac_at_run_clock"] == pytest.approx(r2["frac"])


def test_step_stats_percentiles():
    st = bench.step_stats([float(x) for x in range(1, 101)])
    assert st["median"] == pytest.approx(50.5)
    assert st["p10"] == pytest.approx(10.9)
    assert st["p90"] == pytest.approx(90.1)
    assert st["min"] == 1.0 and st["max"] == 100.0


def test_sampled_rel_err_compares_the_problem_rows():
    import numpy as np
    wl = synth.WORKLOADS["tiny"].replace(tiles=3)
    rng = np.random.default_rng(0)
    ref = {0: rng.standard_normal((wl.N, wl.d)), 1: rng.standard_normal((wl.N, wl.d))}
    probs = [(0, 0, 0), (1, 2, 7)]
    exact = bench.sampled_rel_err(wl, probs, ref, lambda bh, rows: ref[bh][rows])
    assert exact["value"] == 0.0
    assert exact["rows"] == sum(len(bench.problem_rows(wl, g, c)) for _, g, c in probs)
    off = bench.sampled_rel_err(wl, probs, ref, lambda bh, rows: 1.01 * ref[bh][rows])
    assert off["value"] == pytest.approx(0.01)
    # the rows of a problem are the tile's block rows at its column
    assert list(bench.problem_rows(wl, 1, 2)) == [u * wl.b2 + 2 for u in range(8, 16)]


def test_rstep_roofline_counts_every_tile():
    wl = synth.WORKLOADS["720p"]
    r = bench.kernel_roofline("tc_rstep_kernel", 2.0, wl, PEAKS, "measured")
    flops = 6.0 * wl.tiles * wl.N * wl.b2 * wl.d * wl.B * wl.H
    assert r["achieved"] == pytest.approx(flops / 2e-3 / 1e12)


def test_query_aggregation_is_bandwidth_bound():
    wl = synth.WORKLOADS["720p"]
    r = bench.kernel_roofline("tc_qbar_kernel", 0.05, wl, PEAKS, "measured")
    nbytes = wl.B * wl.H * wl.N * wl.d * 2
    assert r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(nbytes / 0.05e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6000.0)


def test_generic_kernels_report_against_the_alu_peak():
    wl = synth.WORKLOADS["480p_chunk"]
    r = bench.kernel_roofline("lstep_kernel", 1.0, wl, PEAKS, "measured")
    assert r["bound"] == "alu"
    assert r["peak"] == pytest.approx(148 * 128 * 2 * 1965.0e6 / 1e12)


def _fake_tree(tmp_path, source_text, recorded_text, header_text="h", recorded_header="h"):
    csrc = tmp_path / "structured_attention_video_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(source_text)
    (csrc / "k.cuh").write_text(header_text)
    (tmp_path / "profiles").mkdir()
    digest = hashlib.sha256((recorded_text + recorded_header).encode()).hexdigest()
    rec = {"tc_lstep_kernel": {"sources": ["k.cu", "k.cuh"], "sources_sha256": digest,
                               "dram_bytes_per_launch": 123.0}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))


def test_traffic_is_reported_for_the_source_it_was_measured_on(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "kernel v1", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("tc_lstep_kernel") == 123.0
    assert bench.kernel_traffic("tc_rstep_kernel") is None


def test_traffic_is_null_once_the_kernel_changed(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "kernel v2", "kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("tc_lstep_kernel") is None


def test_traffic_is_null_once_an_inlined_header_changed(tmp_path, monkeypatch):
    _fake_tree(tmp_path, "kernel v1", "kernel v1", header_text="h2", recorded_header="h1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("tc_lstep_kernel") is None


def test_committed_traffic_record_names_existing_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        rec = json.load(fh)
    for name, entry in rec.items():
        for src in entry["sources"]:
            assert os.path.exists(os.path.join(ROOT, "structured_attention_video_b200", "csrc",
                                               src)), name
        assert entry["dram_bytes_per_launch"] > 0


def test_workload_config_names_the_shape_and_the_l2_policy():
    wl = synth.WORKLOADS["720p"]
    cfg = bench.workload_config(wl, 2)
    assert cfg["N"] == 75600 and cfg["b1"] == 945 and cfg["b2"] == 80 and cfg["tiles"] == 4
    assert "720p" in cfg["workload"] and "x2" in cfg["parallelism"]
    assert "L2" in cfg["l2"]


def test_keytile_cpu_baseline_reports_the_oracle_time_and_error():
    """The key-tile line's CPU-baseline leg: the oracle's time scaled to a whole
    step, and the error of a device output that is the oracle's own output rounded
    to bfloat16 (so the error is the rounding alone)."""
    from oracle import oracle
    wl = synth.WORKLOADS["tiny"].replace(dtype="bf16", tiles=3)
    q, k, v = synth.make_inputs(wl)
    y = oracle.monarch_attn_keytiles(q, k, v, wl.b1, wl.b2, wl.tiles, wl.iters)
    bits = synth.to_device_bits(synth.round_to_dtype(y, "bf16"), "bf16")
    rec = bench.keytile_cpu_baseline(wl, bits, 4)
    assert rec["kind"] == "oracle" and rec["unit"] == "ms" and rec["value"] > 0
    assert rec["cores"] >= 1
    assert 0 < rec["rel_err"]["value"] < 4e-3
    assert rec["rel_err"]["rows"] % wl.b1 == 0
