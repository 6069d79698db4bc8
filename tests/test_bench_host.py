"""CPU checks of bench.py's host logic: the recorded DRAM traffic is used only
while the profiled kernel source is unchanged, the peak comes from the
measured-peaks file when it exists, and the argument rules of the timing
contract hold."""
import hashlib
import json
import os
import sys

import pytest

from tests.conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_traffic_is_read_while_the_kernel_source_matches(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    prof = tmp_path / "p.txt"
    prof.write_text(f"header\ntraffic_bytes_per_launch_full_size: 123456789\nkernel_source_sha256: {sha}\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCE", str(src))
    monkeypatch.setattr(bench, "TRAFFIC_FILES", {"c3": str(prof)})
    assert bench.recorded_traffic("c3") == 123456789.0
    assert bench.recorded_traffic("c4") is None  # no summary for that workload
    src.write_text("// kernel v2\n")  # the kernel changed since the capture
    assert bench.recorded_traffic("c3") is None
    prof.write_text("no figures here\n")
    assert bench.recorded_traffic("c3") is None


def test_committed_summaries_parse():
    for cfg, path in bench.TRAFFIC_FILES.items():
        assert os.path.exists(path), path
        text = open(path).read()
        assert "traffic_bytes_per_launch_full_size:" in text and "kernel_source_sha256:" in text
        assert "--clock-control none" in text  # the command that made it


def test_measured_peak_or_fallback(tmp_path, monkeypatch):
    root = tmp_path / "root"
    root.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.measured_peak_gbs() == (bench.FALLBACK_HBM_GBS, "fallback")
    (root / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6546.9}))
    assert bench.measured_peak_gbs() == (6546.9, "measured")
    (root / "MEASURED_PEAKS.json").write_text("{}")
    assert bench.measured_peak_gbs()[1] == "fallback"


def test_too_few_warmup_steps_are_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])


def test_every_config_has_a_workload_description():
    assert set(bench.CONFIGS) >= {"c1", "c2", "c3", "c4", "c5"}
    assert bench.U8_CONFIGS <= set(bench.CONFIGS)
    assert all(isinstance(v, str) and v for v in bench.CONFIGS.values())


def test_step_stats_median_min_max():
    st = bench.step_stats([0.3, 0.1, 0.2, 0.5, 0.4])
    assert st == {"median": 0.3, "min": 0.1, "max": 0.5, "n": 5}
    assert bench.step_stats([1.0])["median"] == 1.0


def test_extra_workloads_are_described_and_distinct():
    assert len(set(bench.EXTRA_CONFIGS)) == len(bench.EXTRA_CONFIGS)
    for c in bench.EXTRA_CONFIGS:
        assert bench.EXTRA_VARIANTS.get(c, (c, {}))[0] in bench.CONFIGS
    # every synthetic workload of the edge sweep has a full-size line
    assert {"edge_uniform", "edge_one_value", "edge_zipf"} <= set(bench.EXTRA_CONFIGS)
    assert bench.EDGE_N == 2 ** 26 + 13


def test_edge_workload_uses_the_parity_sweep_seed():
    from lossless_entropy_coded_dfloat11_b200 import inputs as I
    w = bench.make_workloads("edge_zipf", 0, "cpu")[0]
    ref = I.edge_case(bench.EDGE_N, "zipf", 500 + len(I.EDGE_SIZES) - 1)
    assert w.n_elems == bench.EDGE_N
    assert (w.flat_u16()[:4096] == ref.flat_u16()[:4096]).all()
