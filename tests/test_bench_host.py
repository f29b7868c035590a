"""Host bookkeeping of bench.py on CPU: tile counts, algorithmic flop, the
config object, peak lookup and the traffic lookup keyed by kernel source."""
import json
import os
import shutil

import pytest

import bench
import synth


def test_tile_counts_and_flop_accounting():
    assert bench.tiles_of([1000, 128, 129], 2) == (8 * 8 + 1 + 2 * 2) * 2
    S, D, H = 75600, 128, 40
    dense = 4.0 * S * S * D * H
    assert bench.algorithmic_flop([S], D, H, 0.0) == pytest.approx(dense)
    assert bench.algorithmic_flop([S], D, H, 1.0) == pytest.approx(dense / 2)  # QK^T only
    assert bench.algorithmic_flop([S, 100], D, H, 0.5) == pytest.approx(3.0 * (S * S + 100 * 100) * D * H)
    assert synth.WAN14B.dense_flop() == pytest.approx(dense)


def test_config_object_is_shared_by_both_arms():
    cfg = bench.bench_config(synth.WAN14B, 1, "tsf=1")
    assert cfg["workload"] == synth.WAN14B.name and cfg["seq_len"] == 75600 and cfg["heads"] == 40
    assert cfg["head_dim"] == 128 and cfg["global_batch"] == 1 and cfg["threshold"] == "tsf=1"
    assert "inputs larger than L2" in cfg["l2"]


def _fake_root(tmp_path, traffic_records, peaks=None):
    src = os.path.join(bench.ROOT, "block_sparse_flashattention_ssa_b200", "csrc")
    dst = tmp_path / "block_sparse_flashattention_ssa_b200" / "csrc"
    dst.mkdir(parents=True)
    for f in ("ssa_kernel.cu", "sm100.cuh"):
        shutil.copy(os.path.join(src, f), dst / f)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(traffic_records))
    if peaks is not None:
        (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(peaks))
    return str(tmp_path)


def test_traffic_is_reported_only_for_the_profiled_kernel_source(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    root = _fake_root(tmp_path, [{"hash": h, "workload": "wan14b", "tsf": 24285.8487367675, "bytes": 3567250000},
                                 {"hash": h, "workload": "wan14b", "tsf": 0.0, "bytes": 3591750000},
                                 {"hash": "0000000000000000", "workload": "wan14b", "tsf": 5000.0, "bytes": 1}])
    monkeypatch.setattr(bench, "ROOT", root)
    path = os.path.join(root, "profiles", "traffic.json")
    assert bench.kernel_source_hash() == h
    assert bench.measured_traffic("wan14b", 24285.8487367675, path) == 3567250000.0
    assert bench.measured_traffic("wan14b", 0.0, path) == 3591750000.0
    assert bench.measured_traffic("wan14b", 5000.0, path) is None  # another kernel source
    assert bench.measured_traffic("wan5b", 0.0, path) is None
    # any edit of the kernel sources invalidates the stored counters
    with open(os.path.join(root, "block_sparse_flashattention_ssa_b200", "csrc", "sm100.cuh"), "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic("wan14b", 0.0, path) is None


def test_peaks_prefer_the_measured_file(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, [], peaks={"bf16_tflops": 1625.5, "bf16_tflops_sustained": 1389.3, "hbm_gbs": 6558})
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.peaks() == (1625.5, 1389.3, 6558, "measured")
    os.remove(os.path.join(root, "MEASURED_PEAKS.json"))
    assert bench.peaks()[3] == "fallback"


def test_threshold_sweeps_are_the_specified_values():
    """--tsf-sweep times the forward at the thresholds each workload is
    specified at; the S = 75,600 ones come from the pages' example formula
    tsf = 0.0003 * exp(7.5 * s) at s = 0.5 / 0.7 / 0.9."""
    assert bench.SWEEPS["tiny"] == [0.0, 100.0, 1000.0]
    assert bench.SWEEPS["wan5b"] == [0.0, 1e2, 1e3, 5e3, 2e4]
    assert bench.SWEEPS["varlen"] == [0.0, 5000.0]
    got = bench.SWEEPS["wan14b"]
    assert got[0] == 0.0
    for g, want in zip(got[1:], [0.012756, 0.057170, 0.256218]):
        assert abs(g - want) < 1e-6
