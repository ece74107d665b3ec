"""CPU checks of bench.py's bookkeeping: the algorithmic MAC counts behind the roofline and
the lookup of the committed DRAM-traffic record (matched on kernel variant, workload and the
kernel source it was captured from)."""
import hashlib
import json
import os
import shutil

import numpy as np
import pytest

import bench


def _chain_macs(d, r, upto):
    """MACs of a naive left-to-right contraction of the first `upto` slices of one row,
    counted one multiply-add at a time: the running product has prod(d[:j]) rows and r[j]
    columns; multiplying it by slice j (r[j] x d[j] r[j+1]) costs rows x r[j] x d[j] r[j+1]."""
    rows, macs = d[0], 0
    left = np.ones((d[0], r[1]))
    for j in range(1, upto):
        right = np.ones((r[j], d[j] * r[j + 1]))
        out = np.zeros((left.shape[0], right.shape[1]))
        for a in range(left.shape[0]):
            for b in range(right.shape[1]):
                for c in range(left.shape[1]):
                    out[a, b] += left[a, c] * right[c, b]
                    macs += 1
        rows *= d[j]
        left = out.reshape(rows, r[j + 1])
    return macs


@pytest.mark.parametrize("d,r", [
    ((2, 3, 2), (1, 2, 3, 1)),
    ((4, 4, 8), (1, 5, 3, 1)),
    ((2, 2, 3, 2), (1, 2, 3, 2, 1)),
])
def test_prefix_and_suffix_macs_match_a_counted_contraction(d, r):
    k = len(d)
    prefix = _chain_macs(d, r, k - 1)          # the shared chain: slices 1 .. k-1
    full = _chain_macs(d, r, k)                # the whole row
    assert bench.macs_per_prefix(d, r) == prefix
    assert bench.macs_per_suffix(d, r) == full - prefix


def test_benchmark_shape_counts():
    # rank 64, d = (4, 4, 8): 4 x 64 x 4 x 64 MACs per prefix group, 16 x 64 x 8 per distinct row
    assert bench.macs_per_prefix((4, 4, 8), (1, 64, 64, 1)) == 65536
    assert bench.macs_per_suffix((4, 4, 8), (1, 64, 64, 1)) == 8192


def _fake_repo(tmp_path, monkeypatch, source="fused_k3.cu"):
    """A copy of the kernel source with a traffic record taken on it (config 4, split mode,
    a capture of 2.2 M lookups moving 1.1 GB)."""
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "tensor_train_compressed_mixed_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = os.path.join(bench.ROOT, "tensor_train_compressed_mixed_b200", "csrc", source)
    shutil.copy(src, csrc / source)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    rec = {"bwd_fused": {"source": source, "source_sha": sha, "precision": "split", "config": 4,
                         "lookups": 2_200_000, "dram_bytes_per_launch": 1.1e9}}
    json.dump(rec, open(root / "profiles" / "ncu_traffic.json", "w"))
    monkeypatch.setattr(bench, "ROOT", str(root))
    return csrc / source


def test_traffic_record_is_scaled_by_lookups(tmp_path, monkeypatch):
    _fake_repo(tmp_path, monkeypatch)
    assert bench.kernel_traffic("bwd_fused", "split", 4, 2_200_000) == 1.1e9
    assert abs(bench.kernel_traffic("bwd_fused", "split", 4, 17_600_000) - 8.8e9) < 1.0


def test_traffic_record_needs_same_variant_and_workload(tmp_path, monkeypatch):
    _fake_repo(tmp_path, monkeypatch)
    assert bench.kernel_traffic("bwd_fused", "fp32", 4, 1000) is None
    assert bench.kernel_traffic("bwd_fused", "split", 3, 1000) is None
    assert bench.kernel_traffic("no_such_kernel", "split", 4, 1000) is None


def test_traffic_record_ignored_once_the_kernel_source_changes(tmp_path, monkeypatch):
    src = _fake_repo(tmp_path, monkeypatch)
    assert bench.kernel_traffic("bwd_fused", "split", 4, 2_200_000) == 1.1e9
    with open(src, "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_traffic("bwd_fused", "split", 4, 2_200_000) is None


def test_committed_traffic_records_are_well_formed():
    path = os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return
    for name, r in json.load(open(path)).items():
        assert {"source", "source_sha", "precision", "config", "lookups", "dram_bytes_per_launch"} <= set(r), name
        assert r["lookups"] > 0 and r["dram_bytes_per_launch"] > 0


def test_measured_peaks_fallback_and_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.measured_peaks()
    assert p["hbm_gbs"] == bench.FALLBACK_HBM_GBS and p["hbm_source"] == "of fallback"
    json.dump({"hbm": {"hbm_gbs": 6500.5}, "gemm": {"bf16_tflops": 1600.25, "bf16_tflops_sustained": 1400.0}},
              open(tmp_path / "MEASURED_PEAKS.json", "w"))
    p = bench.measured_peaks()
    assert p["hbm_gbs"] == 6500.5 and p["bf16_tflops"] == 1600.25
    assert p["hbm_source"].startswith("of measured")
