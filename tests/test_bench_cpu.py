"""CPU checks of bench.py's bookkeeping: the algorithmic MAC counts behind the roofline and
the lookup of the committed DRAM-traffic record (matched on kernel variant, workload and the
kernel source it was captured from)."""
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


def _record():
    path = os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")
    return json.load(open(path))


def test_traffic_record_matches_current_source():
    rec = _record()
    for name, r in rec.items():
        got = bench.kernel_traffic(name, r["precision"], r["workload_name"])
        assert got == r["dram_bytes_per_launch"], name


def test_traffic_record_needs_same_variant_and_workload():
    name, r = next(iter(_record().items()))
    other = "fp32" if r["precision"] != "fp32" else "split"
    assert bench.kernel_traffic(name, other, r["workload_name"]) is None
    assert bench.kernel_traffic(name, r["precision"], r["workload_name"] + "_other") is None
    assert bench.kernel_traffic("no_such_kernel", r["precision"], r["workload_name"]) is None


def test_traffic_record_ignored_once_the_kernel_source_changes(tmp_path, monkeypatch):
    name, r = next(iter(_record().items()))
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "tensor_train_compressed_mixed_b200" / "csrc"
    csrc.mkdir(parents=True)
    shutil.copy(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json"), root / "profiles")
    src = os.path.join(bench.ROOT, "tensor_train_compressed_mixed_b200", "csrc", r["source"])
    shutil.copy(src, csrc / r["source"])
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.kernel_traffic(name, r["precision"], r["workload_name"]) == r["dram_bytes_per_launch"]
    with open(csrc / r["source"], "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_traffic(name, r["precision"], r["workload_name"]) is None
