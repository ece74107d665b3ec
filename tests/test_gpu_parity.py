"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Segmentation is compared bit-exactly; pooled outputs, core gradients and the
SGD-updated cores within max relative error 1e-4 (fp32 accumulation), read
normwise per bag row / per digit slice (tests/parity.py).  Inputs are the seeded workloads of
workloads/gen.py: small random shapes for k = 1..4 (ragged and empty bags)
and the five benchmark shapes at batch sizes the oracle finishes in seconds
(several tiles of every kernel, with ragged tails).
"""
import numpy as np
import pytest

import oracle
from tests.parity import FP32_TOL, core_grad_err, gpu_forward, gpu_train_step, output_err
from workloads import config_workload, random_workload

pytestmark = pytest.mark.gpu

RANDOM_SHAPES = [
    ((5,), (1, 1), [(13,)], None),
    ((2, 3), (1, 4, 1), [(3, 5)], None),
    ((2, 3, 2), (1, 3, 2, 1), [(4, 3, 5)], None),
    ((1, 2, 3, 2), (1, 2, 3, 2, 1), [(3, 2, 2, 3)], None),
    ((2, 2, 2), (1, 2, 3, 1), [(3, 4, 2), (2, 2, 5), (7, 1, 3)], [20, 17, 19]),
    ((4, 4, 8), (1, 32, 32, 1), [(30, 31, 29), (11, 12, 13)], None),
    ((2, 4, 4, 4), (1, 16, 8, 16, 1), [(9, 8, 7, 6)], None),
]


def _seg_match(emb, w):
    got = emb.segmentation()
    want = oracle.workload_segmentation(w)
    kb = got["key_bits"]
    assert np.array_equal(got["perm"].astype(np.int64), want["perm"])
    uk = got["uniq_keys"].astype(np.uint64)
    assert np.array_equal((uk >> np.uint64(kb)).astype(np.int64), want["uniq_table"])
    assert np.array_equal((uk & np.uint64((1 << kb) - 1)).astype(np.int64), want["uniq_row"])
    assert np.array_equal(got["uniq_start"].astype(np.int64), want["uniq_start"])
    assert np.array_equal(got["grp_start"].astype(np.int64), want["grp_start"])
    assert np.array_equal(got["bag_sorted"].astype(np.int64), want["bag_sorted"])
    sk = got["sorted_keys"].astype(np.uint64)
    assert np.all(sk[1:] >= sk[:-1])


@pytest.mark.parametrize("case", range(len(RANDOM_SHAPES)))
def test_random_shapes_forward_and_segmentation(case):
    d, r, n, rows = RANDOM_SHAPES[case]
    w = random_workload(500 + case, d, r, n, rows, batch=37,
                        pooling={"kind": "uniform", "lo": 0, "hi": 9}, core_std=0.5)
    emb, cores, out = gpu_forward(w)
    _seg_match(emb, w)
    want = oracle.workload_forward(w)
    assert output_err(out.cpu().numpy(), want, w.dim) <= FP32_TOL


@pytest.mark.parametrize("case", range(len(RANDOM_SHAPES)))
def test_random_shapes_backward_and_sgd(case):
    d, r, n, rows = RANDOM_SHAPES[case]
    w = random_workload(600 + case, d, r, n, rows, batch=29,
                        pooling={"kind": "uniform", "lo": 0, "hi": 7}, core_std=0.5)
    emb, out, grads, new = gpu_train_step(w, lr=0.05)
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)
    upd = oracle.sgd(w.cores, want, 0.05)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(new[t][j], upd[t][j]) <= FP32_TOL, (t, j)


@pytest.mark.parametrize("cfg,batch,tables", [(1, None, None), (2, 300, None), (3, 48, 5),
                                              (4, 40, 4), (5, 24, 3)])
def test_benchmark_shapes_forward(cfg, batch, tables):
    w = config_workload(cfg, batch=batch, tables=tables, with_grad=False)
    emb, cores, out = gpu_forward(w)
    _seg_match(emb, w)
    want = oracle.workload_forward(w)
    assert output_err(out.cpu().numpy(), want, w.dim) <= FP32_TOL


@pytest.mark.parametrize("cfg,batch,tables", [(4, 24, 3), (5, 12, 2)])
def test_benchmark_shapes_backward(cfg, batch, tables):
    w = config_workload(cfg, batch=batch, tables=tables, with_grad=True)
    emb, out, grads, new = gpu_train_step(w, lr=0.01)
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)
    upd = oracle.sgd(w.cores, want, 0.01)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(new[t][j], upd[t][j]) <= FP32_TOL, (t, j)


def test_unique_only_grouping_gives_the_same_rows():
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(3, batch=32, tables=3, with_grad=False)
    o = abi.tt_emb_default_options()
    o.grouping = abi.TT_GROUP_UNIQUE_ONLY
    emb, cores, out = gpu_forward(w, options=o)
    seg = emb.segmentation()
    assert seg["num_groups"] == seg["num_unique"]
    want = oracle.workload_forward(w)
    assert output_err(out.cpu().numpy(), want, w.dim) <= FP32_TOL


def test_all_bags_empty_and_single_lookup():
    w = random_workload(77, (2, 2, 2), (1, 3, 3, 1), [(4, 4, 4)], batch=5,
                        pooling={"kind": "explicit", "sizes": [0, 0, 0, 0, 0]})
    emb, cores, out = gpu_forward(w, with_grads=True)
    assert not out.cpu().numpy().any()
    import torch
    emb.backward(torch.ones(5, 8, device="cuda"))
    emb.sync()
    assert all(not g.cpu().numpy().any() for g in emb.grads)
    w1 = random_workload(78, (2, 2, 2), (1, 3, 3, 1), [(4, 4, 4)], batch=1,
                         pooling={"kind": "explicit", "sizes": [1]})
    emb1, _, out1 = gpu_forward(w1)
    np.testing.assert_allclose(out1.cpu().numpy(), oracle.workload_forward(w1), rtol=1e-5, atol=1e-6)
