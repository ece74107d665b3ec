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
    ((2, 4, 4, 4), (1, 16, 32, 32, 1), [(5, 6, 7, 9), (3, 4, 5, 6)], [1800, 300]),
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


def _forward_with(w, sched, grid):
    from tensor_train_compressed_mixed_b200 import abi
    o = abi.tt_emb_default_options()
    o.sched = sched
    o.grid = grid
    emb, cores, out = gpu_forward(w, options=o)
    return out.cpu().numpy()


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_scheduler_modes_and_grids_give_identical_rows(cfg):
    """Pooling sums each bag in bag order, so every schedule yields the same bits."""
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(cfg, batch=96, tables=3, with_grad=False)
    ref = _forward_with(w, abi.TT_SCHED_STEAL_L2, 0)
    assert output_err(ref, oracle.workload_forward(w), w.dim) <= FP32_TOL
    for sched in (abi.TT_SCHED_STATIC, abi.TT_SCHED_STEAL, abi.TT_SCHED_STEAL_L2):
        for grid in (1, 2, 5, 0):
            got = _forward_with(w, sched, grid)
            assert np.array_equal(got, ref), (sched, grid)


@pytest.mark.parametrize("sched", [0, 1, 2])
def test_scheduler_modes_backward(sched):
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(4, batch=32, tables=2, with_grad=True)
    o = abi.tt_emb_default_options()
    o.sched = sched
    o.grid = 3
    emb, out, grads, new = gpu_train_step(w, options=o)
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)


def test_single_hot_row_batch():
    """Every lookup hits one row: one group, one distinct row, ~5000 lookups split across warps."""
    from workloads.gen import Workload
    base = config_workload(4, batch=256, tables=1, with_grad=True)
    rng = np.random.default_rng(9)
    sizes = rng.integers(1, 40, size=base.batch)
    offsets = np.zeros(base.batch + 1, dtype=np.int64)
    np.cumsum(sizes, out=offsets[1:])
    hot = int(rng.integers(0, base.n_rows[0]))
    w = Workload(name="hot", d=base.d, r=base.r, n=base.n, n_rows=base.n_rows, batch=base.batch,
                 indices=np.full(offsets[-1], hot, dtype=np.int64), offsets=offsets,
                 cores=base.cores, grad_out=base.grad_out, train=True)
    emb, out, grads, new = gpu_train_step(w)
    assert output_err(out, oracle.workload_forward(w), w.dim) <= FP32_TOL
    want = oracle.workload_backward(w)
    for j in range(w.num_cores):
        assert core_grad_err(grads[0][j], want[0][j]) <= FP32_TOL, j


@pytest.mark.parametrize("cfg,batch,tables", [(3, 40, 3), (4, 24, 2), (5, 16, 2)])
def test_generic_and_specialised_paths_agree(cfg, batch, tables):
    """The shape-generic kernels and the specialised ones compute the same rows and gradients."""
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(cfg, batch=batch, tables=tables, with_grad=True)
    o = abi.tt_emb_default_options()
    o.force_generic = 1
    _, out_g, grads_g, _ = gpu_train_step(w, options=o)
    _, out_f, grads_f, _ = gpu_train_step(w)
    assert output_err(out_f, out_g, w.dim) <= FP32_TOL
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads_f[t][j], grads_g[t][j]) <= FP32_TOL, (t, j)


def _hot_prefix_workload(cfg, batch, seed):
    """Lookups concentrated on 32 prefixes (i_1 < 16, i_2 < 2) of each table, every last digit
    possible: chunks of thousands of distinct rows, split into many subtasks, so stealing and
    the C checkpoint of split chunks are exercised."""
    from workloads.gen import Workload
    base = config_workload(cfg, batch=batch, tables=2, with_grad=True)
    rng = np.random.default_rng(seed)
    T, B = base.num_tables, base.batch
    sizes = rng.integers(1, 48, size=T * B)
    offsets = np.zeros(T * B + 1, dtype=np.int64)
    np.cumsum(sizes, out=offsets[1:])
    idx = []
    for t in range(T):
        n1, n2, n3 = base.n[t]
        m = int(sizes[t * B:(t + 1) * B].sum())
        row = (rng.integers(0, 16, m) * n2 + rng.integers(0, 2, m)) * n3 + rng.integers(0, n3, m)
        idx.append(np.minimum(row, base.n_rows[t] - 1).astype(np.int64))
    return Workload(name="hot_prefixes", d=base.d, r=base.r, n=base.n, n_rows=base.n_rows, batch=B,
                    indices=np.concatenate(idx), offsets=offsets, cores=base.cores,
                    grad_out=base.grad_out, train=True)


@pytest.mark.parametrize("cfg,prec", [(3, "fp32"), (4, "split"), (3, "split")])
def test_split_chunks_stealing_and_checkpoint_give_identical_rows(cfg, prec):
    from tensor_train_compressed_mixed_b200 import abi
    w = _hot_prefix_workload(cfg, 1024, 40 + cfg)
    want = oracle.workload_forward(w)
    ref = None
    for sched in (abi.TT_SCHED_STATIC, abi.TT_SCHED_STEAL, abi.TT_SCHED_STEAL_L2):
        for grid in (1, 3, 7, 0):
            o = abi.tt_emb_default_options()
            o.sched, o.grid = sched, grid
            o.precision = abi.TT_PREC_FP32 if prec == "fp32" else abi.TT_PREC_FP32_SPLIT_TC
            emb, cores, out = gpu_forward(w, options=o)
            got = out.cpu().numpy()
            emb.close()
            if ref is None:
                ref = got
                assert output_err(got, want, w.dim) <= FP32_TOL
            assert np.array_equal(got, ref), (sched, grid)
    for chunk in (1, 32, 100, 256):   # subtask sizes: the rows are the same bits
        o = abi.tt_emb_default_options()
        o.chunk, o.grid = chunk, 7
        o.precision = abi.TT_PREC_FP32 if prec == "fp32" else abi.TT_PREC_FP32_SPLIT_TC
        emb, cores, out = gpu_forward(w, options=o)
        assert np.array_equal(out.cpu().numpy(), ref), chunk
        emb.close()


def test_balance_probe_counts_every_task():
    import torch
    from tensor_train_compressed_mixed_b200 import abi
    w = _hot_prefix_workload(4, 512, 7)
    o = abi.tt_emb_default_options()
    o.precision = abi.TT_PREC_FP32_SPLIT_TC
    o.grid = 6
    emb, cores, out = gpu_forward(w, options=o, with_grads=True)
    cap = 16
    rec = torch.zeros(2 * cap * 4, dtype=torch.int64, device="cuda")
    abi.tt_emb_set_probe(emb.handle, rec, cap)
    emb.forward(torch.from_numpy(w.indices).cuda(), torch.from_numpy(w.offsets).cuda(), w.batch, out)
    emb.backward(torch.from_numpy(w.grad_out).cuda())
    emb.sync()
    abi.tt_emb_set_probe(emb.handle, None, 0)
    r = rec.view(2, cap, 4).cpu().numpy()
    fwd, bwd = r[0][:6], r[1]
    assert (fwd[:, 1] > 0).all() and (fwd[:, 2] >= fwd[:, 1]).all()
    assert not r[0][6:].any()                              # blocks beyond the grid: no record
    n_pool = w.num_tables * ((w.batch + 63) // 64)
    assert int((fwd[:, 0] >> 32).sum()) >= n_pool + 1       # every pooling task and >= 1 subtask
    seg = emb.segmentation()
    assert (bwd[:, 1] > 0).sum() >= 1
    assert int((bwd[:, 0] >> 32).sum()) <= seg["num_groups"]   # columns taken, at most one per group
    assert output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim) <= FP32_TOL
