"""Parity of the bf16 tensor-core forward (TT_PREC_BF16_TC) with the fp64 oracle.

The prefix contraction C_p = G_1[0, i_1] . G_2[:, i_2] runs on tcgen05 with bf16
operands and fp32 accumulation in tensor memory; the bound is the pages' 2e-2 for a
bf16 tensor-core step, read normwise per bag row like the fp32 bound (tests/parity.py).
At rank 64 the backward's prefix-level products also run in bf16 on the tensor cores
(same 2e-2 bound per digit slice of the core gradients); at rank 32 the backward stays
fp32 and must agree with the fp32 handle's up to the order of the vector reductions.  Shapes: the two supported ones, with factors
that give several chunks per column group, ragged and empty bags.
"""
import numpy as np
import pytest

import oracle
from tests.parity import FP32_TOL, core_grad_err, gpu_forward, gpu_train_step, output_err
from workloads import config_workload, random_workload

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2

TC_SHAPES = [
    # d, r, n per table, rows per table, batch
    ((4, 4, 8), (1, 64, 64, 1), [(40, 3, 17), (9, 5, 11)], None, 300),
    ((4, 4, 8), (1, 32, 32, 1), [(70, 2, 13), (25, 7, 9), (3, 3, 3)], [1800, 1500, 20], 200),
]


def _opts(precision):
    from tensor_train_compressed_mixed_b200 import abi
    o = abi.tt_emb_default_options()
    o.precision = precision
    return o


@pytest.mark.parametrize("case", range(len(TC_SHAPES)))
def test_bf16_forward_matches_oracle(case):
    from tensor_train_compressed_mixed_b200 import abi
    d, r, n, rows, batch = TC_SHAPES[case]
    w = random_workload(900 + case, d, r, n, rows, batch=batch,
                        pooling={"kind": "uniform", "lo": 0, "hi": 40}, with_grad=False)
    emb, cores, out = gpu_forward(w, options=_opts(abi.TT_PREC_BF16_TC))
    got = out.cpu().numpy()
    want = oracle.workload_forward(w)
    err = output_err(got, want, w.dim)
    assert err <= BF16_TOL, err
    # bf16 rounding is visible: the result is not the fp32 one
    emb32, _, out32 = gpu_forward(w)
    assert output_err(out32.cpu().numpy(), want, w.dim) <= FP32_TOL
    assert not np.array_equal(got, out32.cpu().numpy())


@pytest.mark.parametrize("cfg,batch,tables", [(3, 64, 4), (4, 40, 3)])
def test_bf16_forward_benchmark_shapes(cfg, batch, tables):
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(cfg, batch=batch, tables=tables, with_grad=False)
    emb, cores, out = gpu_forward(w, options=_opts(abi.TT_PREC_BF16_TC))
    err = output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim)
    assert err <= BF16_TOL, err


def test_bf16_training_step_rank64():
    """Rank 64: the backward's prefix-level products (C recomputed, dG_1 = dC G_2^T,
    dG_2 = G_1^T dC) run on the tensor cores too; every core gradient and the SGD step
    stay within the bf16 bound per digit slice."""
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(4, batch=24, tables=3, with_grad=True)
    _, out_tc, g_tc, new_tc = gpu_train_step(w, options=_opts(abi.TT_PREC_BF16_TC), lr=0.01)
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(g_tc[t][j], want[t][j]) <= BF16_TOL, (t, j)
    upd = oracle.sgd(w.cores, want, 0.01)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(new_tc[t][j], upd[t][j]) <= BF16_TOL, (t, j)
    assert output_err(out_tc, oracle.workload_forward(w), w.dim) <= BF16_TOL


def test_bf16_training_step_many_chunks_per_column():
    """Small second factor: every column group holds several chunks, so dB accumulates in
    tensor memory across chunks before it is written."""
    from tensor_train_compressed_mixed_b200 import abi
    w = random_workload(960, (4, 4, 8), (1, 64, 64, 1), [(60, 2, 9), (33, 3, 5)], batch=120,
                        pooling={"kind": "uniform", "lo": 0, "hi": 30}, with_grad=True)
    _, out_tc, g_tc, _ = gpu_train_step(w, options=_opts(abi.TT_PREC_BF16_TC))
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(g_tc[t][j], want[t][j]) <= BF16_TOL, (t, j)


def test_bf16_rank32_training_keeps_fp32_backward():
    """Rank 32 has a tensor-core forward only; its backward is the FP32 one."""
    from tensor_train_compressed_mixed_b200 import abi
    w = random_workload(961, (4, 4, 8), (1, 32, 32, 1), [(20, 5, 9)], batch=60, with_grad=True)
    _, _, g_tc, _ = gpu_train_step(w, options=_opts(abi.TT_PREC_BF16_TC))
    _, _, g_32, _ = gpu_train_step(w)
    want = oracle.workload_backward(w)
    for j in range(w.num_cores):
        assert core_grad_err(g_tc[0][j], g_32[0][j]) <= 1e-5, j
        assert core_grad_err(g_tc[0][j], want[0][j]) <= FP32_TOL, j


def test_bf16_all_bags_empty():
    from tensor_train_compressed_mixed_b200 import abi
    w = random_workload(950, (4, 4, 8), (1, 64, 64, 1), [(5, 6, 7)], batch=16,
                        pooling={"kind": "uniform", "lo": 0, "hi": 0}, with_grad=False)
    assert w.num_lookups == 0
    emb, cores, out = gpu_forward(w, options=_opts(abi.TT_PREC_BF16_TC))
    assert not out.cpu().numpy().any()


def test_bf16_scheduler_modes_agree_bitwise():
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(3, batch=48, tables=4, with_grad=False)
    outs = []
    for sched in (abi.TT_SCHED_STATIC, abi.TT_SCHED_STEAL, abi.TT_SCHED_STEAL_L2):
        o = _opts(abi.TT_PREC_BF16_TC)
        o.sched = sched
        outs.append(gpu_forward(w, options=o)[2].cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


# ---------------------------------------------------------------------------
# TT_PREC_FP32_SPLIT_TC: two bf16 terms per operand value, three products; the fp32 bound
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", range(len(TC_SHAPES)))
def test_split_forward_meets_fp32_bound(case):
    from tensor_train_compressed_mixed_b200 import abi
    d, r, n, rows, batch = TC_SHAPES[case]
    w = random_workload(900 + case, d, r, n, rows, batch=batch,
                        pooling={"kind": "uniform", "lo": 0, "hi": 40}, with_grad=False)
    emb, cores, out = gpu_forward(w, options=_opts(abi.TT_PREC_FP32_SPLIT_TC))
    err = output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim)
    assert err <= FP32_TOL, err


@pytest.mark.parametrize("cfg,batch,tables", [(3, 64, 4), (4, 40, 3)])
def test_split_forward_benchmark_shapes(cfg, batch, tables):
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(cfg, batch=batch, tables=tables, with_grad=False)
    emb, cores, out = gpu_forward(w, options=_opts(abi.TT_PREC_FP32_SPLIT_TC))
    err = output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim)
    assert err <= FP32_TOL, err


def test_split_training_step_rank64_meets_fp32_bound():
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(4, batch=24, tables=3, with_grad=True)
    _, out, grads, new = gpu_train_step(w, options=_opts(abi.TT_PREC_FP32_SPLIT_TC), lr=0.01)
    assert output_err(out, oracle.workload_forward(w), w.dim) <= FP32_TOL
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)
    upd = oracle.sgd(w.cores, want, 0.01)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(new[t][j], upd[t][j]) <= FP32_TOL, (t, j)


def test_split_training_many_chunks_per_column():
    from tensor_train_compressed_mixed_b200 import abi
    w = random_workload(960, (4, 4, 8), (1, 64, 64, 1), [(60, 2, 9), (33, 3, 5)], batch=120,
                        pooling={"kind": "uniform", "lo": 0, "hi": 30}, with_grad=True)
    _, out, grads, _ = gpu_train_step(w, options=_opts(abi.TT_PREC_FP32_SPLIT_TC))
    assert output_err(out, oracle.workload_forward(w), w.dim) <= FP32_TOL
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)


@pytest.mark.parametrize("precision_name,tol", [("TT_PREC_FP32_SPLIT_TC", FP32_TOL), ("TT_PREC_BF16_TC", BF16_TOL)])
def test_rank64_training_chunks_beyond_row_table(precision_name, tol):
    """One column group of 20 prefixes with 64 last-digit values each, nearly every row
    looked up: the first 16-prefix chunk holds about 1000 distinct rows, more than the
    backward's per-chunk row table (512), so its later rows take the path that reads their
    keys from the sorted distinct keys; the forward splits the chunk into subtasks of at most
    256 rows, each with its own table."""
    from tensor_train_compressed_mixed_b200 import abi
    w = random_workload(962, (4, 4, 8), (1, 64, 64, 1), [(20, 1, 64)], batch=300,
                        pooling={"kind": "uniform", "lo": 10, "hi": 30}, with_grad=True)
    rows = np.unique(w.indices)
    assert len(rows[rows // 64 < 16]) > 512 + 100   # distinct rows of the first chunk
    _, out, grads, new = gpu_train_step(w, options=_opts(getattr(abi, precision_name)), lr=0.01)
    assert output_err(out, oracle.workload_forward(w), w.dim) <= tol
    want = oracle.workload_backward(w)
    for j in range(w.num_cores):
        assert core_grad_err(grads[0][j], want[0][j]) <= tol, j
    upd = oracle.sgd(w.cores, want, 0.01)
    for j in range(w.num_cores):
        assert core_grad_err(new[0][j], upd[0][j]) <= tol, j


@pytest.mark.parametrize("precision_name,tol", [("TT_PREC_FP32", FP32_TOL), ("TT_PREC_FP32_SPLIT_TC", FP32_TOL),
                                                ("TT_PREC_BF16_TC", BF16_TOL)])
def test_rank64_training_with_64bit_keys(precision_name, tol):
    """Three tables of 1.1e9 rows: 31 row bits + 2 table bits do not fit a 32-bit key, so
    the sort, the segmentation and the fused kernels run their 64-bit key variants."""
    from tensor_train_compressed_mixed_b200 import abi
    w = random_workload(963, (4, 4, 8), (1, 64, 64, 1), [(1100, 1000, 1000)] * 3, batch=64,
                        pooling={"kind": "uniform", "lo": 1, "hi": 8}, with_grad=True)
    _, out, grads, new = gpu_train_step(w, options=_opts(getattr(abi, precision_name)), lr=0.01)
    assert output_err(out, oracle.workload_forward(w), w.dim) <= tol
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(grads[t][j], want[t][j]) <= tol, (t, j)
    upd = oracle.sgd(w.cores, want, 0.01)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(new[t][j], upd[t][j]) <= tol, (t, j)
