"""Parity at the benchmark sizes, in the launch configuration bench.py times.

The oracle cannot run a whole step at these sizes, so the tests check
  * the segmentation (sort, distinct rows, prefix groups, lookup-to-bag map) bit for bit
    against the oracle's numpy derivation, which does run at full size, including the
    64-bit sort keys of the eight 1e9-row tables;
  * the whole output where the oracle is cheap enough (one rank-16 table at batch 32768);
  * sampled bags: the GPU rows of a seeded sample of bags (plus the largest bags)
    against the oracle run on exactly those bags;
  * whole digit slices of the core gradients (and of the cores after the fused
    backward + SGD call bench.py times): only the lookups with that digit touch a slice,
    so the oracle run on those lookups alone gives it exactly;
  * a property of the backward that holds at any size: every pooled output is linear
    in each core, so for each table t and core j
        <dG_{t,j}, G_{t,j}> = <grad_out[:, t], out[:, t]>
    (Euler's identity for a function homogeneous of degree one in G_{t,j}).  The
    difference is measured against ||dG|| ||G|| + ||grad_out[:, t]|| ||out[:, t]||, the
    Cauchy-Schwarz bounds of the two inner products, so cancellation inside them does
    not inflate it.
"""
import numpy as np
import pytest

import oracle
from tests.parity import FP32_TOL, output_err
from workloads import config_workload, sub_batch

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def _sample_bags(w, n=48, seed=5):
    rng = np.random.default_rng(seed)
    sizes = np.diff(w.offsets).reshape(w.num_tables, w.batch).sum(axis=0)
    heavy = np.argsort(sizes)[-8:]
    return np.unique(np.concatenate([rng.choice(w.batch, size=n, replace=False), heavy]))


def _forward_full(w, options=None):
    import torch
    from tensor_train_compressed_mixed_b200 import from_workload
    emb, cores, idx, off = from_workload(w, options=options, with_grads=w.grad_out is not None)
    emb.reserve(w.num_lookups, w.batch)
    out = torch.empty(w.batch, w.num_tables * w.dim, dtype=torch.float32, device="cuda")
    emb.forward(idx, off, w.batch, out)
    emb.sync()
    return emb, cores, out


@pytest.mark.parametrize("cfg", [4, 5])
def test_full_size_forward_sampled_bags(cfg):
    w = config_workload(cfg, with_grad=False)
    emb, cores, out = _forward_full(w)
    bags = _sample_bags(w)
    got = out.cpu().numpy()[bags]
    want = oracle.workload_forward(sub_batch(w, bags))
    assert output_err(got, want, w.dim) <= FP32_TOL
    emb.close()


@pytest.mark.parametrize("cfg,prec", [(3, "bf16"), (3, "split"), (4, "bf16"), (4, "split")])
def test_full_size_tensor_core_forward_sampled_bags(cfg, prec):
    from tensor_train_compressed_mixed_b200 import abi
    w = config_workload(cfg, with_grad=False)
    o = abi.tt_emb_default_options()
    o.precision = abi.TT_PREC_BF16_TC if prec == "bf16" else abi.TT_PREC_FP32_SPLIT_TC
    emb, cores, out = _forward_full(w, o)
    bags = _sample_bags(w)
    got = out.cpu().numpy()[bags]
    want = oracle.workload_forward(sub_batch(w, bags))
    assert output_err(got, want, w.dim) <= (BF16_TOL if prec == "bf16" else FP32_TOL)
    emb.close()


@pytest.mark.parametrize("cfg", [4, 5])
def test_full_size_backward_euler_identity(cfg):
    import torch
    w = config_workload(cfg, with_grad=True)
    emb, cores, out = _forward_full(w)
    g = torch.from_numpy(w.grad_out).cuda()
    emb.backward(g)
    emb.sync()
    o64 = out.double().reshape(w.batch, w.num_tables, w.dim)
    g64 = g.double().reshape(w.batch, w.num_tables, w.dim)
    lhs_all = (o64 * g64).sum(dim=(0, 2)).cpu().numpy()
    lhs_scale = (o64.pow(2).sum(dim=(0, 2)).sqrt() * g64.pow(2).sum(dim=(0, 2)).sqrt()).cpu().numpy()
    worst = 0.0
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            G = cores[t][j].double()
            dG = emb.grads[t * w.num_cores + j].double()
            val = float((G * dG).sum())
            scale = float(G.norm() * dG.norm()) + float(lhs_scale[t])
            assert scale > 0, (t, j)
            worst = max(worst, abs(val - lhs_all[t]) / scale)
    assert worst <= FP32_TOL, worst
    emb.close()


def _digit_of(idx, n, j):
    stride = int(np.prod(n[j + 1:])) if j + 1 < len(n) else 1
    return (idx // stride) % n[j]


def _restrict(w, t, j, digit):
    """The lookups of table t whose core-j digit is `digit`, with the same bags and grad_out."""
    from workloads.gen import Workload
    T, B = w.num_tables, w.batch
    parts, sizes = [], np.zeros(T * B, dtype=np.int64)
    lo_t, hi_t = w.offsets[t * B], w.offsets[(t + 1) * B]
    seg = w.indices[lo_t:hi_t]
    keep = _digit_of(seg, w.n[t], j) == digit
    bag = np.repeat(np.arange(B), np.diff(w.offsets[t * B:(t + 1) * B + 1]))
    sizes[t * B:(t + 1) * B] = np.bincount(bag[keep], minlength=B)
    offsets = np.zeros(T * B + 1, dtype=np.int64)
    np.cumsum(sizes, out=offsets[1:])
    return Workload(name=w.name + "_slice", d=w.d, r=w.r, n=w.n, n_rows=w.n_rows, batch=B,
                    indices=seg[keep].astype(np.int64), offsets=offsets, cores=w.cores,
                    grad_out=w.grad_out, lr=w.lr, train=w.train, meta=dict(w.meta))


@pytest.mark.parametrize("prec", ["fp32", "split"])
def test_full_size_backward_sampled_slices(prec):
    """Whole digit slices dG_{t,j}[:, i] of the rank-64 training step: only the lookups
    with digit i touch the slice, so the oracle run on those lookups alone gives it."""
    import torch
    from tensor_train_compressed_mixed_b200 import abi
    from tests.parity import core_grad_err
    w = config_workload(4, with_grad=True)
    o = abi.tt_emb_default_options()
    o.precision = abi.TT_PREC_FP32 if prec == "fp32" else abi.TT_PREC_FP32_SPLIT_TC
    emb, cores, out = _forward_full(w, o)
    g = torch.from_numpy(w.grad_out).cuda()
    emb.backward(g)
    emb.sync()
    t = int(np.argmin([np.prod(x) for x in w.n]))   # the smallest table: fewest lookups per slice
    rng = np.random.default_rng(11)
    for j in range(w.num_cores):
        digit = int(rng.integers(0, w.n[t][j]))
        sub = _restrict(w, t, j, digit)
        assert sub.num_lookups > 0
        want = oracle.workload_backward(sub)[t][j][:, digit:digit + 1]
        got = emb.grads[t * w.num_cores + j][:, digit:digit + 1].cpu().numpy()
        assert core_grad_err(got, want) <= FP32_TOL, (j, digit)
    emb.close()


@pytest.mark.parametrize("cfg,tables", [(4, None), (5, None), (2, None)])
def test_full_size_segmentation_bit_exact(cfg, tables):
    """The grouping of the whole benchmark batch: 32-bit keys (26 tables of up to 4e7 rows, and
    one 1e7-row table) and 64-bit keys (eight 178^4 tables: 30 row bits + 3 table bits)."""
    from tests.test_gpu_parity import _seg_match
    w = config_workload(cfg, tables=tables, with_grad=False)
    emb, cores, out = _forward_full(w)
    seg = emb.segmentation()
    assert seg["sorted_keys"].dtype.itemsize == (8 if cfg == 5 else 4)
    _seg_match(emb, w)
    emb.close()


def test_full_size_single_table_forward_every_bag():
    """One 1e7-row rank-16 table at batch 32768: the oracle computes every bag."""
    w = config_workload(2, with_grad=False)
    assert w.batch == 32768
    emb, cores, out = _forward_full(w)
    want = oracle.workload_forward(w)
    assert output_err(out.cpu().numpy(), want, w.dim) <= FP32_TOL
    emb.close()


def _touched_digits(w, t, j, k, rng):
    """k digits of core j of table t that lookups touch: a seeded random pick among them."""
    lo, hi = w.offsets[t * w.batch], w.offsets[(t + 1) * w.batch]
    digits = np.unique(_digit_of(w.indices[lo:hi], w.n[t], j))
    return [int(x) for x in rng.choice(digits, size=min(k, digits.size), replace=False)]


def test_full_size_fused_backward_sgd_sampled_slices():
    """The call bench.py times on the rank-64 training step: tt_emb_backward_sgd in the
    split-bf16 mode, with the middle cores updated in place.  Digit slices of every core of
    three tables, after the step, against G - lr dG from the oracle run on the lookups that
    touch each slice; the slice's implied gradient (G_before - G_after) / lr is checked too."""
    import torch
    from tensor_train_compressed_mixed_b200 import abi
    from tests.parity import core_grad_err
    w = config_workload(4, with_grad=True)
    o = abi.tt_emb_default_options()
    o.precision = abi.TT_PREC_FP32_SPLIT_TC
    emb, cores, out = _forward_full(w, o)
    before = [[c.detach().cpu().numpy() for c in tab] for tab in cores]
    g = torch.from_numpy(w.grad_out).cuda()
    emb.backward_sgd(g, w.lr)
    emb.sync()
    rng = np.random.default_rng(21)
    sizes = [int(np.prod(x)) for x in w.n]
    tables = [int(np.argmin(sizes)), int(np.argmax(sizes)), int(rng.integers(0, w.num_tables))]
    for t in tables:
        for j in range(w.num_cores):
            after = cores[t][j].detach().cpu().numpy()
            for digit in _touched_digits(w, t, j, 2, rng):
                sub = _restrict(w, t, j, digit)
                dg = oracle.workload_backward(sub)[t][j][:, digit:digit + 1]
                g0 = before[t][j][:, digit:digit + 1].astype(np.float64)
                got = after[:, digit:digit + 1]
                assert core_grad_err(got, g0 - w.lr * dg) <= FP32_TOL, (t, j, digit)
                implied = (g0 - got.astype(np.float64)) / w.lr
                assert core_grad_err(implied, dg) <= FP32_TOL, (t, j, digit)
    emb.close()


def test_full_size_four_core_backward_sampled_slices():
    """The 178^4 workload (eight four-core tables, batch 65536, 90 % Zipf 1.4): digit slices of
    every core of two tables against the oracle run on the lookups that touch them."""
    import torch
    from tests.parity import core_grad_err
    w = config_workload(5, with_grad=True)
    emb, cores, out = _forward_full(w)
    g = torch.from_numpy(w.grad_out).cuda()
    emb.backward(g)
    emb.sync()
    rng = np.random.default_rng(31)
    for t in (0, int(rng.integers(1, w.num_tables))):
        for j in range(w.num_cores):
            for digit in _touched_digits(w, t, j, 2, rng):
                sub = _restrict(w, t, j, digit)
                if sub.num_lookups > 400_000:   # the hottest digits: keep the oracle to seconds
                    continue
                want = oracle.workload_backward(sub)[t][j][:, digit:digit + 1]
                got = emb.grads[t * w.num_cores + j][:, digit:digit + 1].cpu().numpy()
                assert core_grad_err(got, want) <= FP32_TOL, (t, j, digit)
    emb.close()
