"""Pins of the fp64 oracle against things other than itself.

Each test fixes the oracle to mathematics it must reproduce: the fully
materialised TT table (built with tensordot, a different route than the
oracle's per-row digit loop), the Kronecker product of rank-1 slices, the
plain embedding bag for k = 1, finite differences (exact here, because the
loss is affine in every single core entry), torch autograd of the
materialised table, numpy's row-major unravel for the mixed-radix digits, a
hand-derived worked example, and invariants of sum pooling.  A last group
plants plausible mistakes (transposed slice, reversed digit order, dropped
core) in the oracle's inputs and checks that the pins catch them.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
from workloads import random_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

SHAPES = [
    # (d, r, n per table, n_rows per table)
    ((3,), (1, 1), [(7,)], None),
    ((2, 3), (1, 4, 1), [(3, 5)], None),
    ((2, 3, 2), (1, 3, 2, 1), [(4, 3, 5)], None),
    ((1, 2, 3, 2), (1, 2, 3, 2, 1), [(3, 2, 2, 3)], None),
    ((2, 2, 2), (1, 2, 3, 1), [(3, 4, 2), (2, 2, 5)], [20, 17]),
]


def materialise(cores, n_rows=None):
    """The full table W [N, D] from the cores by tensordot (row-major rows and columns)."""
    k = len(cores)
    acc = cores[0][0]                       # [n1, d1, r1]  (r0 = 1 dropped)
    for j in range(1, k):
        acc = np.tensordot(acc, cores[j], axes=([-1], [0]))   # [..., n_j, d_j, r_j]
    acc = acc[..., 0]                       # r_k = 1
    # axes now: n1, d1, n2, d2, ..., nk, dk
    order = [2 * j for j in range(k)] + [2 * j + 1 for j in range(k)]
    W = np.transpose(acc, order)
    N = int(np.prod(W.shape[:k]))
    D = int(np.prod(W.shape[k:]))
    W = W.reshape(N, D)
    return W if n_rows is None else W[:n_rows]


def pool(W_list, w):
    T, B, D = w.num_tables, w.batch, w.dim
    out = np.zeros((B, T * D))
    for g in range(T * B):
        t, b = divmod(g, B)
        for l in range(w.offsets[g], w.offsets[g + 1]):
            out[b, t * D:(t + 1) * D] += W_list[t][w.indices[l]]
    return out


def as64(w):
    return [[c.astype(np.float64) for c in tab] for tab in w.cores]


@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_forward_equals_materialised_table(case):
    d, r, n, rows = SHAPES[case]
    w = random_workload(100 + case, d, r, n, rows, batch=9,
                        pooling={"kind": "uniform", "lo": 0, "hi": 6})
    Ws = [materialise(c, w.n_rows[t]) for t, c in enumerate(as64(w))]
    want = pool(Ws, w)
    got = oracle.workload_forward(w)
    assert got.shape == want.shape
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_rank_one_row_is_kronecker_product():
    d, r, n = (2, 3, 2, 2), (1, 1, 1, 1, 1), (3, 4, 2, 5)
    w = random_workload(7, d, r, [n], batch=2)
    cores = as64(w)[0]
    rng = np.random.default_rng(0)
    for i in rng.integers(0, int(np.prod(n)), size=20):
        dig = np.unravel_index(int(i), n)
        want = np.array([1.0])
        for j in range(len(d)):
            want = np.kron(want, cores[j][0, dig[j], :, 0])
        np.testing.assert_allclose(oracle.row(d, r, n, cores, int(i)), want, rtol=1e-14, atol=0)


def test_single_core_is_embedding_bag():
    torch = pytest.importorskip("torch")
    w = random_workload(11, (5,), (1, 1), [(13,)], batch=12,
                        pooling={"kind": "uniform", "lo": 0, "hi": 7})
    weight = torch.from_numpy(w.cores[0][0][0][:, :, 0].astype(np.float64))
    want = torch.nn.functional.embedding_bag(
        torch.from_numpy(w.indices), weight, torch.from_numpy(w.offsets), mode="sum",
        include_last_offset=True).numpy()
    np.testing.assert_allclose(oracle.workload_forward(w), want, rtol=1e-14, atol=1e-14)


def test_digits_are_row_major_unravel():
    n = (7, 3, 11, 5)
    rows = np.arange(int(np.prod(n)))
    want = np.stack(np.unravel_index(rows, n), axis=1)
    assert np.array_equal(oracle.digits(n, rows), want)


def test_golden_worked_example():
    vals = {}
    with open(os.path.join(GOLDEN, "tt_worked_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = np.array([float(x) for x in rest])
    n = tuple(int(x) for x in vals["n"])
    d = tuple(int(x) for x in vals["d"])
    r = tuple(int(x) for x in vals["r"])
    G1 = vals["G1"].reshape(r[0], n[0], d[0], r[1])
    G2 = vals["G2"].reshape(r[1], n[1], d[1], r[2])
    idx = vals["indices"].astype(np.int64)
    off = vals["offsets"].astype(np.int64)
    B = off.size - 1
    out = oracle.forward(d, r, [n], [4], [[G1, G2]], idx, off, B)
    assert np.array_equal(out.reshape(-1), vals["out"])
    g = vals["grad_out"].reshape(B, 2)
    dG = oracle.backward(d, r, [n], [4], [[G1, G2]], idx, off, B, g)[0]
    assert np.array_equal(dG[0].reshape(-1), vals["dG1"])
    assert np.array_equal(dG[1].reshape(-1), vals["dG2"])
    new = oracle.sgd([[G1, G2]], [dG], float(vals["lr"][0]))[0]
    assert np.array_equal(new[0].reshape(-1), vals["G1_after_sgd"])


def loss(w, cores):
    out = oracle.forward(w.d, w.r, w.n, w.n_rows, cores, w.indices, w.offsets, w.batch)
    return float(np.sum(out * w.grad_out.astype(np.float64)))


@pytest.mark.parametrize("case", [1, 2, 3, 4])
def test_backward_equals_central_differences(case):
    """L is affine in each single core entry, so the central difference is exact."""
    d, r, n, rows = SHAPES[case]
    w = random_workload(200 + case, d, r, n, rows, batch=5,
                        pooling={"kind": "uniform", "lo": 0, "hi": 4})
    base = as64(w)
    grads = oracle.workload_backward(w)
    rng = np.random.default_rng(case)
    h = 0.5
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            flat = base[t][j].size
            picks = rng.choice(flat, size=min(flat, 25), replace=False)
            # make sure touched entries are sampled too
            nz = np.flatnonzero(grads[t][j])
            if nz.size:
                picks = np.unique(np.concatenate([picks, rng.choice(nz, size=min(nz.size, 25))]))
            for e in picks:
                plus = [[c.copy() for c in tab] for tab in base]
                minus = [[c.copy() for c in tab] for tab in base]
                plus[t][j].reshape(-1)[e] += h
                minus[t][j].reshape(-1)[e] -= h
                fd = (loss(w, plus) - loss(w, minus)) / (2 * h)
                assert abs(fd - grads[t][j].reshape(-1)[e]) <= 1e-10 * (1 + abs(fd)), (t, j, e)


@pytest.mark.parametrize("case", [0, 2, 3, 4])
def test_backward_equals_torch_autograd(case):
    torch = pytest.importorskip("torch")
    d, r, n, rows = SHAPES[case]
    w = random_workload(300 + case, d, r, n, rows, batch=7,
                        pooling={"kind": "uniform", "lo": 0, "hi": 5})
    T, B, D = w.num_tables, w.batch, w.dim
    leaves = [[torch.tensor(c, dtype=torch.float64, requires_grad=True) for c in tab]
              for tab in as64(w)]
    out = torch.zeros(B, T * D, dtype=torch.float64)
    for t in range(T):
        acc = leaves[t][0][0]
        for j in range(1, w.num_cores):
            acc = torch.tensordot(acc, leaves[t][j], dims=([acc.dim() - 1], [0]))
        acc = acc[..., 0]
        k = w.num_cores
        W = acc.permute([2 * j for j in range(k)] + [2 * j + 1 for j in range(k)]).reshape(-1, D)
        W = W[:w.n_rows[t]]
        lo, hi = w.offsets[t * B], w.offsets[(t + 1) * B]
        bags = torch.repeat_interleave(torch.arange(B), torch.from_numpy(np.diff(w.offsets[t * B:(t + 1) * B + 1])))
        rowsel = W[torch.from_numpy(w.indices[lo:hi])]
        pooled = torch.zeros(B, D, dtype=torch.float64).index_add(0, bags, rowsel)
        out[:, t * D:(t + 1) * D] = pooled
    L = (out * torch.from_numpy(w.grad_out.astype(np.float64))).sum()
    L.backward()
    grads = oracle.workload_backward(w)
    for t in range(T):
        for j in range(w.num_cores):
            want = leaves[t][j].grad.numpy()
            np.testing.assert_allclose(grads[t][j], want, rtol=1e-12, atol=1e-12 * (1 + np.abs(want).max()))


def test_invariants_of_pooling():
    w = random_workload(17, (2, 2, 3), (1, 3, 2, 1), [(5, 4, 3)], batch=6,
                        pooling={"kind": "uniform", "lo": 1, "hi": 6})
    base = oracle.workload_forward(w)
    rng = np.random.default_rng(3)
    # permuting the indices inside each bag leaves the bag unchanged
    perm_idx = w.indices.copy()
    for g in range(w.batch):
        lo, hi = w.offsets[g], w.offsets[g + 1]
        perm_idx[lo:hi] = rng.permutation(perm_idx[lo:hi])
    got = oracle.forward(w.d, w.r, w.n, w.n_rows, w.cores, perm_idx, w.offsets, w.batch)
    np.testing.assert_allclose(got, base, rtol=1e-13, atol=1e-13)
    # duplicating every index doubles every bag
    dup_idx = np.repeat(w.indices, 2)
    got = oracle.forward(w.d, w.r, w.n, w.n_rows, w.cores, dup_idx, 2 * w.offsets, w.batch)
    np.testing.assert_allclose(got, 2 * base, rtol=1e-13, atol=1e-13)
    # splitting the batch into two calls gives the same rows
    h = 3
    a = oracle.forward(w.d, w.r, w.n, w.n_rows, w.cores, w.indices[:w.offsets[h]],
                       w.offsets[:h + 1], h)
    b = oracle.forward(w.d, w.r, w.n, w.n_rows, w.cores, w.indices[w.offsets[h]:],
                       w.offsets[h:] - w.offsets[h], w.batch - h)
    np.testing.assert_allclose(np.vstack([a, b]), base, rtol=1e-13, atol=1e-13)
    # scaling core j by s scales the rows by s and the other cores' gradients by s
    s = 1.75
    scaled = [[c.astype(np.float64) * (s if j == 1 else 1.0) for j, c in enumerate(tab)]
              for tab in w.cores]
    got = oracle.forward(w.d, w.r, w.n, w.n_rows, scaled, w.indices, w.offsets, w.batch)
    np.testing.assert_allclose(got, s * base, rtol=1e-13, atol=1e-13)
    g0 = oracle.workload_backward(w)[0]
    g1 = oracle.backward(w.d, w.r, w.n, w.n_rows, scaled, w.indices, w.offsets, w.batch,
                         w.grad_out)[0]
    np.testing.assert_allclose(g1[0], s * g0[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g1[2], s * g0[2], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g1[1], g0[1], rtol=1e-12, atol=1e-13)


def test_empty_bags_and_padding_rows():
    # n = (3, 4, 5) -> 60 rows, only 37 valid: i1 = 2 is reachable only from rows >= 40
    w = random_workload(19, (2, 1, 2), (1, 2, 2, 1), [(3, 4, 5)], [37], batch=8,
                        pooling={"kind": "explicit", "sizes": [0, 3, 0, 0, 5, 1, 0, 2]})
    out = oracle.workload_forward(w)
    for b in (0, 2, 3, 6):
        assert not out[b].any()
    grads = oracle.workload_backward(w)[0]
    assert not grads[0][:, 2].any()
    assert (w.indices < 37).all()
    bad = w.indices.copy()
    bad[0] = 37
    with pytest.raises(oracle.OracleError):
        oracle.forward(w.d, w.r, w.n, w.n_rows, w.cores, bad, w.offsets, w.batch)


def test_segmentation_equals_brute_force():
    w = random_workload(23, (2, 2, 2), (1, 2, 2, 1), [(3, 4, 5), (2, 3, 4)], [60, 21], batch=7,
                        pooling={"kind": "uniform", "lo": 0, "hi": 9})
    seg = oracle.workload_segmentation(w)
    T, B = w.num_tables, w.batch
    items = []
    for g in range(T * B):
        for l in range(w.offsets[g], w.offsets[g + 1]):
            items.append((g // B, int(w.indices[l]), l, g))
    items.sort(key=lambda x: (x[0], x[1], x[2]))
    assert seg["perm"].tolist() == [x[2] for x in items]
    assert seg["bag_sorted"].tolist() == [x[3] for x in items]
    uniq, starts = [], []
    for pos, (key, grp) in enumerate(itertools.groupby(enumerate(items), key=lambda e: e[1][:2])):
        first = next(grp)
        uniq.append(key)
        starts.append(first[0])
    starts.append(len(items))
    assert list(zip(seg["uniq_table"].tolist(), seg["uniq_row"].tolist())) == uniq
    assert seg["uniq_start"].tolist() == starts
    nk = [n[-1] for n in w.n]
    gstarts = [u for u in range(len(uniq))
               if u == 0 or (uniq[u][0], uniq[u][1] // nk[uniq[u][0]])
               != (uniq[u - 1][0], uniq[u - 1][1] // nk[uniq[u - 1][0]])]
    assert seg["grp_start"].tolist() == gstarts + [len(uniq)]


def test_sgd_closed_form():
    rng = np.random.default_rng(5)
    c = [[rng.normal(size=(1, 3, 2, 2))]]
    g = [[rng.normal(size=(1, 3, 2, 2))]]
    new = oracle.sgd(c, g, 0.25)[0][0]
    np.testing.assert_array_equal(new, c[0][0] - 0.25 * g[0][0])


# ---- the pins catch plausible mistakes (planted in the oracle's inputs, on the CPU) ----
def test_pins_catch_transposed_slice():
    d, r, n = (2, 3, 2), (1, 3, 3, 1), (4, 3, 5)
    w = random_workload(31, d, r, [n], batch=6)
    cores = as64(w)[0]
    W = materialise(cores)
    bad = [cores[0], np.ascontiguousarray(np.transpose(cores[1], (3, 1, 2, 0))), cores[2]]
    wrong = np.stack([oracle.row(d, r, n, bad, i) for i in range(W.shape[0])])
    assert not np.allclose(wrong, W, rtol=1e-6, atol=1e-9)


def test_pins_catch_reversed_digit_order():
    d, r, n = (2, 3, 2), (1, 3, 2, 1), (4, 3, 5)
    w = random_workload(37, d, r, [n], batch=6)
    cores = as64(w)[0]
    W = materialise(cores)
    # reading i_1 as the least significant digit is the same as reversing n
    rev = np.stack([oracle.digits(n[::-1], [i])[0][::-1] for i in range(W.shape[0])])
    right = oracle.digits(n, np.arange(W.shape[0]))
    assert not np.array_equal(rev, right)


def test_pins_catch_dropped_core():
    d, r, n = (2, 2, 2), (1, 1, 1, 1), (3, 3, 3)
    w = random_workload(41, d, r, [n], batch=4)
    cores = as64(w)[0]
    W = materialise(cores)
    ones = [cores[0], cores[1], np.ones_like(cores[2])]
    wrong = np.stack([oracle.row(d, r, n, ones, i) for i in range(W.shape[0])])
    assert not np.allclose(wrong, W)
