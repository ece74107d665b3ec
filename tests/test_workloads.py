"""Host checks of the seeded workload generator (no TT arithmetic here)."""
import numpy as np

from workloads import FeistelPermutation, config_workload, near_cubic_factors, zipf_ranks


def test_feistel_is_a_bijection():
    for n in (1, 2, 3, 17, 1000, 4097):
        p = FeistelPermutation(n, seed=n)
        y = p(np.arange(n))
        assert np.array_equal(np.sort(y), np.arange(n))


def test_zipf_ranks_in_range_and_skewed():
    r = zipf_ranks(np.random.default_rng(0), 1.1, 1000, 200000)
    assert r.min() >= 1 and r.max() <= 1000
    assert (r == 1).mean() > (r == 2).mean() > (r == 10).mean()


def test_near_cubic_factors_cover_rows():
    for N in (100000, 1234567, 40000000):
        n = near_cubic_factors(N)
        assert np.prod(n) >= N
        assert max(n) - min(n) <= 2


def test_config_workloads_are_seeded_and_shaped():
    a = config_workload(3, batch=64, tables=3)
    b = config_workload(3, batch=64, tables=3)
    assert np.array_equal(a.indices, b.indices)
    assert a.offsets.size == 3 * 64 + 1 and a.offsets[-1] == a.indices.size
    for t in range(3):
        lo, hi = a.offsets[t * 64], a.offsets[(t + 1) * 64]
        assert (a.indices[lo:hi] < a.n_rows[t]).all() and (a.indices[lo:hi] >= 0).all()
        assert [c.shape for c in a.cores[t]] == [(1, a.n[t][0], 4, 32), (32, a.n[t][1], 4, 32),
                                                 (32, a.n[t][2], 8, 1)]
    c4 = config_workload(4, batch=64, tables=3)
    assert np.array_equal(c4.indices, a.indices)          # same lookups, ranks 64
    assert c4.cores[0][1].shape[0] == 64 and c4.grad_out.shape == (64, 3 * 128)
    w1 = config_workload(1)
    assert w1.indices.size == 1024 and w1.dim == 16
    w5 = config_workload(5, batch=16, tables=2)
    assert w5.num_cores == 4 and w5.dim == 128 and (w5.indices < 10**9).all()
