"""Seeded synthetic workloads for TT-embedding gather.

This module only draws numbers: table shapes, TT cores, lookup indices, bag
offsets and upstream gradients.  It holds none of the TT arithmetic, so both
the fp64 oracle (``oracle/``) and the CUDA path consume exactly the same bytes
without sharing any of the method's code.

Shapes follow the five workloads of the TT-gather benchmark set:

1. one 3-core table, N = 1e6 (100x100x100), D = 16 (2x2x4), ranks (1,8,8,1),
   1024 bags of one uniform index, forward only;
2. one 3-core table, N = 1e7 (200x200x250), D = 64 (4x4x4), ranks
   (1,16,16,1), 32768 bags of Poisson(8)+1 Zipf(1.05) indices, forward;
3. 26 3-core tables, rows log-uniform in [1e5, 4e7] with near-cubic
   factors, D = 128 (4x4x8), ranks (1,32,32,1), 32768 samples with one bag
   per table of Poisson(20)+1 Zipf(1.1) indices, forward;
4. workload 3 with ranks (1,64,64,1): forward + backward + SGD (lr 0.01);
5. 8 4-core tables of 178^4 rows (1e9 valid), D = 128 (2x4x4x4), ranks
   (1,32,32,32,1), 65536 samples, bags of U{1..64} indices, 90 % Zipf(1.4)
   / 10 % uniform, forward + backward.

Conventions (the same on every side):
* cores of table t are float32 arrays ``G[j]`` of shape
  ``[r_{j-1}, n_j, d_j, r_j]`` with ``r_0 = r_k = 1``, drawn N(0, 0.1);
* indices are int64, table-major: the bags of table t occupy
  ``offsets[t*B] .. offsets[(t+1)*B]``; ``offsets`` is int64 of length
  ``T*B + 1`` with ``offsets[0] = 0`` and ``offsets[-1] = L``;
* the pooled output and its gradient are float32 ``[B, T*D]``: bag ``(t, b)``
  writes columns ``t*D .. (t+1)*D`` of row ``b``.

Zipf ranks are drawn with numpy's Zipf sampler and values above N are
rejected, so the law is exactly Zipf truncated to 1..N.  Ranks map to rows
through a seeded bijection of [0, N): a 4-round Feistel network over the
next even bit width, with the splitmix64 finaliser (Steele, Lea & Flood,
2014) as round function, and cycle walking (Black & Rogaway, 2002) to stay
inside [0, N).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BASE_SEED = 20260001
_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)


# --------------------------------------------------------------------------
# seeded bijection of [0, N)
# --------------------------------------------------------------------------
def _splitmix64(x: np.ndarray) -> np.ndarray:
    z = (x + np.uint64(0x9E3779B97F4A7C15)) & _M64
    z = ((z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)) & _M64
    z = ((z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)) & _M64
    return z ^ (z >> np.uint64(31))


class FeistelPermutation:
    """A seeded bijection of [0, n) (balanced Feistel + cycle walking)."""

    def __init__(self, n: int, seed: int):
        if n < 1:
            raise ValueError("n must be >= 1")
        self.n = int(n)
        bits = max(2, math.ceil(math.log2(max(self.n, 2))))
        bits += bits & 1
        self.half = bits // 2
        self.mask = np.uint64((1 << self.half) - 1)
        rng = np.random.default_rng(seed)
        self.keys = [np.uint64(k) for k in rng.integers(0, 2**63, size=4, dtype=np.int64)]

    def _round_trip(self, x: np.ndarray) -> np.ndarray:
        h = np.uint64(self.half)
        left = x >> h
        right = x & self.mask
        for k in self.keys:
            left, right = right, left ^ (_splitmix64(right ^ k) & self.mask)
        return (left << h) | right

    def __call__(self, x) -> np.ndarray:
        y = self._round_trip(np.asarray(x, dtype=np.uint64))
        bad = y >= np.uint64(self.n)
        while bad.any():
            y[bad] = self._round_trip(y[bad])
            bad = y >= np.uint64(self.n)
        return y.astype(np.int64)


# --------------------------------------------------------------------------
# index laws
# --------------------------------------------------------------------------
def zipf_ranks(rng: np.random.Generator, alpha: float, n: int, size: int) -> np.ndarray:
    """Zipf(alpha) over ranks 1..n (truncation by rejection), as int64."""
    out = np.empty(size, dtype=np.int64)
    filled = 0
    while filled < size:
        need = size - filled
        draw = rng.zipf(alpha, size=int(need * 1.25) + 64)
        draw = draw[(draw >= 1) & (draw <= n)]
        take = min(need, draw.size)
        out[filled:filled + take] = draw[:take]
        filled += take
    return out


def _draw_indices(rng, law: dict, n_rows: int, size: int, perm: FeistelPermutation):
    kind = law["kind"]
    if kind == "uniform":
        return rng.integers(0, n_rows, size=size, dtype=np.int64)
    if kind == "zipf":
        return perm(zipf_ranks(rng, law["alpha"], n_rows, size) - 1)
    if kind == "mix":  # per index: Zipf with probability p_zipf, else uniform
        pick = rng.random(size) < law["p_zipf"]
        out = rng.integers(0, n_rows, size=size, dtype=np.int64)
        nz = int(pick.sum())
        out[pick] = perm(zipf_ranks(rng, law["alpha"], n_rows, nz) - 1)
        return out
    raise ValueError(f"unknown index law {kind!r}")


def _draw_bag_sizes(rng, pooling: dict, batch: int) -> np.ndarray:
    kind = pooling["kind"]
    if kind == "fixed":
        return np.full(batch, pooling["size"], dtype=np.int64)
    if kind == "poisson_plus1":
        return rng.poisson(pooling["mean"], size=batch).astype(np.int64) + 1
    if kind == "uniform":
        return rng.integers(pooling["lo"], pooling["hi"] + 1, size=batch, dtype=np.int64)
    if kind == "explicit":
        return np.asarray(pooling["sizes"], dtype=np.int64)
    raise ValueError(f"unknown pooling law {kind!r}")


# --------------------------------------------------------------------------
# workload container
# --------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    d: tuple                       # d_1..d_k
    r: tuple                       # r_0..r_k (r_0 = r_k = 1)
    n: list                        # per table: (n_1..n_k)
    n_rows: list                   # per table: valid rows N_t <= prod(n)
    batch: int                     # B (bags per table)
    indices: np.ndarray            # int64 [L], table-major
    offsets: np.ndarray            # int64 [T*B + 1]
    cores: list                    # per table: list of k float32 arrays
    grad_out: np.ndarray | None = None   # float32 [B, T*D]
    lr: float = 0.01
    train: bool = False
    meta: dict = field(default_factory=dict)

    @property
    def num_tables(self) -> int:
        return len(self.n)

    @property
    def num_cores(self) -> int:
        return len(self.d)

    @property
    def dim(self) -> int:
        return int(np.prod(self.d))

    @property
    def num_lookups(self) -> int:
        return int(self.indices.size)

    def n_matrix(self) -> np.ndarray:
        return np.asarray(self.n, dtype=np.int64).reshape(self.num_tables, self.num_cores)


def draw_cores(seed: int, n: tuple, d: tuple, r: tuple, std: float = 0.1) -> list:
    rng = np.random.default_rng(seed)
    return [rng.normal(0.0, std, size=(r[j], n[j], d[j], r[j + 1])).astype(np.float32)
            for j in range(len(d))]


def build_workload(name, d, r, n_list, n_rows_list, batch, pooling, law, index_seeds,
                   core_seeds, grad_seed=None, train=False, lr=0.01, perm_seeds=None,
                   core_std=0.1) -> Workload:
    """Assemble a workload from explicit shapes, laws and per-table seeds."""
    T = len(n_list)
    idx_parts, sizes_parts = [], []
    for t in range(T):
        rng = np.random.default_rng(index_seeds[t])
        sizes = _draw_bag_sizes(rng, pooling, batch)
        perm = FeistelPermutation(n_rows_list[t], (perm_seeds or index_seeds)[t] ^ 0x5EED)
        idx = _draw_indices(rng, law, n_rows_list[t], int(sizes.sum()), perm)
        idx_parts.append(idx)
        sizes_parts.append(sizes)
    sizes = np.concatenate(sizes_parts)
    offsets = np.zeros(T * batch + 1, dtype=np.int64)
    np.cumsum(sizes, out=offsets[1:])
    indices = np.concatenate(idx_parts).astype(np.int64)
    cores = [draw_cores(core_seeds[t], tuple(n_list[t]), tuple(d), tuple(r), core_std)
             for t in range(T)]
    grad = None
    if grad_seed is not None:
        D = int(np.prod(d))
        grad = np.random.default_rng(grad_seed).normal(
            0.0, 1.0, size=(batch, T * D)).astype(np.float32)
    return Workload(name=name, d=tuple(d), r=tuple(r), n=[tuple(x) for x in n_list],
                    n_rows=[int(x) for x in n_rows_list], batch=int(batch), indices=indices,
                    offsets=offsets, cores=cores, grad_out=grad, lr=lr, train=train)


def near_cubic_factors(N: int) -> tuple:
    n1 = math.ceil(N ** (1.0 / 3.0) - 1e-9)
    n2 = math.ceil(math.sqrt(N / n1) - 1e-9)
    n3 = math.ceil(N / (n1 * n2))
    return (n1, n2, n3)


def table_rows_log_uniform(seed: int, T: int, lo=1e5, hi=4e7) -> list:
    rng = np.random.default_rng(seed)
    return [int(round(math.exp(u))) for u in rng.uniform(math.log(lo), math.log(hi), size=T)]


CONFIG_NAMES = {
    1: "tt3_n1e6_d16_r8_b1024_uniform_fwd",
    2: "tt3_n1e7_d64_r16_b32768_zipf1.05_fwd",
    3: "tt3x26_d128_r32_b32768_zipf1.1_fwd",
    4: "tt3x26_d128_r64_b32768_zipf1.1_train",
    5: "tt4x8_n1e9_d128_r32_b65536_skew_fwdbwd",
}


SHARD_SEED_STRIDE = 1_000_003


def config_workload(cfg: int, batch: int | None = None, with_grad: bool | None = None,
                    tables: int | None = None, shard: int = 0) -> Workload:
    """One of the five benchmark workloads; ``batch``/``tables`` shrink it.

    ``shard`` > 0 draws another batch of the same workload (data-parallel ranks): the cores,
    the tables and the popularity of their rows (the rank-to-row bijection) are shared; the
    bag sizes, the drawn indices and the upstream gradient come from shifted seeds.  Shard 0
    is the workload itself."""
    s = BASE_SEED
    build = build_workload
    if shard:
        def build(name, d, r, n_list, n_rows_list, B, pooling, law, index_seeds, core_seeds,
                  grad_seed=None, **kw):
            return build_workload(name, d, r, n_list, n_rows_list, B, pooling, law,
                                  [x + shard * SHARD_SEED_STRIDE for x in index_seeds], core_seeds,
                                  grad_seed=None if grad_seed is None else grad_seed + shard * SHARD_SEED_STRIDE,
                                  perm_seeds=list(index_seeds), **kw)
    if cfg == 1:
        B = batch or 1024
        w = build(CONFIG_NAMES[1], (2, 2, 4), (1, 8, 8, 1), [(100, 100, 100)], [1_000_000],
                           B, {"kind": "fixed", "size": 1}, {"kind": "uniform"},
                           [s + 1000], [s + 1500], grad_seed=(s + 1777) if with_grad else None)
    elif cfg == 2:
        B = batch or 32768
        w = build(CONFIG_NAMES[2], (4, 4, 4), (1, 16, 16, 1), [(200, 200, 250)],
                           [10_000_000], B, {"kind": "poisson_plus1", "mean": 8},
                           {"kind": "zipf", "alpha": 1.05}, [s + 2000], [s + 2500],
                           grad_seed=(s + 2777) if with_grad else None)
    elif cfg in (3, 4):
        B = batch or 32768
        T = tables or 26
        rows = table_rows_log_uniform(s + 3999, 26)[:T]
        n_list = [near_cubic_factors(N) for N in rows]
        r = (1, 32, 32, 1) if cfg == 3 else (1, 64, 64, 1)
        train = cfg == 4
        if with_grad is None:
            with_grad = train
        w = build(CONFIG_NAMES[cfg], (4, 4, 8), r, n_list, rows, B,
                           {"kind": "poisson_plus1", "mean": 20}, {"kind": "zipf", "alpha": 1.1},
                           [s + 3000 + t for t in range(T)],
                           [s + 1000 * cfg + 500 + t for t in range(T)],
                           grad_seed=(s + 1000 * cfg + 777) if with_grad else None,
                           train=train, lr=0.01)
    elif cfg == 5:
        B = batch or 65536
        T = tables or 8
        if with_grad is None:
            with_grad = True
        w = build(CONFIG_NAMES[5], (2, 4, 4, 4), (1, 32, 32, 32, 1),
                           [(178, 178, 178, 178)] * T, [1_000_000_000] * T, B,
                           {"kind": "uniform", "lo": 1, "hi": 64},
                           {"kind": "mix", "alpha": 1.4, "p_zipf": 0.9},
                           [s + 5000 + t for t in range(T)], [s + 5500 + t for t in range(T)],
                           grad_seed=(s + 5777) if with_grad else None, train=False)
    else:
        raise ValueError(f"no workload {cfg}")
    if with_grad and w.grad_out is None:
        D = w.dim
        w.grad_out = np.random.default_rng(s + 1000 * cfg + 777 + shard * SHARD_SEED_STRIDE).normal(
            0.0, 1.0, size=(w.batch, w.num_tables * D)).astype(np.float32)
    w.meta["config"] = cfg
    w.meta["shard"] = shard
    return w


def random_workload(seed: int, d, r, n_list, n_rows_list=None, batch=8, pooling=None,
                    law=None, with_grad=True, core_std=0.5) -> Workload:
    """Small workloads for tests: arbitrary shapes, uniform indices by default."""
    T = len(n_list)
    if n_rows_list is None:
        n_rows_list = [int(np.prod(x)) for x in n_list]
    pooling = pooling or {"kind": "uniform", "lo": 0, "hi": 5}
    law = law or {"kind": "uniform"}
    return build_workload(f"random{seed}", tuple(d), tuple(r), [tuple(x) for x in n_list],
                          n_rows_list, batch, pooling, law,
                          [seed * 7919 + t for t in range(T)],
                          [seed * 7919 + 104729 + t for t in range(T)],
                          grad_seed=(seed * 7919 + 1299709) if with_grad else None,
                          core_std=core_std)


def sub_batch(w: Workload, bags: np.ndarray) -> Workload:
    """The same tables restricted to the samples ``bags`` (rows of the output)."""
    bags = np.asarray(bags, dtype=np.int64)
    T, B = w.num_tables, w.batch
    parts, sizes = [], []
    for t in range(T):
        for b in bags:
            lo, hi = w.offsets[t * B + b], w.offsets[t * B + b + 1]
            parts.append(w.indices[lo:hi])
            sizes.append(hi - lo)
    offsets = np.zeros(T * bags.size + 1, dtype=np.int64)
    np.cumsum(np.asarray(sizes, dtype=np.int64), out=offsets[1:])
    idx = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    grad = None if w.grad_out is None else w.grad_out[bags]
    return Workload(name=w.name + "_sub", d=w.d, r=w.r, n=w.n, n_rows=w.n_rows,
                    batch=int(bags.size), indices=idx.astype(np.int64), offsets=offsets,
                    cores=w.cores, grad_out=grad, lr=w.lr, train=w.train, meta=dict(w.meta))
