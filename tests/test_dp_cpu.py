"""Data-parallel decomposition, checked on the CPU with two gloo ranks.

Each rank takes its own batch of the same workload (workloads.config_workload(...,
shard=rank)), computes the core gradients of its batch with the oracle, and the ranks sum
them with an all-reduce, as the GPU ranks do with NCCL over the flat gradient buffer.  The
sum must equal the oracle's gradient of the union of the two batches (the loss is a sum over
bags and the gradients are linear in the upstream gradient).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from tensor_train_compressed_mixed_b200.dp import ALIGN_FLOATS, grad_layout
from workloads import config_workload
from workloads.gen import Workload


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _union(ws):
    """Bags of several batches of one workload side by side (same tables and cores)."""
    T = ws[0].num_tables
    idx, sizes = [], []
    for t in range(T):
        for w in ws:
            lo, hi = w.offsets[t * w.batch], w.offsets[(t + 1) * w.batch]
            idx.append(w.indices[lo:hi])
            sizes.append(np.diff(w.offsets[t * w.batch:(t + 1) * w.batch + 1]))
    offsets = np.zeros(sum(len(x) for x in sizes) + 1, dtype=np.int64)
    np.cumsum(np.concatenate(sizes), out=offsets[1:])
    w0 = ws[0]
    return Workload(name="union", d=w0.d, r=w0.r, n=w0.n, n_rows=w0.n_rows, batch=sum(w.batch for w in ws),
                    indices=np.concatenate(idx), offsets=offsets, cores=w0.cores,
                    grad_out=np.vstack([w.grad_out for w in ws]), lr=w0.lr, train=w0.train)


def _flat(grads):
    return np.concatenate([g.reshape(-1) for tab in grads for g in tab])


class _FlatGrads:
    """Stands in for a TTEmbeddingBag with flat_grads=True (only grad_flat is used)."""

    def __init__(self, flat):
        self.grad_flat = flat


def _rank_main(rank, world, port, out_path):
    from tensor_train_compressed_mixed_b200.dp import allreduce_grads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = config_workload(4, batch=6, tables=2, with_grad=True, shard=rank)
        holder = _FlatGrads(torch.from_numpy(_flat(oracle.workload_backward(w, threads=1))))
        allreduce_grads(holder)   # the exchange bench.py runs between backward and SGD
        if rank == 0:
            np.save(out_path, holder.grad_flat.numpy())
    finally:
        dist.destroy_process_group()


def test_shards_differ_but_share_cores():
    a = config_workload(4, batch=6, tables=2, with_grad=True, shard=0)
    b = config_workload(4, batch=6, tables=2, with_grad=True, shard=1)
    assert not np.array_equal(a.indices[:20], b.indices[:20])
    assert not np.array_equal(a.grad_out, b.grad_out)
    for t in range(2):
        for j in range(3):
            assert np.array_equal(a.cores[t][j], b.cores[t][j])
    ref = config_workload(4, batch=6, tables=2, with_grad=True)
    assert np.array_equal(ref.indices, a.indices) and np.array_equal(ref.grad_out, a.grad_out)


def test_allreduced_shard_gradients_equal_the_global_batch_gradient(tmp_path):
    world, port = 2, _free_port()
    out = str(tmp_path / "sum.npy")
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    got = np.load(out)
    ws = [config_workload(4, batch=6, tables=2, with_grad=True, shard=r) for r in range(world)]
    want = _flat(oracle.workload_backward(_union(ws), threads=1))
    scale = np.max(np.abs(want))
    assert np.max(np.abs(got - want)) <= 1e-12 * max(scale, 1.0)


def test_flat_gradient_layout_is_aligned_and_disjoint():
    shapes = [(1, 7, 4, 64), (64, 7, 4, 64), (64, 9, 8, 1), (1, 3, 3, 5)]
    offs, total = grad_layout(shapes)
    sizes = [int(np.prod(s)) for s in shapes]
    assert all(o % ALIGN_FLOATS == 0 for o in offs)
    for q in range(len(shapes) - 1):
        assert offs[q] + sizes[q] <= offs[q + 1]
    assert offs[-1] + sizes[-1] <= total < offs[-1] + sizes[-1] + ALIGN_FLOATS
