"""bench.py's multi-process plumbing, run with two gloo ranks on the CPU.

Each rank goes through the same calls a data-parallel training step of ``bench.py --gpus 2``
makes around the library: the process-group join (``dist_init``), the exchange of the flat
core-gradient buffer (``dp.allreduce_grads``), the max-over-ranks of the device time
(``max_over_ranks``) and the teardown (``dist_teardown``), which must destroy the group
exactly once.  A rank that raises makes the spawn fail, so the test also proves every rank
exits cleanly.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tensor_train_compressed_mixed_b200.dp import grad_layout

SHAPES = [(1, 7, 4, 64), (64, 5, 4, 64), (64, 9, 8, 1)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _Holder:
    """Stands in for a TTEmbeddingBag created with flat_grads=True."""

    def __init__(self, flat):
        self.grad_flat = flat


def _rank_main(rank, world, port, out_dir):
    import bench
    from tensor_train_compressed_mixed_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_init(world)
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    offs, total = grad_layout(SHAPES)
    rng = np.random.default_rng(100 + rank)
    flat = torch.from_numpy(rng.standard_normal(total).astype(np.float32))
    np.save(os.path.join(out_dir, f"in{rank}.npy"), flat.numpy())
    holder = _Holder(flat)
    dp.allreduce_grads(holder)
    m = bench.max_over_ranks(w, 10.0 + rank)
    bench.barrier(w)
    np.save(os.path.join(out_dir, f"out{rank}.npy"), holder.grad_flat.numpy())
    np.save(os.path.join(out_dir, f"max{rank}.npy"), np.array([m]))
    bench.dist_teardown(w)
    assert not dist.is_initialized()
    bench.dist_teardown(w)   # a second call is a no-op, not an error


def test_two_rank_gradient_exchange_and_single_teardown(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    ins = [np.load(tmp_path / f"in{r}.npy") for r in range(world)]
    want = ins[0].astype(np.float64) + ins[1]
    for r in range(world):
        got = np.load(tmp_path / f"out{r}.npy")
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-6)
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == 10.0 + world - 1


def test_single_process_needs_no_group():
    import bench
    os.environ.pop("WORLD_SIZE", None)
    w, r, local = bench.dist_init(1)
    assert (w, r, local) == (1, 0, 0)
    assert bench.max_over_ranks(1, 3.5) == 3.5
    bench.dist_teardown(1)
