"""TTEmbeddingBag: a handle of libttemb plus the torch tensors it borrows.

PyTorch supplies device memory and the current stream; every step of the
gather, its backward and the SGD step runs in the library's CUDA kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import abi


class TTEmbeddingBag:
    """T TT-compressed tables sharing (d, r), pooled by sum.

    n_factors: per table (n_1..n_k); n_rows: valid rows per table;
    d: (d_1..d_k); r: (r_0..r_k) with r_0 = r_k = 1.
    """

    def __init__(self, n_factors, n_rows, d, r, options: abi.Options | None = None,
                 device="cuda"):
        self.device = torch.device(device)
        with torch.cuda.device(self.device):
            self.handle = abi.tt_emb_create(n_factors, n_rows, d, r, options)
        self.n = [tuple(int(x) for x in row) for row in n_factors]
        self.n_rows = [int(x) for x in n_rows]
        self.d, self.r = tuple(int(x) for x in d), tuple(int(x) for x in r)
        self.T, self.k = len(self.n), len(self.d)
        self.D = int(np.prod(self.d))
        self.cores = None
        self.grads = None
        self.grad_flat = None
        self._ws = None
        self._ws_dims = (0, 0)

    def core_shape(self, t: int, j: int) -> tuple:
        return (self.r[j], self.n[t][j], self.d[j], self.r[j + 1])

    def set_cores(self, cores, with_grads: bool = True, flat_grads: bool = False):
        """cores: [T][k] float32 CUDA tensors (borrowed); allocates gradient buffers.

        flat_grads: the gradients are views of one buffer (``self.grad_flat``), so that a
        data-parallel exchange is a single collective (dp.allreduce_grads)."""
        flat = [cores[t][j] for t in range(self.T) for j in range(self.k)]
        for q, c in enumerate(flat):
            if tuple(c.shape) != self.core_shape(q // self.k, q % self.k):
                raise ValueError(f"core {q} has shape {tuple(c.shape)}")
        self.cores = flat
        self.grad_flat = None
        if with_grads and flat_grads:
            from .dp import grad_layout
            offs, total = grad_layout([tuple(c.shape) for c in flat])
            self.grad_flat = torch.zeros(total, dtype=torch.float32, device=self.device)
            self.grads = [self.grad_flat[o:o + c.numel()].view(c.shape) for o, c in zip(offs, flat)]
        else:
            self.grads = [torch.empty_like(c) for c in flat] if with_grads else None
        abi.tt_emb_set_cores(self.handle, flat, self.grads)

    def reserve(self, max_lookups: int, batch: int):
        """Allocates (or grows) the workspace for batches up to these sizes."""
        L0, B0 = self._ws_dims
        if self._ws is not None and max_lookups <= L0 and batch <= B0:
            return
        L, B = max(max_lookups, L0), max(batch, B0)
        nbytes = abi.tt_emb_workspace_size(self.handle, L, B)
        self._ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        abi.tt_emb_set_workspace(self.handle, self._ws, L, B)
        self._ws_dims = (L, B)

    def forward(self, indices: torch.Tensor, offsets: torch.Tensor, batch: int,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        self.reserve(indices.numel(), batch)
        if out is None:
            out = torch.empty(batch, self.T * self.D, dtype=torch.float32, device=self.device)
        abi.tt_emb_forward(self.handle, indices, offsets, batch, out, stream)
        return out

    def backward(self, grad_out: torch.Tensor, stream=None):
        abi.tt_emb_backward(self.handle, grad_out, stream)
        return self.grads

    def sgd_update(self, lr: float, stream=None):
        abi.tt_emb_sgd_update(self.handle, lr, stream)

    def backward_sgd(self, grad_out: torch.Tensor, lr: float, stream=None):
        """Backward and SGD step fused (the middle cores are updated sparsely in place)."""
        abi.tt_emb_backward_sgd(self.handle, grad_out, lr, stream)

    def sync(self):
        abi.tt_emb_sync(self.handle)

    def segmentation(self) -> dict:
        return abi.tt_emb_copy_segmentation(self.handle)

    def close(self):
        if getattr(self, "handle", None) is not None:
            abi.tt_emb_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def from_workload(w, device="cuda", options=None, with_grads=None, flat_grads=False):
    """A TTEmbeddingBag holding a seeded workload's cores, plus its inputs on the device."""
    emb = TTEmbeddingBag(w.n, w.n_rows, w.d, w.r, options=options, device=device)
    cores = [[torch.from_numpy(c).to(device) for c in tab] for tab in w.cores]
    emb.set_cores(cores, with_grads=w.train if with_grads is None else with_grads, flat_grads=flat_grads)
    idx = torch.from_numpy(w.indices).to(device)
    off = torch.from_numpy(w.offsets).to(device)
    return emb, cores, idx, off
