"""Helpers of the parity tests: the error metric and CUDA-path runners.

Error metric.  The pages state only "max relative error" bounds: 1e-4 with
fp32 accumulation and 2e-2 where a bf16 tensor-core step is used.  The bf16
bound is only meaningful normwise (bf16's unit roundoff is 3.9e-3, so any
elementwise relative error is unbounded where a value cancels to ~0), and
the fp32 bound is read the same way: for each group of values y (one bag's
pooled row of D values, or one digit slice G_j[:, i_j] of a core gradient)
and the result x,
    err = max_e |x_e - y_e| / max_e |y_e|,
and the reported error is the largest over groups.  A group whose reference
is all zeros (an empty bag, an untouched slice) must come out exactly zero.
"""
from __future__ import annotations

import numpy as np

FP32_TOL = 1e-4


def grouped_rel_err(got, want, axis_groups):
    """Max relative error with one floor per group; axis_groups: axes that span a group."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if want.size == 0:
        return 0.0
    scale = np.max(np.abs(want), axis=axis_groups, keepdims=True)
    diff = np.max(np.abs(got - want), axis=axis_groups, keepdims=True)
    zero = scale == 0
    if np.any(zero & (diff != 0)):
        return float("inf")
    return float(np.max(np.where(zero, 0.0, diff / np.where(zero, 1.0, scale))))


def output_err(got, want, D):
    """Per bag row: out is [B, T*D]; each (b, t) block of D values is one group."""
    B = want.shape[0]
    return grouped_rel_err(np.asarray(got).reshape(B, -1, D), np.asarray(want).reshape(B, -1, D),
                           (2,))


def core_grad_err(got, want):
    """Per digit slice: a core is [r0, n, d, r1]; G[:, i] is one group."""
    return grouped_rel_err(got, want, (0, 2, 3))


def gpu_forward(w, options=None, device="cuda", with_grads=None):
    import torch
    from tensor_train_compressed_mixed_b200 import from_workload
    emb, cores, idx, off = from_workload(w, device=device, options=options, with_grads=with_grads)
    out = emb.forward(idx, off, w.batch)
    emb.sync()
    torch.cuda.synchronize()
    return emb, cores, out


def gpu_train_step(w, options=None, device="cuda", lr=None):
    """forward + backward (+ SGD when lr is given); returns numpy results."""
    import torch
    emb, cores, out = gpu_forward(w, options, device, with_grads=True)
    g = torch.from_numpy(w.grad_out).to(device)
    emb.backward(g)
    emb.sync()
    grads = [[x.cpu().numpy() for x in emb.grads[t * emb.k:(t + 1) * emb.k]] for t in range(emb.T)]
    new = None
    if lr is not None:
        emb.sgd_update(lr)
        emb.sync()
        new = [[c.cpu().numpy() for c in tab] for tab in cores]
    return emb, out.cpu().numpy(), grads, new
