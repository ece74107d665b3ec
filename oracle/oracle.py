"""fp64 oracle for Tensor-Train embedding gather.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path and never imports it.

What each function follows (FlowTT: Exploiting Computation Flow Reuse in
Irregular Tensor-Train Embedding):

* ``forward`` / ``backward`` / ``row`` -- the C library ``tt_oracle.c``: each
  lookup's slices are contracted on their own, left to right ("C = A.B, then
  E = C.D, followed by pooling", section 3.2), in fp64, then sum-pooled into
  its bag; the backward is the textbook TT gradient (left partial^T x
  upstream x right partial^T) accumulated per lookup.
* ``segmentation`` -- the grouping pipeline of sections 3.3 and 4 ("index
  sorting, unique extraction, mixed-radix conversion, prefix extraction and
  run-length encoding") written with numpy's stable argsort and run starts.
* ``sgd`` -- plain gradient descent G - lr * dG in fp64.

Readings of the pages that these functions fix (the pages give no formulas):
the first digit i_1 is the most significant (the prefix is the "early
mixed-radix digits", section 2.4); row columns flatten (a_1..a_k) row-major;
the prefix of a row is its first k-1 digits, i.e. i // n_k; sort ties keep
input order (stable).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        lib.tto_forward.argtypes = [i32, i32, P, P, P, P, P, P, P, i64, P, i32]
        lib.tto_forward.restype = ctypes.c_int
        lib.tto_backward.argtypes = [i32, i32, P, P, P, P, P, P, P, i64, P, P, i32]
        lib.tto_backward.restype = ctypes.c_int
        lib.tto_row.argtypes = [i32, P, P, P, P, i64, P]
        lib.tto_row.restype = ctypes.c_int
        lib.tto_digits_batch.argtypes = [i32, P, P, i64, P]
        lib.tto_digits_batch.restype = ctypes.c_int
        _LIB = lib
    return _LIB


class OracleError(RuntimeError):
    pass


_ERRORS = {1: "bad argument", 2: "index out of range", 3: "bad offsets", 4: "out of memory"}


def _check(rc: int):
    if rc != 0:
        raise OracleError(f"oracle: {_ERRORS.get(rc, rc)}")


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _prep(d, r, n, n_rows, cores):
    T, k = len(n), len(d)
    n_arr = np.ascontiguousarray(np.asarray(n, dtype=np.int64).reshape(T, k))
    rows = np.ascontiguousarray(np.asarray(n_rows, dtype=np.int64).reshape(T))
    d_arr = np.ascontiguousarray(np.asarray(d, dtype=np.int32))
    r_arr = np.ascontiguousarray(np.asarray(r, dtype=np.int32))
    c64 = [np.ascontiguousarray(np.asarray(c, dtype=np.float64)) for tab in cores for c in tab]
    for t in range(T):
        for j in range(k):
            want = (r[j], n_arr[t, j], d[j], r[j + 1])
            if c64[t * k + j].shape != tuple(int(x) for x in want):
                raise OracleError(f"core ({t},{j}) has shape {c64[t * k + j].shape}, want {want}")
    cptr = (ctypes.c_void_p * (T * k))(*[_ptr(c) for c in c64])
    return T, k, n_arr, rows, d_arr, r_arr, c64, cptr


def forward(d, r, n, n_rows, cores, indices, offsets, batch, threads=None) -> np.ndarray:
    """Pooled rows, fp64 [batch, T*D]; bags are table-major in ``offsets``."""
    T, k, n_arr, rows, d_arr, r_arr, keep, cptr = _prep(d, r, n, n_rows, cores)
    D = int(np.prod(d))
    idx = np.ascontiguousarray(np.asarray(indices, dtype=np.int64))
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    if off.size != T * batch + 1 or off[-1] != idx.size:
        raise OracleError("offsets must have T*B+1 entries ending at len(indices)")
    out = np.zeros((batch, T * D), dtype=np.float64)
    _check(_lib().tto_forward(T, k, _ptr(n_arr), _ptr(rows), _ptr(d_arr), _ptr(r_arr), cptr,
                              _ptr(idx), _ptr(off), batch, _ptr(out), threads or default_threads()))
    return out


def backward(d, r, n, n_rows, cores, indices, offsets, batch, grad_out, threads=None) -> list:
    """dL/dG for L = <grad_out, forward(...)>: per table, a list of fp64 core gradients."""
    T, k, n_arr, rows, d_arr, r_arr, keep, cptr = _prep(d, r, n, n_rows, cores)
    D = int(np.prod(d))
    idx = np.ascontiguousarray(np.asarray(indices, dtype=np.int64))
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    g = np.ascontiguousarray(np.asarray(grad_out, dtype=np.float64).reshape(batch, T * D))
    grads = [np.zeros_like(c) for c in keep]
    gptr = (ctypes.c_void_p * (T * k))(*[_ptr(x) for x in grads])
    _check(_lib().tto_backward(T, k, _ptr(n_arr), _ptr(rows), _ptr(d_arr), _ptr(r_arr), cptr,
                               _ptr(idx), _ptr(off), batch, _ptr(g), gptr,
                               threads or default_threads()))
    return [grads[t * k:(t + 1) * k] for t in range(T)]


def row(d, r, n, cores_of_table, i) -> np.ndarray:
    """Row ``i`` of one table, fp64 [D]."""
    T, k, n_arr, rows, d_arr, r_arr, keep, cptr = _prep(d, r, [n], [int(np.prod(n))],
                                                        [cores_of_table])
    out = np.zeros(int(np.prod(d)), dtype=np.float64)
    _check(_lib().tto_row(k, _ptr(n_arr), _ptr(d_arr), _ptr(r_arr), cptr, int(i), _ptr(out)))
    return out


def digits(n, rows) -> np.ndarray:
    """Mixed-radix digits (i_1 first) of each row, int64 [count, k]."""
    n_arr = np.ascontiguousarray(np.asarray(n, dtype=np.int64))
    rr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    out = np.zeros((rr.size, n_arr.size), dtype=np.int64)
    _check(_lib().tto_digits_batch(n_arr.size, _ptr(n_arr), _ptr(rr), rr.size, _ptr(out)))
    return out


def sgd(cores, grads, lr) -> list:
    """G - lr * dG in fp64, per table and core."""
    return [[np.asarray(c, np.float64) - float(lr) * np.asarray(g, np.float64)
             for c, g in zip(ct, gt)] for ct, gt in zip(cores, grads)]


def segmentation(indices, offsets, batch, n_last) -> dict:
    """Canonical grouping of a batch of lookups (numpy, exact).

    ``n_last[t]`` is n_k of table t.  Returns int64 arrays:
      perm        [L]    input positions in sorted (table, row) order, ties by position
      uniq_table  [U], uniq_row [U]   the distinct (table, row) pairs, sorted
      uniq_start  [U+1]  start of each distinct pair's run in sorted order
      grp_start   [G+1]  start of each prefix group (table, row // n_k) in the unique list
      bag_sorted  [L]    bag id t*B + b of each sorted lookup
    """
    idx = np.asarray(indices, dtype=np.int64)
    off = np.asarray(offsets, dtype=np.int64)
    L = idx.size
    pos = np.arange(L, dtype=np.int64)
    bag = np.searchsorted(off, pos, side="right") - 1
    table = bag // batch
    span = int(idx.max()) + 1 if L else 1
    key = table * span + idx
    perm = np.argsort(key, kind="stable")
    st, si = table[perm], idx[perm]
    if L:
        new_u = np.ones(L, dtype=bool)
        new_u[1:] = (st[1:] != st[:-1]) | (si[1:] != si[:-1])
        ustart = np.flatnonzero(new_u)
    else:
        ustart = np.zeros(0, dtype=np.int64)
    uniq_table, uniq_row = st[ustart], si[ustart]
    nk = np.asarray(n_last, dtype=np.int64)
    prefix = uniq_row // nk[uniq_table] if ustart.size else uniq_row
    U = ustart.size
    if U:
        new_g = np.ones(U, dtype=bool)
        new_g[1:] = (uniq_table[1:] != uniq_table[:-1]) | (prefix[1:] != prefix[:-1])
        gstart = np.flatnonzero(new_g)
    else:
        gstart = np.zeros(0, dtype=np.int64)
    return {
        "perm": perm.astype(np.int64),
        "uniq_table": uniq_table.astype(np.int64),
        "uniq_row": uniq_row.astype(np.int64),
        "uniq_start": np.append(ustart, L).astype(np.int64),
        "grp_start": np.append(gstart, U).astype(np.int64),
        "bag_sorted": bag[perm].astype(np.int64),
    }


def workload_forward(w, threads=None) -> np.ndarray:
    return forward(w.d, w.r, w.n, w.n_rows, w.cores, w.indices, w.offsets, w.batch, threads)


def workload_backward(w, grad_out=None, threads=None) -> list:
    g = w.grad_out if grad_out is None else grad_out
    return backward(w.d, w.r, w.n, w.n_rows, w.cores, w.indices, w.offsets, w.batch, g, threads)


def workload_segmentation(w) -> dict:
    return segmentation(w.indices, w.offsets, w.batch, [n[-1] for n in w.n])
