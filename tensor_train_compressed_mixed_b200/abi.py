"""ctypes binding of libttemb (include/tt_emb.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: tensors are checked for device, dtype and layout,
their pointers and the current CUDA stream are passed through, and a non-OK
status becomes a ``TTEmbError``.  There is no CPU path: without the built
library (``python -m tensor_train_compressed_mixed_b200.build``) importing
the functions raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
# TTEMB_LIB names another build of the same library (e.g. a variant compiled for a comparison)
LIB_PATH = os.environ.get("TTEMB_LIB") or os.path.join(PKG, "libttemb.so")

TT_OK, TT_ERR_ARG, TT_ERR_SHAPE, TT_ERR_INDEX_RANGE, TT_ERR_OFFSETS = 0, 1, 2, 3, 4
TT_ERR_WORKSPACE, TT_ERR_STATE, TT_ERR_CUDA, TT_ERR_TIMEOUT, TT_ERR_UNSUPPORTED = 5, 6, 7, 8, 9
TT_SCHED_STATIC, TT_SCHED_STEAL, TT_SCHED_STEAL_L2 = 0, 1, 2
TT_GROUP_PREFIX, TT_GROUP_UNIQUE_ONLY = 0, 1
TT_PREC_FP32, TT_PREC_BF16_TC, TT_PREC_FP32_SPLIT_TC = 0, 1, 2
TT_INJECT_NONE, TT_INJECT_POOL_WAIT, TT_INJECT_MMA_WAIT_FWD, TT_INJECT_MMA_WAIT_BWD = 0, 1, 2, 3
MAX_TABLES, MAX_CORES = 64, 4


class TTEmbError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (status {code})")


class Options(ctypes.Structure):
    _fields_ = [("sched", ctypes.c_int32), ("grouping", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("grid", ctypes.c_int32),
                ("force_generic", ctypes.c_int32), ("precision", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 10)]


class SegView(ctypes.Structure):
    _fields_ = [("num_lookups", ctypes.c_int64), ("num_unique", ctypes.c_int64),
                ("num_groups", ctypes.c_int64), ("key_bits", ctypes.c_int32),
                ("key_bytes", ctypes.c_int32), ("sorted_keys", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("uniq_keys", ctypes.c_void_p),
                ("uniq_start", ctypes.c_void_p), ("grp_start", ctypes.c_void_p),
                ("bag_sorted", ctypes.c_void_p)]


_LIB = None

_SIGS = {
    "tt_emb_abi_version": ([], ctypes.c_int),
    "tt_emb_default_options": ([ctypes.POINTER(Options)], None),
    "tt_emb_error_string": ([ctypes.c_int], ctypes.c_char_p),
    "tt_emb_create": ([ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                       ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Options),
                       ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
    "tt_emb_set_cores": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "tt_emb_workspace_size": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                               ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "tt_emb_set_workspace": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64,
                              ctypes.c_int64], ctypes.c_int),
    "tt_emb_forward": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "tt_emb_backward": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "tt_emb_sgd_update": ([ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p], ctypes.c_int),
    "tt_emb_backward_sgd": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p], ctypes.c_int),
    "tt_emb_get_segmentation": ([ctypes.c_void_p, ctypes.POINTER(SegView)], ctypes.c_int),
    "tt_emb_copy_segmentation": ([ctypes.c_void_p] + [ctypes.c_void_p] * 6, ctypes.c_int),
    "tt_emb_sync": ([ctypes.c_void_p], ctypes.c_int),
    "tt_emb_enable_timing": ([ctypes.c_void_p, ctypes.c_int], ctypes.c_int),
    "tt_emb_phase_times": ([ctypes.c_void_p, ctypes.POINTER(ctypes.c_double),
                            ctypes.POINTER(ctypes.c_int64)], ctypes.c_int),
    "tt_emb_forward_noalloc": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "tt_emb_last_error": ([ctypes.c_void_p], ctypes.c_int),
    "tt_emb_set_probe": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32], ctypes.c_int),
    "tt_emb_debug_inject": ([ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32], ctypes.c_int),
    "tt_emb_destroy": ([ctypes.c_void_p], None),
}

NOALLOC_MAX_LOOKUPS = 262144

PHASES = ("fwd_keys", "fwd_sort", "fwd_segment", "fwd_fused", "bwd_fused", "bwd_reduce", "sgd",
          "bwd_rowsum")


def lib() -> ctypes.CDLL:
    """The loaded libttemb.so; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m tensor_train_compressed_mixed_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = h
    return _LIB


def error_string(code: int) -> str:
    return lib().tt_emb_error_string(int(code)).decode()


def _check(rc: int, where: str):
    if rc != TT_OK:
        raise TTEmbError(rc, where)


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_ptr(t, dtype, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def tt_emb_abi_version() -> int:
    return lib().tt_emb_abi_version()


def tt_emb_default_options() -> Options:
    o = Options()
    lib().tt_emb_default_options(ctypes.byref(o))
    return o


def tt_emb_create(n_factors, n_rows, d_factors, ranks, options: Options | None = None):
    """n_factors: [T][k] ints; n_rows: [T]; d_factors: [k]; ranks: [k+1]. Returns a handle."""
    n = np.ascontiguousarray(np.asarray(n_factors, dtype=np.int64))
    if n.ndim != 2:
        raise ValueError("n_factors must be [T][k]")
    rows = np.ascontiguousarray(np.asarray(n_rows, dtype=np.int64).reshape(-1))
    d = np.ascontiguousarray(np.asarray(d_factors, dtype=np.int32).reshape(-1))
    r = np.ascontiguousarray(np.asarray(ranks, dtype=np.int32).reshape(-1))
    T, k = n.shape
    if rows.size != T or d.size != k or r.size != k + 1:
        raise ValueError("inconsistent table shapes")
    h = ctypes.c_void_p()
    opt = ctypes.byref(options) if options is not None else None
    _check(lib().tt_emb_create(T, k, n.ctypes.data, rows.ctypes.data, d.ctypes.data, r.ctypes.data,
                               opt, ctypes.byref(h)), "tt_emb_create")
    return h


def tt_emb_set_cores(h, cores, core_grads=None):
    """cores / core_grads: flat lists of T*k float32 CUDA tensors, table-major."""
    import torch
    ptrs = (ctypes.c_void_p * len(cores))(*[_dev_ptr(c, torch.float32, "core").value for c in cores])
    gptrs = None
    if core_grads is not None:
        gptrs = (ctypes.c_void_p * len(core_grads))(
            *[_dev_ptr(g, torch.float32, "core_grad").value for g in core_grads])
    _check(lib().tt_emb_set_cores(h, ptrs, gptrs), "tt_emb_set_cores")


def tt_emb_workspace_size(h, max_lookups: int, batch: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().tt_emb_workspace_size(h, int(max_lookups), int(batch), ctypes.byref(out)),
           "tt_emb_workspace_size")
    return int(out.value)


def tt_emb_set_workspace(h, workspace, max_lookups: int, batch: int):
    import torch
    ptr = _dev_ptr(workspace, torch.uint8, "workspace")
    _check(lib().tt_emb_set_workspace(h, ptr, workspace.numel(), int(max_lookups), int(batch)),
           "tt_emb_set_workspace")


def tt_emb_forward(h, indices, offsets, batch: int, out, stream=None):
    import torch
    _check(lib().tt_emb_forward(h, _dev_ptr(indices, torch.int64, "indices"),
                                _dev_ptr(offsets, torch.int64, "offsets"), indices.numel(),
                                int(batch), _dev_ptr(out, torch.float32, "out"), _stream(stream)),
           "tt_emb_forward")


def tt_emb_backward(h, grad_out, stream=None):
    import torch
    _check(lib().tt_emb_backward(h, _dev_ptr(grad_out, torch.float32, "grad_out"), _stream(stream)),
           "tt_emb_backward")


def tt_emb_sgd_update(h, lr: float, stream=None):
    _check(lib().tt_emb_sgd_update(h, float(lr), _stream(stream)), "tt_emb_sgd_update")


def tt_emb_backward_sgd(h, grad_out, lr: float, stream=None):
    import torch
    _check(lib().tt_emb_backward_sgd(h, _dev_ptr(grad_out, torch.float32, "grad_out"), float(lr),
                                     _stream(stream)), "tt_emb_backward_sgd")


def tt_emb_sync(h):
    _check(lib().tt_emb_sync(h), "tt_emb_sync")


def tt_emb_get_segmentation(h) -> SegView:
    v = SegView()
    _check(lib().tt_emb_get_segmentation(h, ctypes.byref(v)), "tt_emb_get_segmentation")
    return v


def tt_emb_copy_segmentation(h) -> dict:
    """The last forward's segmentation, copied to host numpy arrays."""
    v = tt_emb_get_segmentation(h)
    L, U, G = v.num_lookups, v.num_unique, v.num_groups
    kt = np.uint64 if v.key_bytes == 8 else np.uint32
    out = {
        "sorted_keys": np.zeros(L, kt), "perm": np.zeros(L, np.int32),
        "uniq_keys": np.zeros(U, kt), "uniq_start": np.zeros(U + 1, np.int32),
        "grp_start": np.zeros(G + 1, np.int32), "bag_sorted": np.zeros(L, np.int32),
    }
    _check(lib().tt_emb_copy_segmentation(
        h, out["sorted_keys"].ctypes.data, out["perm"].ctypes.data, out["uniq_keys"].ctypes.data,
        out["uniq_start"].ctypes.data, out["grp_start"].ctypes.data, out["bag_sorted"].ctypes.data),
        "tt_emb_copy_segmentation")
    if L == 0:
        out["uniq_start"][:] = 0
        out["grp_start"][:] = 0
    out.update(num_lookups=L, num_unique=U, num_groups=G, key_bits=v.key_bits)
    return out


def tt_emb_forward_noalloc(h, indices, offsets, batch: int, out, stream=None):
    """Forward pass using the library's fixed device scratch instead of a workspace."""
    import torch
    _check(lib().tt_emb_forward_noalloc(h, _dev_ptr(indices, torch.int64, "indices"),
                                        _dev_ptr(offsets, torch.int64, "offsets"), indices.numel(),
                                        int(batch), _dev_ptr(out, torch.float32, "out"),
                                        _stream(stream)),
           "tt_emb_forward_noalloc")


def tt_emb_enable_timing(h, enable: bool = True):
    _check(lib().tt_emb_enable_timing(h, 1 if enable else 0), "tt_emb_enable_timing")


def tt_emb_phase_times(h):
    """(per-phase milliseconds as a dict, kernels launched) since timing was enabled."""
    ms = (ctypes.c_double * len(PHASES))()
    n = ctypes.c_int64()
    _check(lib().tt_emb_phase_times(h, ms, ctypes.byref(n)), "tt_emb_phase_times")
    return dict(zip(PHASES, list(ms))), int(n.value)


def tt_emb_last_error(h) -> int:
    """The most recent failure recorded on the handle (a status code), then cleared."""
    return int(lib().tt_emb_last_error(h))


def tt_emb_set_probe(h, records, max_blocks: int):
    """Balance probe: records is a CUDA int64 tensor of 2 * max_blocks * 4 entries, or None."""
    import torch
    ptr = ctypes.c_void_p(0) if records is None else _dev_ptr(records, torch.int64, "records")
    _check(lib().tt_emb_set_probe(h, ptr, int(max_blocks) if records is not None else 0), "tt_emb_set_probe")


def tt_emb_debug_inject(h, what: int, spin_limit: int = 0):
    """Test hook: arms one injected failure of a bounded device wait (TT_INJECT_*)."""
    _check(lib().tt_emb_debug_inject(h, int(what), int(spin_limit)), "tt_emb_debug_inject")


def tt_emb_destroy(h):
    if h is not None and h.value:
        lib().tt_emb_destroy(h)
