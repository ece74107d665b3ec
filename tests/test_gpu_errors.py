"""Error behaviour on the device: bad inputs are reported at tt_emb_sync, the
handle stays usable afterwards, and out-of-order calls fail on the host.
No test here faults the GPU: the kernels check every index and offset and
record the first error in the handle's status block."""
import numpy as np
import pytest
import torch

import oracle
from tensor_train_compressed_mixed_b200 import TTEmbeddingBag, abi, from_workload
from tests.parity import FP32_TOL, output_err
from workloads import random_workload

pytestmark = pytest.mark.gpu


def _emb():
    w = random_workload(91, (2, 2, 2), (1, 3, 3, 1), [(4, 4, 4), (3, 3, 3)], [64, 20], batch=6,
                        pooling={"kind": "uniform", "lo": 1, "hi": 4})
    emb, cores, idx, off = from_workload(w, with_grads=True)
    return w, emb, idx, off


def test_index_out_of_range_is_reported_and_cleared():
    w, emb, idx, off = _emb()
    bad = idx.clone()
    bad[-1] = 20            # table 1 has 20 valid rows
    emb.forward(bad, off, w.batch)
    with pytest.raises(abi.TTEmbError) as e:
        emb.sync()
    assert e.value.code == abi.TT_ERR_INDEX_RANGE
    neg = idx.clone()
    neg[0] = -1
    emb.forward(neg, off, w.batch)
    with pytest.raises(abi.TTEmbError):
        emb.sync()
    out = emb.forward(idx, off, w.batch)
    emb.sync()
    assert output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim) <= FP32_TOL


@pytest.mark.parametrize("mutate", ["decreasing", "first", "last", "beyond"])
def test_bad_offsets_are_reported(mutate):
    w, emb, idx, off = _emb()
    o = off.clone()
    if mutate == "decreasing":
        o[3], o[4] = o[4].item(), o[3].item() - 1
    elif mutate == "first":
        o[0] = 1
    elif mutate == "last":
        o[-1] = o[-1] - 1
    else:
        o[5] = idx.numel() + 100
    emb.forward(idx, o, w.batch)
    with pytest.raises(abi.TTEmbError) as e:
        emb.sync()
    assert e.value.code == abi.TT_ERR_OFFSETS
    emb.forward(idx, off, w.batch)
    emb.sync()


def test_out_of_order_and_capacity_errors_on_host():
    w = random_workload(92, (2, 2), (1, 3, 1), [(4, 4)], batch=4)
    emb = TTEmbeddingBag(w.n, w.n_rows, w.d, w.r)
    idx = torch.from_numpy(w.indices).cuda()
    off = torch.from_numpy(w.offsets).cuda()
    out = torch.empty(w.batch, w.dim, device="cuda")
    with pytest.raises(abi.TTEmbError) as e:      # no cores
        abi.tt_emb_forward(emb.handle, idx, off, w.batch, out)
    assert e.value.code == abi.TT_ERR_STATE
    emb.set_cores([[torch.from_numpy(c).cuda() for c in w.cores[0]]], with_grads=True)
    with pytest.raises(abi.TTEmbError) as e:      # no workspace
        abi.tt_emb_forward(emb.handle, idx, off, w.batch, out)
    assert e.value.code == abi.TT_ERR_WORKSPACE
    emb.reserve(idx.numel(), w.batch)
    with pytest.raises(abi.TTEmbError) as e:      # backward before any forward
        abi.tt_emb_backward(emb.handle, out)
    assert e.value.code == abi.TT_ERR_STATE
    big = torch.zeros(idx.numel() + 10, dtype=torch.int64, device="cuda")
    with pytest.raises(abi.TTEmbError) as e:      # more lookups than reserved
        abi.tt_emb_forward(emb.handle, big, off, w.batch, out)
    assert e.value.code == abi.TT_ERR_WORKSPACE
    with pytest.raises(abi.TTEmbError) as e:      # workspace below the asked size
        ws = torch.empty(16, dtype=torch.uint8, device="cuda")
        abi.tt_emb_set_workspace(emb.handle, ws, idx.numel(), w.batch)
    assert e.value.code == abi.TT_ERR_WORKSPACE
    emb.forward(idx, off, w.batch, out)
    emb.sync()
    assert output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim) <= FP32_TOL


# ---------------------------------------------------------------------------
# Bounded device waits that run out (failure detection without a GPU fault):
# a test hook arms one injected failure; the kernel's wait gives up after its
# iteration limit, records TT_ERR_TIMEOUT and returns, the code surfaces at
# tt_emb_sync, and the next call on the same handle is correct again.
# ---------------------------------------------------------------------------
def _fast_handle(precision=None, cfg=4, batch=64, tables=3):
    from workloads import config_workload
    w = config_workload(cfg, batch=batch, tables=tables, with_grad=True)
    o = abi.tt_emb_default_options()
    if precision is not None:
        o.precision = precision
    emb, cores, idx, off = from_workload(w, options=o, with_grads=True)
    return w, emb, idx, off


def test_pooling_wait_timeout_is_reported_and_handle_recovers():
    w, emb, idx, off = _fast_handle()
    want = oracle.workload_forward(w)
    abi.tt_emb_debug_inject(emb.handle, abi.TT_INJECT_POOL_WAIT, 2000)
    emb.forward(idx, off, w.batch)
    with pytest.raises(abi.TTEmbError) as e:
        emb.sync()
    assert e.value.code == abi.TT_ERR_TIMEOUT
    assert abi.tt_emb_last_error(emb.handle) == abi.TT_ERR_TIMEOUT
    assert abi.tt_emb_last_error(emb.handle) == abi.TT_OK      # read once, then cleared
    out = emb.forward(idx, off, w.batch)                       # the hook was consumed
    emb.sync()
    assert output_err(out.cpu().numpy(), want, w.dim) <= FP32_TOL


@pytest.mark.parametrize("stage", ["fwd", "bwd"])
def test_tensor_core_wait_timeout_exit_path(stage):
    w, emb, idx, off = _fast_handle(abi.TT_PREC_FP32_SPLIT_TC)
    g = torch.from_numpy(w.grad_out).cuda()
    what = abi.TT_INJECT_MMA_WAIT_FWD if stage == "fwd" else abi.TT_INJECT_MMA_WAIT_BWD
    abi.tt_emb_debug_inject(emb.handle, what, 0)
    emb.forward(idx, off, w.batch)
    emb.backward(g)
    with pytest.raises(abi.TTEmbError) as e:
        emb.sync()
    assert e.value.code == abi.TT_ERR_TIMEOUT
    # tensor memory was freed and the handle works: a full step matches the oracle
    out = emb.forward(idx, off, w.batch)
    emb.backward(g)
    emb.sync()
    assert output_err(out.cpu().numpy(), oracle.workload_forward(w), w.dim) <= FP32_TOL
    from tests.parity import core_grad_err
    want = oracle.workload_backward(w)
    for t in range(w.num_tables):
        for j in range(3):
            got = emb.grads[t * 3 + j].cpu().numpy()
            assert core_grad_err(got, want[t][j]) <= FP32_TOL, (t, j)


def test_injection_needs_a_wait_of_that_kind():
    w = random_workload(93, (2, 2), (1, 3, 1), [(4, 4)], batch=4)
    emb, cores, idx, off = from_workload(w, with_grads=True)    # generic kernels: no such waits
    for what in (abi.TT_INJECT_POOL_WAIT, abi.TT_INJECT_MMA_WAIT_FWD, abi.TT_INJECT_MMA_WAIT_BWD):
        with pytest.raises(abi.TTEmbError) as e:
            abi.tt_emb_debug_inject(emb.handle, what, 0)
        assert e.value.code == abi.TT_ERR_UNSUPPORTED
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_debug_inject(emb.handle, 99, 0)
    assert e.value.code == abi.TT_ERR_ARG
    abi.tt_emb_debug_inject(emb.handle, abi.TT_INJECT_NONE, 0)
    assert abi.tt_emb_last_error(emb.handle) == abi.TT_ERR_ARG


def test_last_error_records_host_failures():
    w = random_workload(94, (2, 2), (1, 3, 1), [(4, 4)], batch=4)
    emb = TTEmbeddingBag(w.n, w.n_rows, w.d, w.r)
    assert abi.tt_emb_last_error(emb.handle) == abi.TT_OK
    idx = torch.from_numpy(w.indices).cuda()
    off = torch.from_numpy(w.offsets).cuda()
    out = torch.empty(w.batch, w.dim, device="cuda")
    with pytest.raises(abi.TTEmbError):
        abi.tt_emb_forward(emb.handle, idx, off, w.batch, out)   # no cores
    assert abi.tt_emb_last_error(emb.handle) == abi.TT_ERR_STATE
    assert abi.tt_emb_last_error(emb.handle) == abi.TT_OK
