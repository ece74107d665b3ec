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
