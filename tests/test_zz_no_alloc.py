"""tt_emb_forward_noalloc: the forward pass for callers that cannot allocate.

Some callers cannot hand the library device memory: hosts whose plugin
interface offers no allocator or workspace, servers that forbid device
allocation after start-up to keep memory and latency fixed, and plain C
callers without PyTorch.  For them the library keeps its forward scratch in a
fixed 16 MiB device array and this entry point allocates nothing.  These tests
call it through the C ABI and check it against tt_emb_forward (the entry point
with a caller workspace), within the parity tolerance, on consecutive calls
whose inputs differ, so stale scratch contents from one call cannot leak into
the next.  They also check that warmed calls leave the device's allocated and
free memory unchanged, that the wide (64-bit) sort keys of eight 1e9-row tables
work, and that a backward after this forward is refused (its grouping is not
kept).
"""
import pytest
import torch

from tensor_train_compressed_mixed_b200 import abi, from_workload
from tests.parity import FP32_TOL, output_err
from workloads import config_workload, sub_batch

pytestmark = pytest.mark.gpu


def _reference(emb, idx, off, batch):
    out = torch.empty(batch, emb.T * emb.D, device="cuda")
    emb.forward(idx, off, batch, out)
    emb.sync()
    return out.cpu().numpy()


def _noalloc(emb, idx, off, batch):
    out = torch.full((batch, emb.T * emb.D), float("nan"), device="cuda")
    abi.tt_emb_forward_noalloc(emb.handle, idx, off, batch, out)
    emb.sync()
    return out.cpu().numpy()


def test_noalloc_forward_matches_forward_on_consecutive_calls():
    w = config_workload(3, batch=1024, tables=4, with_grad=False)   # 32-bit keys
    small = sub_batch(w, torch.arange(0, 1024, 3).numpy())
    emb, cores, idx, off = from_workload(w, with_grads=False)
    assert idx.numel() <= abi.NOALLOC_MAX_LOOKUPS
    s_idx = torch.from_numpy(small.indices).cuda()
    s_off = torch.from_numpy(small.offsets).cuda()
    want_big = _reference(emb, idx, off, w.batch)
    want_small = _reference(emb, s_idx, s_off, small.batch)
    # two calls in a row, the second smaller than the first
    assert output_err(_noalloc(emb, idx, off, w.batch), want_big, w.dim) <= FP32_TOL
    assert output_err(_noalloc(emb, s_idx, s_off, small.batch), want_small, w.dim) <= FP32_TOL


def test_noalloc_forward_with_wide_keys_and_four_cores():
    # eight tables of 1e9 rows: 30 row bits + 3 table bits, so the sort keys take 64 bits
    w = config_workload(5, batch=256, tables=8, with_grad=False)
    emb, cores, idx, off = from_workload(w, with_grads=False)
    want = _reference(emb, idx, off, w.batch)
    assert emb.segmentation()["sorted_keys"].dtype.itemsize == 8
    assert idx.numel() <= abi.NOALLOC_MAX_LOOKUPS
    for _ in range(2):
        assert output_err(_noalloc(emb, idx, off, w.batch), want, w.dim) <= FP32_TOL


def test_noalloc_call_allocates_no_device_memory():
    w = config_workload(3, batch=512, tables=4, with_grad=False)
    emb, cores, idx, off = from_workload(w, with_grads=False)
    out = torch.empty(w.batch, emb.T * emb.D, device="cuda")
    # first call on the device: looks up the scratch (and loads its module); not measured
    abi.tt_emb_forward_noalloc(emb.handle, idx, off, w.batch, out)
    emb.sync()
    torch.cuda.synchronize()
    used0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        abi.tt_emb_forward_noalloc(emb.handle, idx, off, w.batch, out)
    emb.sync()
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == used0
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_backward_after_a_noalloc_forward_is_refused():
    w = config_workload(4, batch=16, tables=2, with_grad=True)
    emb, cores, idx, off = from_workload(w, with_grads=True)
    g = torch.from_numpy(w.grad_out).cuda()
    emb.forward(idx, off, w.batch)
    out = torch.empty(w.batch, emb.T * emb.D, device="cuda")
    abi.tt_emb_forward_noalloc(emb.handle, idx, off, w.batch, out)
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_backward(emb.handle, g)
    assert e.value.code == abi.TT_ERR_STATE
    emb.sync()


def test_noalloc_rejects_batches_above_its_capacity():
    w = config_workload(1, with_grad=False)
    emb, cores, idx, off = from_workload(w, with_grads=False)
    n = abi.NOALLOC_MAX_LOOKUPS + 1
    big_idx = torch.zeros(n, dtype=torch.int64, device="cuda")
    big_off = torch.tensor([0, n], dtype=torch.int64, device="cuda")
    out = torch.empty(1, w.dim, device="cuda")
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_forward_noalloc(emb.handle, big_idx, big_off, 1, out)
    assert e.value.code == abi.TT_ERR_WORKSPACE
    emb.sync()
