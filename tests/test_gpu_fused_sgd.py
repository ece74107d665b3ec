"""tt_emb_backward_sgd: backward and SGD step fused, with the middle core updated sparsely
in place by the block that reduces its column group (its gradient is never materialised).
The resulting cores must be those of the oracle's SGD step within the fp32 bound; the
first and last cores' gradients are still returned; G_2 slices no lookup touched are
bit-for-bit unchanged; four-core tables take the unfused path with the same result."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import FP32_TOL, core_grad_err, gpu_forward
from workloads import config_workload, random_workload

pytestmark = pytest.mark.gpu


def _fused_step(w, options=None, lr=0.01):
    emb, cores, out = gpu_forward(w, options=options, with_grads=True)
    before = [[c.detach().clone().cpu().numpy() for c in tab] for tab in cores]
    g = torch.from_numpy(w.grad_out).cuda()
    emb.backward_sgd(g, lr)
    emb.sync()
    after = [[c.cpu().numpy() for c in tab] for tab in cores]
    grads = [[x.cpu().numpy() for x in emb.grads[t * emb.k:(t + 1) * emb.k]] for t in range(emb.T)]
    return before, after, grads


@pytest.mark.parametrize("prec", ["fp32", "split"])
def test_fused_step_matches_oracle_sgd(prec):
    from tensor_train_compressed_mixed_b200 import abi
    o = abi.tt_emb_default_options()
    o.precision = abi.TT_PREC_FP32 if prec == "fp32" else abi.TT_PREC_FP32_SPLIT_TC
    w = config_workload(4, batch=24, tables=3, with_grad=True)
    before, after, grads = _fused_step(w, o)
    want = oracle.workload_backward(w)
    upd = oracle.sgd(w.cores, want, 0.01)
    for t in range(w.num_tables):
        for j in range(3):
            assert core_grad_err(after[t][j], upd[t][j]) <= FP32_TOL, (t, j)
        for j in (0, 2):   # the first and last cores' gradients are still returned
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)


def test_untouched_middle_slices_are_not_written():
    # a small column factor and few lookups: many G_2[:, i_2] no lookup reaches
    w = random_workload(970, (4, 4, 8), (1, 32, 32, 1), [(6, 40, 7)], batch=5,
                        pooling={"kind": "uniform", "lo": 0, "hi": 3}, with_grad=True)
    before, after, _ = _fused_step(w)
    n2 = w.n[0][1]
    touched = np.zeros(n2, dtype=bool)
    touched[(w.indices // w.n[0][2]) % n2] = True
    assert (~touched).any() and touched.any()
    assert np.array_equal(after[0][1][:, ~touched], before[0][1][:, ~touched])
    upd = oracle.sgd(w.cores, oracle.workload_backward(w), 0.01)
    assert core_grad_err(after[0][1], upd[0][1]) <= FP32_TOL


def test_four_core_tables_take_the_unfused_path():
    w = config_workload(5, batch=12, tables=2, with_grad=True)
    before, after, grads = _fused_step(w)
    want = oracle.workload_backward(w)
    upd = oracle.sgd(w.cores, want, 0.01)
    for t in range(w.num_tables):
        for j in range(w.num_cores):
            assert core_grad_err(after[t][j], upd[t][j]) <= FP32_TOL, (t, j)
            assert core_grad_err(grads[t][j], want[t][j]) <= FP32_TOL, (t, j)


def test_fused_step_with_no_lookups_keeps_the_cores():
    w = random_workload(971, (4, 4, 8), (1, 64, 64, 1), [(5, 6, 7)], batch=8,
                        pooling={"kind": "uniform", "lo": 0, "hi": 0}, with_grad=True)
    before, after, _ = _fused_step(w)
    for j in range(3):
        assert np.array_equal(after[0][j], before[0][j])
