"""The two error metrics of the parity tests on hand-made cases (CPU)."""
import numpy as np

from tests.parity import floor_elementwise_err, grouped_rel_err


def test_normwise_metric_scales_by_the_group_maximum():
    y = np.array([[4.0, 1e-6, -2.0], [0.0, 0.0, 0.0]])
    x = y.copy()
    x[0, 1] += 4e-4
    assert grouped_rel_err(x, y, (1,)) == 1e-4
    x[1, 0] = 1e-30                       # an all-zero group must stay exactly zero
    assert grouped_rel_err(x, y, (1,)) == float("inf")


def test_elementwise_metric_uses_each_element_down_to_the_floor():
    y = np.array([[4.0, 1e-6, -2.0]])
    x = y.copy()
    x[0, 2] -= 2e-4                       # 1e-4 of that element
    assert np.isclose(floor_elementwise_err(x, y, (1,)), 1e-4)
    x = y.copy()
    x[0, 1] += 4e-7                       # tiny element: compared with the floor 4e-3
    assert np.isclose(floor_elementwise_err(x, y, (1,)), 4e-7 / 4e-3)
    assert floor_elementwise_err(y, y, (1,)) == 0.0
