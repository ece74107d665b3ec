"""CPU-side checks of the C ABI: the library loads, exports every symbol that
include/tt_emb.h declares, and rejects bad shapes and options on the host
before touching a device."""
import ctypes
import os
import re

import pytest

from tensor_train_compressed_mixed_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tt_emb_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(abi.LIB_PATH)
    names = declared_functions()
    assert "tt_emb_forward" in names and "tt_emb_backward" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_entry_point():
    for n in declared_functions():
        assert n in abi._SIGS, n
        assert hasattr(abi, n) or n in ("tt_emb_error_string",), n


def test_version_strings_and_options():
    assert abi.tt_emb_abi_version() == 1
    assert "index" in abi.error_string(abi.TT_ERR_INDEX_RANGE)
    assert abi.error_string(12345) == "unknown status code"
    o = abi.tt_emb_default_options()
    assert o.sched == abi.TT_SCHED_STEAL_L2 and o.grouping == abi.TT_GROUP_PREFIX


@pytest.mark.parametrize("n,rows,d,r", [
    ([[2, 3]], [6], [2, 2], [2, 4, 1]),          # r_0 != 1
    ([[2, 3]], [6], [2, 2], [1, 4, 2]),          # r_k != 1
    ([[2, 3]], [7], [2, 2], [1, 4, 1]),          # more rows than prod(n)
    ([[2, 3]], [0], [2, 2], [1, 4, 1]),          # no rows
    ([[2, 0]], [1], [2, 2], [1, 4, 1]),          # zero factor
    ([[2, 3]], [6], [64, 32], [1, 4, 1]),        # D > 1024
    ([[2, 3]], [6], [2, 2], [1, 129, 1]),        # rank above 128
    ([[2, 2, 2, 2, 2]], [32], [1] * 5, [1] * 6),  # k = 5
    ([[2]] * 65, [2] * 65, [2], [1, 1]),         # T = 65
])
def test_create_rejects_bad_shapes_on_host(n, rows, d, r):
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_create(n, rows, d, r)
    assert e.value.code == abi.TT_ERR_SHAPE


def test_create_rejects_bad_options_on_host():
    o = abi.tt_emb_default_options()
    o.sched = 7
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_create([[2, 3]], [6], [2, 2], [1, 4, 1], o)
    assert e.value.code == abi.TT_ERR_ARG
    o = abi.tt_emb_default_options()
    o.force_generic = 2
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_create([[2, 3]], [6], [2, 2], [1, 4, 1], o)
    assert e.value.code == abi.TT_ERR_ARG
    o = abi.tt_emb_default_options()
    o.precision = 3
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_create([[2, 3]], [6], [2, 2], [1, 4, 1], o)
    assert e.value.code == abi.TT_ERR_ARG
    o = abi.tt_emb_default_options()
    o.reserved[3] = 1
    with pytest.raises(abi.TTEmbError) as e:
        abi.tt_emb_create([[2, 3]], [6], [2, 2], [1, 4, 1], o)
    assert e.value.code == abi.TT_ERR_ARG
    for chunk in (-1, 257):   # subtask size: 1..256 distinct rows (0 = default)
        o = abi.tt_emb_default_options()
        o.chunk = chunk
        with pytest.raises(abi.TTEmbError) as e:
            abi.tt_emb_create([[2, 3]], [6], [2, 2], [1, 4, 1], o)
        assert e.value.code == abi.TT_ERR_ARG


def test_null_handle_calls_fail_cleanly():
    lib = abi.lib()
    assert lib.tt_emb_forward(None, None, None, 0, 1, None, None) == abi.TT_ERR_ARG
    assert lib.tt_emb_backward(None, None, None) == abi.TT_ERR_ARG
    assert lib.tt_emb_sgd_update(None, 0.1, None) == abi.TT_ERR_ARG
    assert lib.tt_emb_backward_sgd(None, None, 0.1, None) == abi.TT_ERR_ARG
    assert lib.tt_emb_sync(None) == abi.TT_ERR_ARG
    lib.tt_emb_destroy(None)


@pytest.mark.parametrize("n,d,r", [
    ([[5, 6, 7]], [4, 4, 4], [1, 32, 32, 1]),      # d_3 = 4
    ([[5, 6, 7]], [4, 4, 8], [1, 16, 16, 1]),      # rank 16
    ([[5, 6, 7]], [4, 4, 8], [1, 32, 64, 1]),      # r_1 != r_2
    ([[2, 3]], [2, 2], [1, 4, 1]),                 # two cores
    ([[2, 5, 6, 7]], [2, 4, 4, 4], [1, 32, 32, 32, 1]),  # four cores
])
def test_tensor_core_precisions_reject_other_shapes(n, d, r):
    rows = [int(__import__("numpy").prod(x)) for x in n]
    for prec in (abi.TT_PREC_BF16_TC, abi.TT_PREC_FP32_SPLIT_TC):
        o = abi.tt_emb_default_options()
        o.precision = prec
        with pytest.raises(abi.TTEmbError) as e:
            abi.tt_emb_create(n, rows, d, r, o)
        assert e.value.code == abi.TT_ERR_SHAPE


def test_handle_free_calls_reject_a_null_handle():
    assert abi.lib().tt_emb_last_error(None) == abi.TT_ERR_ARG
    assert abi.lib().tt_emb_debug_inject(None, abi.TT_INJECT_POOL_WAIT, 0) == abi.TT_ERR_ARG
    assert abi.lib().tt_emb_sync(None) == abi.TT_ERR_ARG
