"""The C-ABI library on a machine without a GPU: it loads, exports every
function include/rlt.h declares, and its host-only calls (validation, arena
sizing, the scheduler's plan, status strings) behave as documented."""
import ctypes

import numpy as np
import pytest

from token_recurrent_decoding_b200 import configs, rlt


def test_every_declared_symbol_is_exported():
    lib = rlt._lib()
    names = rlt.header_symbols()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_check_config_and_arena_sizes():
    for name, wl in configs.workloads().items():
        assert rlt.check_config(wl.model, wl.batch, wl.max_len) == 0, name
        assert rlt.arena_bytes(wl.model, wl.batch, wl.max_len) > 0
    lib = rlt._lib()
    c = rlt.make_config(configs.M50, 4, 16)
    c.window = 0
    assert lib.rlt_check_config(ctypes.byref(c)) == 1
    c = rlt.make_config(configs.M50, 4, 16)
    c.mem_groups = 3
    assert lib.rlt_check_config(ctypes.byref(c)) == 2
    c = rlt.make_config(configs.M50, 4, 16)
    c.max_prefill_tokens = 8  # below max_len
    assert lib.rlt_check_config(ctypes.byref(c)) == 1
    assert lib.rlt_arena_bytes(ctypes.byref(c)) == 0
    # dh = 48 is not covered by the kernels
    assert rlt.check_config(configs.M50.replace(n_heads=4, head_dim=48, d=192), 4, 16) == 2
    # a bigger window or more sequences never needs less memory
    a = rlt.arena_bytes(configs.M140, 16, 512)
    assert rlt.arena_bytes(configs.M140, 32, 512) > a
    assert rlt.arena_bytes(configs.M140.replace(window=256), 16, 512) > a


def test_status_strings():
    lib = rlt._lib()
    for code in range(9):
        assert lib.rlt_status_string(code)
    assert b"unknown" in lib.rlt_status_string(99)


@pytest.mark.parametrize("steps", [[3, 1, 4, 1, 5], [0, 0], [7], list(range(20, 0, -3))])
def test_ragged_plan(steps):
    order, sizes = rlt.plan_ragged(steps)
    assert sorted(order.tolist()) == list(range(len(steps)))
    # longest first, ties in input order
    assert [steps[i] for i in order] == sorted(steps, reverse=True)
    assert len(sizes) == max(steps)
    for k, c in enumerate(sizes):
        assert c == sum(1 for s in steps if s > k)
    assert sum(sizes) == sum(steps)


def test_ragged_plan_of_the_serving_workload():
    wl = configs.workloads()["ragged_bf16"]
    order, sizes = rlt.plan_ragged(wl.lengths)
    assert sum(sizes) == wl.seq_steps == 1381014
    assert sizes[0] == 1024 and len(sizes) == max(wl.lengths)
    assert np.all(np.diff(sizes) <= 0)


def test_attend_workspace_sizing():
    assert rlt.attend_workspace_bytes(0, 1, 64, 8) == 0
    assert rlt.attend_workspace_bytes(4, 1, 48, 8) == 0
    a = rlt.attend_workspace_bytes(256, 12, 64, 1024)
    assert a > 256 * 12 * 66 * 4  # partials of more than one chunk per (row, head)
    assert rlt.attend_workspace_bytes(256, 12, 64, 2048) > a


def test_backward_workspace_bytes_host_only():
    """rlt_backward_workspace_bytes is host arithmetic: 0 for an invalid
    configuration or empty chunk, growing with rows and positions."""
    from token_recurrent_decoding_b200 import configs, rlt
    lib = rlt._lib()
    c = rlt.make_config(configs.TINY, 4, 64)
    import ctypes as C
    f = lambda n, s: lib.rlt_backward_workspace_bytes(C.byref(c), n, s)
    assert f(0, 8) == 0 and f(2, 0) == 0
    assert 0 < f(1, 8) < f(2, 8) and f(2, 8) < f(2, 16)
    bad = rlt.make_config(configs.TINY.replace(window=2000), 4, 64)
    assert lib.rlt_backward_workspace_bytes(C.byref(bad), 2, 8) == 0
