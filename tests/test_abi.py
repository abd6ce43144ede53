"""The C-ABI library builds, loads and exports every entry point include/ssa.h declares.
No compute calls: argument checks that return before touching a device only."""
import ctypes

import pytest

import spatial_sparse_attention_b200 as ssa


def test_every_declared_symbol_is_exported():
    names = ssa.declared_symbols()
    assert len(names) >= 13
    missing = [n for n in names if not hasattr(ssa.lib, n)]
    assert not missing, missing


def test_status_strings_and_launch_counter():
    assert ssa.lib.ssa_status_string(0) == b"ok"
    assert ssa.lib.ssa_status_string(3) == b"duplicate coordinate"
    assert ssa.lib.ssa_status_string(99) == b"unknown status"
    assert ssa.launch_count() >= 0


@pytest.mark.parametrize("args", [
    (None, 10, None, 8, 2),          # no coords, no grid
])
def test_plan_rejects_null_arguments_before_any_device_work(args):
    h = ctypes.c_void_p()
    assert ssa.lib.ssa_plan(*args, None, ctypes.byref(h)) == 1
    assert not h.value


def test_allocator_hook_must_be_paired():
    assert ssa.lib.ssa_set_allocator(ctypes.c_void_p(1), None, None) == 1
    assert ssa.lib.ssa_set_allocator(None, None, None) == 0
