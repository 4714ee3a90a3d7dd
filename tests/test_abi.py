"""The C-ABI library loads, exports every symbol include/fk.h declares, and
its host-side logic (argument checks, path choice, status strings) works
without a GPU.  No compute call is made here."""
import ctypes
import os
import re

import pytest
import torch

import distance_argmin_flashassign_b200 as fk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "fk.h")).read()
    return re.findall(r"^FK_API\s+[\w\s\*]+?\b(fk_\w+)\s*\(", src, flags=re.M)


def test_header_declares_the_binding_names():
    names = header_functions()
    assert len(names) == len(set(names)) >= 16
    assert set(names) == set(fk.ABI_NAMES)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(fk.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    assert fk.fk_status_string(0) == "ok"
    for code in range(-7, 0):
        assert fk.fk_status_string(code) not in ("", "unknown status")
    assert fk.fk_status_string(-99) == "unknown status"
    assert fk.fk_version() >= 100


def test_assign_path_choice():
    assert fk.fk_assign_path(1000, 128, torch.float16, 1024) == 1
    assert fk.fk_assign_path(1000, 128, torch.bfloat16, 1024) == 1
    assert fk.fk_assign_path(1000, 8, torch.float16, 3) == 1
    assert fk.fk_assign_path(1000, 32, torch.float32, 128) == 1   # fp32: three tf32 passes on tensor cores
    assert fk.fk_assign_path(1000, 30, torch.float32, 128) == 2   # fp32 rows not whole 16-byte groups
    assert fk.fk_assign_path(1000, 32, torch.float32, 128, B=3) == 2  # a batch of fp32 problems
    assert fk.fk_assign_path(1000, 100, torch.float16, 8) == 2    # D not a multiple of 8
    assert fk.fk_assign_path(1000, 256, torch.float16, 8) == 1    # up to 256 dimensions on tensor cores
    assert fk.fk_assign_path(1000, 264, torch.float16, 8) == 2    # D above 256
    assert fk.lib.fk_assign_path(10, 0, 1, 5, 1) == fk.FK_ERR_INVALID_ARG
    assert fk.lib.fk_assign_path(10, 8, 7, 5, 1) == fk.FK_ERR_INVALID_ARG


def test_forced_path_setting():
    try:
        fk.fk_set_assign_path(2)
        assert fk.fk_assign_path(1000, 128, torch.float16, 1024) == 2
        fk.fk_set_assign_path(1)
        assert fk.fk_assign_path(1000, 128, torch.float16, 1024) == 1
        assert fk.fk_assign_path(1000, 30, torch.float32, 1024) < 0
    finally:
        fk.fk_set_assign_path(0)
    with pytest.raises(fk.FKError):
        fk.fk_set_assign_path(5)


@pytest.mark.parametrize("args,what", [
    ((1, -1, 8, 1, 4), "N"), ((1, 10, 0, 1, 4), "D"), ((1, 10, 2000, 1, 4), "D"),
    ((1, 10, 8, 1, 0), "K"), ((1, 10, 8, 9, 4), "dtype"), ((0, 10, 8, 1, 4), "B"),
    ((1, 1 << 31, 8, 1, 4), "B*N"), ((2, 10, 8, 1, (1 << 22)), "B*K"),
])
def test_invalid_arguments_rejected_on_host(args, what):
    B, N, D, dt, K = args
    p = ctypes.c_void_p(16)
    st = fk.lib.fk_assign_batched(p, B, N, D, dt, p, K, p, None, None)
    assert st == fk.FK_ERR_INVALID_ARG
    assert what.split("*")[0] in fk.lib.fk_last_error_message().decode() or what == "dtype"
    assert fk.lib.fk_get_last_error() == fk.FK_ERR_INVALID_ARG
    st = fk.lib.fk_update_batched(p, p, B, N, D, dt, K, p, None, None)
    assert st == fk.FK_ERR_INVALID_ARG


def test_null_pointers_rejected():
    p = ctypes.c_void_p(16)
    assert fk.lib.fk_assign(None, 10, 8, 1, p, 4, p, None, None) == fk.FK_ERR_INVALID_ARG
    assert fk.lib.fk_update(p, p, 10, 8, 1, 4, None, None, None) == fk.FK_ERR_INVALID_ARG
    assert fk.lib.fk_lloyd(p, 10, 8, 1, p, 4, p, None, None, 0, None) == fk.FK_ERR_INVALID_ARG
    assert fk.lib.fk_lloyd_ooc(p, 10, 8, 1, p, 4, None, None, 1, 0, None) == fk.FK_ERR_INVALID_ARG


def test_empty_input_is_a_no_op_without_touching_the_device():
    p = ctypes.c_void_p(16)
    assert fk.lib.fk_assign(p, 0, 8, 1, p, 4, p, None, None) == fk.FK_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_no_device_is_an_error_not_a_crash():
    p = ctypes.c_void_p(16)
    st = fk.lib.fk_assign(p, 10, 8, 1, p, 4, p, None, None)
    assert st == fk.FK_ERR_CUDA
    assert fk.lib.fk_last_error_message()


def test_binding_validates_shapes():
    X = torch.zeros(10, 8, dtype=torch.float16)
    with pytest.raises(ValueError):
        fk.fk_assign(X, torch.zeros(4, 8, dtype=torch.float32))   # C dtype differs from X
    with pytest.raises(ValueError):
        fk.fk_update(X, torch.zeros(9, dtype=torch.int32), torch.zeros(4, 8))


def test_debug_inject_arguments():
    """The fault-injection hook validates its arguments and can be disarmed
    without a device."""
    assert fk.lib.fk_debug_inject(3, 0) == fk.FK_ERR_INVALID_ARG
    assert fk.lib.fk_debug_inject(1, -1) == fk.FK_ERR_INVALID_ARG
    assert fk.lib.fk_debug_inject(0, -1) == fk.FK_OK


def test_new_entry_points_validate_on_the_host():
    """Argument errors of the single-pass, top-2, Gauss and seeding calls are
    reported before any device work (these run without a GPU)."""
    p = ctypes.c_void_p(16)
    q = ctypes.c_void_p(32)
    lib = fk.lib
    # single pass: iters < 1, a K x D too large for shared memory
    assert lib.fk_lloyd_fused(p, 100, 8, 0, p, 4, p, None, None, 0, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_lloyd_fused(p, 100, 128, 0, p, 1024, p, None, None, 1, None) == fk.FK_ERR_UNSUPPORTED
    assert "single-pass" in lib.fk_last_error_message().decode()
    # top-2: aliased outputs, missing outputs
    assert lib.fk_assign_top2(p, 100, 8, 0, p, 4, q, q, None, None, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_assign_top2(p, 100, 8, 0, p, 4, q, None, None, None, None) == fk.FK_ERR_INVALID_ARG
    # Gauss sums: beta, signed weights without weights, no output
    f = ctypes.c_float
    assert lib.fk_gauss_sum(p, 100, 8, 0, p, 4, None, 0, f(0.0), q, None, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_gauss_sum(p, 100, 8, 0, p, 4, None, 1, f(1.0), q, None, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_gauss_sum(p, 100, 8, 0, p, 4, None, 0, f(1.0), None, None, None) == fk.FK_ERR_INVALID_ARG
    # seeding: a uniform outside [0, 1), N = 0
    import numpy as np
    u = np.array([0.5, 1.0], dtype=np.float64)
    assert lib.fk_seed_kmeanspp(p, 100, 8, 0, 2, ctypes.c_void_p(u.ctypes.data), q, None) == fk.FK_ERR_INVALID_ARG
    assert lib.fk_seed_kmeanspp(p, 0, 8, 0, 2, ctypes.c_void_p(u.ctypes.data), q, None) == fk.FK_ERR_INVALID_ARG
