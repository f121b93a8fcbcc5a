"""The C-ABI library loads and exports every symbol include/mole.h declares;
host-only calls and host-side argument checks work without a GPU (no compute)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mole.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mole_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path(mole):
    names = declared_functions()
    for required in ["mole_build_lut", "mole_lookup_combine", "mole_quantize_lut_nf3",
                     "mole_lookup_combine_nf3", "mole_gather_plan", "mole_check"]:
        assert required in names


def test_every_declared_symbol_is_exported(mole):
    lib = ctypes.CDLL(mole.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in mole.h but not exported"
    # and the binding knows the signature of each
    assert set(declared_functions()) <= set(mole.SIGNATURES)


def test_status_strings_and_version(mole):
    assert mole.mole_version() >= 100
    for s in range(9):
        assert mole.mole_status_str(s)
    assert mole.mole_status_str(0) == "ok"


def test_workspace_size(mole):
    import torch
    assert mole.mole_build_lut_workspace(50304, 2048, 16, 8192, torch.bfloat16, 1) == 50304 * 8192 * 2
    assert mole.mole_build_lut_workspace(50304, 2048, 16, 8192, torch.bfloat16, 0) == 50304 * 8192 * 2 * 16
    assert mole.mole_build_lut_workspace(512, 64, 4, 256, torch.float32, 99) == 512 * 256 * 4 * 4
    assert mole.mole_build_lut_workspace(0, 64, 4, 256, torch.float32, 1) == 0


def test_nf3_tables_match_the_oracle(mole, oracle_mod):
    # the library's level/midpoint literals equal the oracle's construction
    assert mole.mole_nf3_levels() == [int(x) for x in oracle_mod.nf3_levels_f16()]
    np.testing.assert_array_equal(np.array(mole.mole_nf3_midpoints(), np.float32), oracle_mod.nf3_midpoints())


def test_argument_checks_without_device(mole):
    lib = mole.lib
    P = 0x100000  # a fake, aligned, never dereferenced address
    # negative / zero sizes and null pointers are rejected before any CUDA call
    assert lib.mole_lookup_combine(P, -1, P, P, P, 10, 4, 64, 1, P, None) == 1
    assert lib.mole_lookup_combine(P, 5, None, P, P, 10, 4, 64, 1, P, None) == 1
    assert lib.mole_lookup_combine(P, 5, P, P, P, 10, 33, 64, 1, P, None) == 3   # N > 32
    assert lib.mole_lookup_combine(P, 5, P, P, P, 10, 4, 24, 1, P, None) == 3   # bf16 needs D % 16
    assert lib.mole_lookup_combine(P, 5, P + 4, P, P, 10, 4, 64, 1, P, None) == 2  # misaligned h
    assert lib.mole_lookup_combine(P, 5, P, P, P, 10, 4, 64, 7, P, None) == 1   # bad dtype
    assert lib.mole_lookup_combine(P, 0, P, P, P, 10, 4, 64, 1, P, None) == 0   # T == 0: no-op
    assert lib.mole_lookup_combine_nf3(P, 5, P, P, P, P, 10, 4, 96, 1, P, None) == 3  # D % 64
    assert lib.mole_quantize_lut_nf3(P, 10, 4, 100, P, P, None) == 3
    assert lib.mole_quantize_lut_nf3(None, 10, 4, 128, P, P, None) == 1
    assert lib.mole_build_lut(P, P, P, 10, 64, 2, 64, 0, 1, P, None, 0, None) == 4   # no workspace
    assert lib.mole_build_lut(P, P, P, 10, 64, 2, 64, 9, 1, P, P, 1 << 20, None) == 1  # bad act
    assert lib.mole_gather_plan(P, -3, 10, P, P, P, None) == 1


def test_valid_arguments_reach_the_device_check(mole):
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    P = 0x100000
    # all checks pass, then there is no sm_100 device here
    assert mole.lib.mole_lookup_combine(P, 5, P, P, P, 10, 4, 64, 1, P, None) == 8
