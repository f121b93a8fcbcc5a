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
    assert lib.mole_check(None, -1) == 1  # no unbounded host wait
    tabs = (ctypes.c_void_p * 2)(P, P + 4096)
    assert lib.mole_prefetch_rows(P, 4, tabs, 2, 10, 24, None) == 2      # row bytes not a multiple of 16
    assert lib.mole_prefetch_rows(P, 4, tabs, 65, 10, 32, None) == 3     # more than 64 tables
    assert lib.mole_prefetch_rows(P, -1, tabs, 2, 10, 32, None) == 1     # negative T
    assert lib.mole_prefetch_rows(P, 4, None, 2, 10, 32, None) == 1      # no table list
    bad = (ctypes.c_void_p * 1)(P + 8)
    assert lib.mole_prefetch_rows(P, 4, bad, 1, 10, 32, None) == 2       # unaligned table
    assert lib.mole_prefetch_rows(P, 0, tabs, 2, 10, 32, None) == 0      # T == 0: no-op


def test_valid_arguments_reach_the_device_check(mole):
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    P = 0x100000
    # all checks pass, then there is no sm_100 device here
    assert mole.lib.mole_lookup_combine(P, 5, P, P, P, 10, 4, 64, 1, P, None) == 8


def test_grouped_workspace_size_and_checks(mole):
    size = mole.mole_lookup_combine_grouped_workspace
    assert size(0, 16) == 0 and size(100, 0) == 0 and size(100, 33) == 0
    s1, s2 = size(16384, 16), size(32768, 16)
    # hash table (2T slots, 12 B each), 4 per-token int arrays, items, gates
    assert s1 >= 16384 * (4 * 4 + 16 + 16 * 4) + 2 * 16384 * 12
    assert s2 > s1 and size(16384, 32) > s1
    lib = mole.lib
    P = 0x100000
    ws = size(5, 4)
    assert lib.mole_lookup_combine_grouped(P, 5, P, P, P, 10, 4, 64, 1, P, None, ws, None) == 4      # no workspace
    assert lib.mole_lookup_combine_grouped(P, 5, P, P, P, 10, 4, 64, 1, P, P, ws - 1, None) == 4     # too small
    assert lib.mole_lookup_combine_grouped(P, 5, P, P, P, 10, 4, 64, 1, P, P + 8, ws, None) == 2     # misaligned
    assert lib.mole_lookup_combine_grouped(P, 5, P, P, P, 10, 4, 24, 1, P, P, ws, None) == 3         # D % 16
    assert lib.mole_lookup_combine_grouped(P, 0, P, P, P, 10, 4, 64, 1, P, None, 0, None) == 0       # T == 0
    import torch
    if not torch.cuda.is_available():
        assert lib.mole_lookup_combine_grouped(P, 5, P, P, P, 10, 4, 64, 1, P, P, ws, None) == 8     # no device


def test_token_groups_checks(mole):
    lib = mole.lib
    P = 0x100000
    assert mole.mole_token_groups_workspace(16384, 16) == mole.mole_lookup_combine_grouped_workspace(16384, 16)
    assert mole.mole_token_groups_workspace(16384, 8) < mole.mole_token_groups_workspace(16384, 16)
    ws = mole.mole_token_groups_workspace(5, 4)
    assert lib.mole_token_groups_build(P, 5, 10, 4, None, ws, None) == 4
    assert lib.mole_token_groups_build(P, 5, 10, 4, P, ws - 1, None) == 4
    assert lib.mole_token_groups_build(P, 5, 10, 4, P + 4, ws, None) == 2
    assert lib.mole_token_groups_build(P, 5, 10, 40, P, ws, None) == 3
    assert lib.mole_token_groups_build(None, 5, 10, 4, P, ws, None) == 1
    assert lib.mole_token_groups_build(P, 0, 10, 4, None, 0, None) == 0
    assert lib.mole_lookup_combine_groups(P, 5, None, ws, P, P, P, 10, 4, 64, 1, P, None) == 4
    assert lib.mole_lookup_combine_groups(P, 5, P, ws, P, P, P, 10, 4, 24, 1, P, None) == 3
    assert lib.mole_lookup_combine_groups(P, 0, None, 0, P, P, P, 10, 4, 64, 1, P, None) == 0


def test_offload_staging_size_and_checks(mole):
    import torch
    size = mole.mole_offload_staging_bytes
    # room for min(T, V) row blocks
    assert size(16384, 50304, 16, 2048) == 16384 * 16 * 2048 * 2
    assert size(100, 40, 16, 2048) == 40 * 16 * 2048 * 2
    assert size(100, 40, 8, 64, torch.float32) == 40 * 8 * 64 * 4
    nb = 16 * 2048 // 64
    assert size(1000, 50304, 16, 2048, nf3=True) == (1000 * nb * 24 + 255) // 256 * 256 + 1000 * nb * 2
    assert size(0, 10, 4, 64) == 0 and size(5, 10, 33, 64) == 0 and size(5, 10, 4, 96, nf3=True) == 0
    lib = mole.lib
    P = 0x100000
    gws = mole.mole_token_groups_workspace(5, 4)
    sws = size(5, 10, 4, 64)
    stage = lib.mole_offload_stage
    assert stage(5, None, gws, P, None, 10, 4, 64, 1, 0, P, sws, None, None) == 4          # no groups
    assert stage(5, P, gws, P, None, 10, 4, 64, 1, 0, P, sws - 1, None, None) == 4         # staging too small
    assert stage(5, P, gws, P, None, 10, 4, 64, 1, 0, P + 8, sws, None, None) == 2         # staging misaligned
    assert stage(5, P, gws, None, None, 10, 4, 64, 1, 0, P, sws, None, None) == 1          # no table
    assert stage(5, P, gws, P + 8, None, 10, 4, 64, 1, 0, P, sws, None, None) == 2         # table misaligned
    assert stage(5, P, gws, P, None, 10, 4, 64, 1, 1, P, size(5, 10, 4, 64, nf3=True), None, None) == 1  # no scales
    assert stage(5, P, gws, P, None, 10, 4, 64, 1, 2, P, sws, None, None) == 1             # bad table kind
    assert stage(5, P, gws, P, None, 10, 4, 24, 1, 0, P, sws, None, None) == 3             # D % 16
    assert stage(5, P, gws, P, None, 10, 4, 64, 1, 0, P, sws, P + 2, None) == 2            # n_rows misaligned
    assert stage(0, None, 0, None, None, 10, 4, 64, 1, 0, None, 0, None, None) == 0         # T == 0
    comb = lib.mole_lookup_combine_offload
    assert comb(5, P, gws, P, P, P, sws - 1, 10, 4, 64, 1, 0, P, None) == 4
    assert comb(5, P, gws, None, P, P, sws, 10, 4, 64, 1, 0, P, None) == 1
    assert comb(5, P, gws, P + 4, P, P, sws, 10, 4, 64, 1, 0, P, None) == 2
    assert comb(0, None, 0, None, None, None, 0, 10, 4, 64, 1, 0, None, None) == 0
    if not torch.cuda.is_available():
        assert stage(5, P, gws, P, None, 10, 4, 64, 1, 0, P, sws, None, None) == 8
        assert comb(5, P, gws, P, P, P, sws, 10, 4, 64, 1, 0, P, None) == 8


def test_ffn_checks(mole):
    import torch
    lib = mole.lib
    P = 0x100000
    assert mole.mole_shared_ffn_workspace(100, 512) == 100 * 512 * 2
    assert mole.mole_ffn_block_workspace(100, 128, 512) >= 100 * 512 * 2 + 100 * 128 * 4
    ws = mole.mole_shared_ffn_workspace(5, 64)
    assert lib.mole_shared_ffn(P, P, P, 5, 64, 64, 9, None, None, P, P, ws, None) == 1       # bad act
    assert lib.mole_shared_ffn(P, P, P, 5, 96, 64, 0, None, None, P, P, ws, None) == 3       # D % 64
    assert lib.mole_shared_ffn(P, P, P, 5, 64, 64, 0, None, None, P, P, ws - 1, None) == 4   # workspace
    assert lib.mole_shared_ffn(P, P, P, 5, 64, 64, 0, P + 4, None, P, P, ws, None) == 2     # misaligned add
    assert lib.mole_shared_ffn(None, P, P, 5, 64, 64, 0, None, None, P, P, ws, None) == 1    # no h
    assert lib.mole_shared_ffn(None, None, None, 0, 64, 64, 0, None, None, None, None, 0, None) == 0  # T == 0
    gws = mole.mole_token_groups_workspace(5, 4)
    fws = mole.mole_ffn_block_workspace(5, 64, 64)
    blk = lib.mole_ffn_block
    assert blk(P, 5, P, gws, P, P, P, 10, 4, P, P, 64, 64, 0, None, P, P, fws - 1, None) == 4
    assert blk(P, 5, P, gws, P, P, P, 10, 4, None, P, 64, 64, 0, None, P, P, fws, None) == 1
    assert blk(P, 5, P, gws, P, P, P, 10, 4, P, P, 64, 96, 0, None, P, P, fws, None) == 3
    assert blk(P, 5, None, gws, P, P, P, 10, 4, P, P, 64, 64, 0, None, P, P, fws, None) == 4
    if not torch.cuda.is_available():
        assert lib.mole_shared_ffn(P, P, P, 5, 64, 64, 0, None, None, P, P, ws, None) == 8
        assert blk(P, 5, P, gws, P, P, P, 10, 4, P, P, 64, 64, 0, None, P, P, fws, None) == 8


def test_build_nf3_checks(mole):
    import torch
    lib = mole.lib
    P = 0x100000
    ws = mole.mole_build_lut_workspace(10, 64, 2, 64, torch.bfloat16, 1)
    f = lib.mole_build_lut_nf3
    assert f(P, P, P, 10, 64, 2, 64, 9, P, P, P, ws, None) == 1       # bad act
    assert f(P, P, P, 10, 96, 2, 64, 0, P, P, P, ws, None) == 3       # D % 64
    assert f(P, P, P, 10, 64, 2, 64, 0, P, P, P, ws - 1, None) == 4   # workspace
    assert f(P, P, P, 10, 64, 2, 64, 0, P + 4, P, P, ws, None) == 2   # codes misaligned
    assert f(P, P, P, 10, 64, 2, 64, 0, None, P, P, ws, None) == 1    # no codes
    if not torch.cuda.is_available():
        assert f(P, P, P, 10, 64, 2, 64, 0, P, P, P, ws, None) == 8
