import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU; runs the CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def mole():
    """The CUDA library binding (built in-tree if the .so is missing)."""
    from mixture_lookup_experts_b200 import _build
    _build.build()
    from mixture_lookup_experts_b200 import mole as m
    return m


def pytest_terminal_summary(terminalreporter):
    """Table-build diagnostics of the session (one line per comparison)."""
    try:
        from helpers import BUILD_DIAG, ERR_DIAG
    except ImportError:
        return
    tr = terminalreporter
    if ERR_DIAG:
        tr.write_sep("-", "measured errors against the oracle")
        for label, v in ERR_DIAG:
            tr.write_line(f"{label[:100]:100s} {v:.3e}")
    if not BUILD_DIAG:
        return
    tr.write_sep("-", "table build vs oracle (bf16 ulps; floor 2^-8 rms(row))")
    for d in BUILD_DIAG:
        tr.write_line(f"{d['label'][:60]:60s} n={d['elements']:>9d} beyond-allow {d['max_ulps_beyond_allowance']:.2f} "
                      f"unfloored-max {d['max_unfloored_ulps']:.3g} >2u-unfloored {d['pct_over_2_unfloored']:.4f}% "
                      f">2u-floored-raw {d['pct_over_2_floored_before_allowance']:.4f}% "
                      f"row-rel {d['max_row_rel_l2']:.2e}")
