"""Host-side checks of the benchmark's output contract: the headline JSON
line stays short enough for a reader that keeps only the tail of stdout."""
import json

import pytest

import bench


def _worst_case_headline():
    cfg = bench.workload_config(16384, "uniform", 16, "grouped")
    roof = {"bound": "hbm", "achieved": 4699.1234567, "peak": 6451.8, "unit": "GB/s", "frac": 0.728383838383,
            "traffic": 454212345.123, "kernel": max(bench.KERNELS.values(), key=len),
            "bytes_per_launch": 1117912345.123, "unique_rows": 13983.4375, "avg_launch_us": 199.612345678,
            "peak_source": "measured hbm_gbs", "frac_of_8TBs": 0.58737373737,
            "traffic_source": "kernel changed since the ncu capture"}
    e2e = {"value": 1.0123456789e7, "unit": "tokens/s", "h2d_bytes_per_step": 16 * 16384 * 2048 * 2 + 16384 * 4,
           "d2h_bytes_per_step": 16 * 16384 * 2048 * 4, "steps": 20,
           "note": "per step: ids + 16 h H2D (pinned), 16 C-ABI calls, 16 outputs D2H"}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap", "sw_thermal_slowdown"],
              "samples": 312}
    cpu = {"value": 8674.123456789, "unit": "tokens/s", "cores": 192, "kind": "oracle",
           "sample": "1024 tokens of one 1B-shaped layer x 12345 repetitions (10.0 s); tokens/s through 16 layers "
                     "= per-layer rate / 16"}
    return bench.headline(value=10023456.123456, world=8, K=1000, W=100, max_ms=1635.123456789, cfg=cfg,
                          roofline=roof, e2e=e2e, launches=34000, prep_us=42.123456789, clocks=clocks, cpu=cpu)


def test_headline_fits_the_tail():
    line = json.dumps(_worst_case_headline())
    assert len(line) <= bench.HEADLINE_MAX_BYTES, len(line)


def test_headline_keeps_the_contract_keys():
    d = _worst_case_headline()
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert k in d, k
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in d["roofline"], k
    assert d["config"]["workload"]


def test_compact_rounds_floats_only():
    assert bench.compact({"a": [1.23456789, 7], "b": "x", "c": None, "d": True}) == \
        {"a": [1.23457, 7], "b": "x", "c": None, "d": True}
    assert bench.compact(1234567890.5) == pytest.approx(1234570000.0)


def test_launch_count_of_the_headline_step():
    """The headline step on 148 SMs: the grouping (plan + shares) and one
    interleaved-kernel launch per layer; past the shares' size, router +
    gather per layer; the plain path two per layer; decode sizes one."""
    assert bench.launches_per_step(16384, 16, 16, "grouped", n_sm=148) == 2 + 16
    assert bench.launches_per_step(4096, 16, 16, "grouped", n_sm=148) == 2 + 16
    assert bench.launches_per_step(40000, 16, 16, "grouped", n_sm=148) == 1 + 2 * 16
    assert bench.launches_per_step(16384, 32, 16, "grouped", n_sm=148) == 2 + 2 * 16
    assert bench.launches_per_step(16384, 16, 16, "plain", n_sm=148) == 32
    assert bench.launches_per_step(64, 16, 12, "grouped", n_sm=148) == 12
