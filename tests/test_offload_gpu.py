"""Offloaded table: the table (or its NF3 codes and scales) in pinned host
memory, each distinct id's row block staged to the device once per batch, the
combine reading the staging buffer.  Results must equal the device-resident
calls bit for bit and the fp64 oracle within 1e-5 per token.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
推理阶段 (the table kept in slower memory, rows fetched by token id) and
复杂度分析 (only the N expert-output rows of a token move).
"""
import numpy as np
import pytest
import torch

from helpers import assert_combine_close, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def pinned(a: np.ndarray) -> torch.Tensor:
    """numpy -> pinned host tensor (uint16 arrays are bf16 bit patterns)."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.pin_memory()


def _layer(seed, V, D, N, T, kind="zipf", dtype="bf16"):
    rng = np.random.default_rng(seed)
    lut = inputs.normal(rng, (V, N, D), 0.02, dtype)
    Wr = inputs.normal(rng, (D, N), 0.02, dtype)
    ids = inputs.draw_ids(rng, T, V, kind)
    h = inputs.normal(rng, (T, D), 1.0, dtype)
    return ids, h, Wr, lut


def _offload(mole, ids, h, Wr, table, V, scales=None):
    """(out, staging, U) through mole_token_groups_build -> mole_offload_stage
    -> mole_lookup_combine_offload."""
    T, N = ids.size, Wr.shape[1]
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    n_rows = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    staging = mole.mole_offload_stage(T, groups, table, scales, n_rows=n_rows)
    out = mole.mole_lookup_combine_offload(groups, dev(h), dev(Wr), staging, V, nf3=scales is not None)
    return out, staging, int(n_rows.item())


def _staged_ids(staged: np.ndarray, rows: np.ndarray, uniq: np.ndarray) -> np.ndarray:
    """The id whose row block each staged block is (rows[k] = table row of
    uniq[k], all distinct); -1 where none matches."""
    index = {rows[k].tobytes(): int(uniq[k]) for k in range(len(uniq))}
    return np.array([index.get(staged[u].tobytes(), -1) for u in range(len(staged))])


@pytest.mark.parametrize("V,D,N,T,kind", [
    (500, 256, 16, 1500, "zipf"),     # grouped kernels, tensor-core router
    (3000, 768, 16, 2000, "zipf"),
    (300, 64, 8, 1100, "uniform"),
    (200, 128, 13, 1024, "zipf"),     # padded expert count
    (400, 96, 24, 1200, "zipf"),      # 24 experts
    (64, 2048, 32, 1030, "uniform"),  # 128 KB row blocks: ungrouped kernels on the staged rows
    (777, 256, 16, 333, "zipf"),      # below the grouping threshold
    (50, 128, 4, 1, "uniform"),       # one token
    (40, 64, 16, 700, "uniform"),     # more tokens than ids: every id staged
])
def test_offload_matches_device_table_and_oracle(mole, oracle_mod, V, D, N, T, kind):
    ids, h, Wr, lut = _layer(700 + D + N + T, V, D, N, T, kind)
    out, staging, U = _offload(mole, ids, h, Wr, pinned(lut), V)
    assert mole.mole_check() == 0
    uniq = np.unique(ids)
    assert U == len(uniq)
    # the staging buffer holds each distinct id's row block once (in the
    # grouping's order, which is not unique: compare as a set)
    staged = host_bits(staging[: U * N * D * 2].view(torch.bfloat16).view(U, N * D))
    got_ids = _staged_ids(staged, lut[uniq].reshape(len(uniq), N * D), uniq)
    np.testing.assert_array_equal(np.sort(got_ids), uniq)
    plain = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), dev(lut))
    assert mole.mole_check() == 0
    assert torch.equal(out, plain)
    ref, nbad = oracle_mod.combine(ids, h, Wr, lut)
    assert nbad == 0
    assert_combine_close(out.cpu().numpy(), ref)


@pytest.mark.parametrize("V,N,D,T,kind", [
    (200, 16, 256, 1500, "zipf"),      # grouped NF3 kernels
    (300, 8, 2048, 1100, "uniform"),
    (100, 5, 128, 1200, "zipf"),       # N * D/64 not a multiple of 8: ungrouped kernels
    (64, 16, 256, 300, "zipf"),        # below the grouping threshold
    (30, 3, 64, 17, "uniform"),        # 8-byte code rows, 2-byte scale rows
])
def test_offload_nf3_matches_device_table_and_oracle(mole, oracle_mod, V, N, D, T, kind):
    rng = np.random.default_rng(T + D + N + 1)
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    codes, scales = oracle_mod.quantize_nf3(lut)
    out, _, U = _offload(mole, ids, h, Wr, pinned(codes), V, pinned(scales).view(torch.float16))
    assert mole.mole_check() == 0
    assert U == len(np.unique(ids))
    plain = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), dev(codes), dev(scales).view(torch.float16))
    assert mole.mole_check() == 0
    assert torch.equal(out, plain)
    ref, _ = oracle_mod.combine_nf3(ids, h, Wr, codes, scales)
    assert_combine_close(out.cpu().numpy(), ref)


@pytest.mark.parametrize("T", [33, 1500])
def test_offload_f32_table(mole, oracle_mod, T):
    V, D, N = 80, 192, 8
    ids, h, Wr, lut = _layer(77 + T, V, D, N, T, "zipf", "f32")
    out, _, U = _offload(mole, ids, h, Wr, pinned(lut), V)
    assert mole.mole_check() == 0
    plain = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), dev(lut))
    assert torch.equal(out, plain)
    ref, _ = oracle_mod.combine(ids, h, Wr, lut)
    assert_combine_close(out.cpu().numpy(), ref)


@pytest.mark.parametrize("T", [20, 1500])
def test_offload_bad_ids(mole, oracle_mod, T):
    V, D, N = 300, 128, 16
    ids, h, Wr, lut = _layer(88 + T, V, D, N, T)
    bad_at = [0, 5, T - 1]
    ids[bad_at] = [-1, V, 2 ** 31 - 1]
    out, _, U = _offload(mole, ids, h, Wr, pinned(lut), V)
    assert mole.mole_check() == 5
    assert mole.mole_check() == 0
    good = np.ones(T, bool)
    good[bad_at] = False
    assert U == len(np.unique(ids[good]))
    got = out.cpu().numpy()
    assert np.isnan(got[~good]).all()
    ref, nbad = oracle_mod.combine(ids, h, Wr, lut)
    assert nbad == 3
    assert_combine_close(got[good], ref[good])


def test_offload_from_device_memory_and_two_layers(mole, oracle_mod):
    """A device-resident table is staged the same way; one grouping and two
    staging buffers serve two layers."""
    V, D, T = 600, 256, 2000
    rng = np.random.default_rng(91)
    ids = inputs.draw_ids(rng, T, V, "zipf")
    groups = mole.mole_token_groups_build(dev(ids), V, 16)
    layers = [(inputs.normal(rng, (V, 16, D), 0.02, "bf16"), inputs.normal(rng, (D, 16), 0.02, "bf16"),
               inputs.normal(rng, (T, D), 1.0, "bf16")) for _ in range(2)]
    tables = [pinned(layers[0][0]), dev(layers[1][0])]
    stagings = [mole.mole_offload_stage(T, groups, tab, device="cuda") for tab in tables]
    for (lut, Wr, h), staging in zip(layers, stagings):
        out = mole.mole_lookup_combine_offload(groups, dev(h), dev(Wr), staging, V)
        assert mole.mole_check() == 0
        plain = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), dev(lut))
        assert torch.equal(out, plain)
        ref, _ = oracle_mod.combine(ids, h, Wr, lut)
        assert_combine_close(out.cpu().numpy(), ref)


def test_offload_rejects_pageable_memory_and_small_buffers(mole):
    V, D, N, T = 100, 128, 16, 1200
    ids, h, Wr, lut = _layer(92, V, D, N, T)
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    pageable = torch.from_numpy(lut.view(np.int16)).view(torch.bfloat16)
    with pytest.raises(mole.MoleError) as e:
        mole.mole_offload_stage(T, groups, pageable)
    assert e.value.status == 1
    need = mole.mole_offload_staging_bytes(T, V, N, D)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mole.MoleError) as e:
        mole.mole_offload_stage(T, groups, pinned(lut), staging=small)
    assert e.value.status == 4
    with pytest.raises(mole.MoleError) as e:
        mole.mole_lookup_combine_offload(groups, dev(h), dev(Wr), small, V)
    assert e.value.status == 4
    assert mole.mole_check() == 0


def test_offload_grouping_of_another_vocabulary(mole):
    """Groups built over a larger vocabulary than the staged table: ids past
    the table are not read (error word), and the combine stays inside the
    staging buffer (grouped kernels: error word and an abandoned layer;
    ungrouped kernels: NaN rows)."""
    for T in (300, 2000):
        V_build, V = 5000, 400
        ids, h, Wr, lut = _layer(93 + T, V_build, 128, 16, T, "uniform")
        table = pinned(lut[:V])
        groups = mole.mole_token_groups_build(dev(ids), V_build, 16)
        n_rows = torch.zeros(1, dtype=torch.int32, device="cuda")
        staging = mole.mole_offload_stage(T, groups, table, n_rows=n_rows)
        out = mole.mole_lookup_combine_offload(groups, dev(h), dev(Wr), staging, V)
        assert mole.mole_check() == 5
        assert 0 <= int(n_rows.item()) <= min(T, V)
        del out
    assert mole.mole_check() == 0


@pytest.mark.parametrize("kind", ["zipf", "uniform"])
def test_offload_full_size(mole, oracle_mod, kind):
    """1B-shaped layer ([50304, 16, 2048] bf16, 3.3 GB) in pinned host memory,
    a 16384-token batch: bit-identical to the device-resident table, sampled
    tokens against the oracle."""
    shape = inputs.SHAPES["1b"]
    V, D, N, T = shape.V, shape.D, shape.N, 16384
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 9)
    lut = (torch.randn((V, N, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    host = torch.empty(lut.shape, dtype=lut.dtype, pin_memory=True)
    host.copy_(lut)
    rng = np.random.default_rng(shape.seed + 13)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    ids[0], ids[-1] = 0, V - 1
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    out, staging, U = _offload(mole, ids, h, Wr, host, V)
    assert mole.mole_check() == 0
    assert U == len(np.unique(ids))
    plain = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), lut)
    assert mole.mole_check() == 0
    assert torch.equal(out, plain)
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 40)]))
    uniq, inv = np.unique(ids[sample], return_inverse=True)
    rows = host_bits(lut[torch.from_numpy(uniq.astype(np.int64)).cuda()])
    ref, _ = oracle_mod.combine(inv.astype(np.int32), h[sample], Wr, rows)
    assert_combine_close(out[torch.from_numpy(sample).cuda()].cpu().numpy(), ref)
    del lut, host, out, plain, staging
    torch.cuda.empty_cache()


def test_offload_nf3_full_size(mole, oracle_mod):
    shape = inputs.SHAPES["1b_nf3"]
    V, D, N, T = shape.V, shape.D, shape.N, 16384
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 17)
    lut = (torch.randn((V, N, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    codes, scales = mole.mole_quantize_lut_nf3(lut)
    del lut
    hc = torch.empty(codes.shape, dtype=codes.dtype, pin_memory=True)
    hs = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
    hc.copy_(codes)
    hs.copy_(scales)
    rng = np.random.default_rng(shape.seed + 19)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, "zipf")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    out, _, U = _offload(mole, ids, h, Wr, hc, V, hs)
    assert mole.mole_check() == 0
    plain = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), codes, scales)
    assert torch.equal(out, plain)
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 30)]))
    uniq, inv = np.unique(ids[sample], return_inverse=True)
    sel = torch.from_numpy(uniq.astype(np.int64)).cuda()
    ref, _ = oracle_mod.combine_nf3(inv.astype(np.int32), h[sample], Wr, codes[sel].cpu().numpy(),
                                    host_bits(scales[sel]))
    assert_combine_close(out[torch.from_numpy(sample).cuda()].cpu().numpy(), ref)
    del codes, scales, hc, hs, out, plain
    torch.cuda.empty_cache()
