"""Parity of mole_lookup_combine_grouped (tokens grouped by id, each distinct
row block fetched once per batch) against the fp64 oracle, and bit-identity
with mole_lookup_combine on the same inputs.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
推理阶段 (rows fetched by token id) and 复杂度分析 (per-token traffic is the token's
expert-output rows).  Tolerance: per-token relative L2 error <= 1e-5.
"""
import numpy as np
import pytest
import torch

from helpers import assert_combine_close, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _layer(seed, V, D, N, T, ids_kind="uniform"):
    rng = np.random.default_rng(seed)
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, ids_kind)
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    return ids, h, Wr, lut


def _both(mole, ids, h, Wr, lut):
    a = mole.mole_lookup_combine_grouped(dev(ids), dev(h), dev(Wr), dev(lut))
    st_a = mole.mole_check()
    b = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), dev(lut))
    st_b = mole.mole_check()
    return a.cpu().numpy(), st_a, b.cpu().numpy(), st_b


@pytest.mark.parametrize("V,D,N,T,kind", [
    (500, 256, 16, 1500, "zipf"),
    (3000, 768, 16, 2000, "zipf"),    # 192 units: two token groups per item
    (300, 64, 8, 1100, "uniform"),     # 16 units: 16 token groups
    (200, 128, 13, 1024, "zipf"),      # padded expert count
    (50, 128, 4, 3000, "uniform"),     # ~60 tokens per id: items split at 16 tokens
    (400, 96, 24, 1200, "zipf"),       # 24 experts padded to 32 (packed rows)
    (128, 64, 32, 2048, "zipf"),       # 32 experts
    (64, 2048, 32, 1030, "uniform"),   # 128 KB row blocks: no ring fits, ungrouped kernels
    (777, 256, 16, 333, "zipf"),       # below the grouping threshold: ungrouped kernels
    (20000, 128, 16, 14080, "zipf"),   # largest batch of the CTA-local kernel (16 experts)
    (20000, 128, 16, 14208, "zipf"),   # smallest batch of the interleaved kernel (148 SMs)
    (60000, 128, 16, 15000, "uniform"),  # interleaved: ~100 single-token items per CTA
    (700, 256, 12, 16000, "zipf"),     # interleaved, padded expert count
    (3000, 64, 8, 20011, "uniform"),   # interleaved, 8 experts, ragged last tile
    (400, 64, 32, 15000, "zipf"),      # 32 experts at a prefill size: router + gather kernels
    (5000, 64, 8, 40000, "zipf"),      # too many tokens per SM for the CTA-local kernel
])
def test_grouped_matches_oracle_and_ungrouped(mole, oracle_mod, V, D, N, T, kind):
    ids, h, Wr, lut = _layer(300 + D + N + T, V, D, N, T, kind)
    got, st, plain, st_plain = _both(mole, ids, h, Wr, lut)
    assert st == 0 and st_plain == 0
    ref, nbad = oracle_mod.combine(ids, h, Wr, lut)
    assert nbad == 0
    assert_combine_close(got, ref)
    np.testing.assert_array_equal(got, plain)


@pytest.mark.parametrize("T", [5000, 16000])
def test_grouped_single_hot_id(mole, oracle_mod, T):
    """All tokens share one id: 313 (1000) work items of that id; at 16000
    tokens each item of the interleaved kernel has a router tile of its own."""
    V, D, N = 100, 256, 16
    ids, h, Wr, lut = _layer(41, V, D, N, T)
    ids[:] = 7
    got, st, plain, _ = _both(mole, ids, h, Wr, lut)
    assert st == 0
    ref, _ = oracle_mod.combine(ids, h, Wr, lut)
    assert_combine_close(got, ref)
    np.testing.assert_array_equal(got, plain)


def test_grouped_every_id_distinct(mole, oracle_mod):
    V, D, N, T = 4096, 128, 8, 4096
    ids, h, Wr, lut = _layer(42, V, D, N, T)
    ids[:] = np.random.default_rng(3).permutation(V).astype(np.int32)
    got, st, plain, _ = _both(mole, ids, h, Wr, lut)
    assert st == 0
    ref, _ = oracle_mod.combine(ids, h, Wr, lut)
    assert_combine_close(got, ref)
    np.testing.assert_array_equal(got, plain)


def test_grouped_bad_ids(mole, oracle_mod):
    V, D, N, T = 300, 128, 16, 1500
    ids, h, Wr, lut = _layer(43, V, D, N, T, "zipf")
    bad_at = [0, 3, 17, 1499]
    ids[bad_at] = [-1, V, 2 ** 31 - 1, -7]
    out = mole.mole_lookup_combine_grouped(dev(ids), dev(h), dev(Wr), dev(lut))
    assert mole.mole_check() == 5  # MOLE_ERR_INDEX
    assert mole.mole_check() == 0
    got = out.cpu().numpy()
    bad = np.zeros(T, bool)
    bad[bad_at] = True
    assert np.isnan(got[bad]).all()
    ref, nbad = oracle_mod.combine(ids, h, Wr, lut)
    assert nbad == 4
    assert_combine_close(got[~bad], ref[~bad])


def test_grouped_all_ids_bad(mole):
    V, D, N, T = 300, 128, 16, 1024
    ids, h, Wr, lut = _layer(44, V, D, N, T)
    ids[:] = -1
    out = mole.mole_lookup_combine_grouped(dev(ids), dev(h), dev(Wr), dev(lut))
    assert mole.mole_check() == 5
    assert torch.isnan(out).all().item()


def test_grouped_workspace_reuse(mole, oracle_mod):
    """One workspace (sized for the largest batch) serves calls of other sizes;
    its contents on entry do not matter."""
    ws = torch.full((mole.mole_lookup_combine_grouped_workspace(4000, 16),), 0x5A, dtype=torch.uint8, device="cuda")
    for seed, T in [(51, 4000), (52, 1024), (53, 2500)]:
        ids, h, Wr, lut = _layer(seed, 900, 256, 16, T, "zipf")
        out = mole.mole_lookup_combine_grouped(dev(ids), dev(h), dev(Wr), dev(lut), workspace=ws)
        assert mole.mole_check() == 0
        ref, _ = oracle_mod.combine(ids, h, Wr, lut)
        assert_combine_close(out.cpu().numpy(), ref)


def test_grouped_workspace_too_small_is_rejected(mole):
    ids, h, Wr, lut = _layer(54, 300, 128, 16, 1500)
    need = mole.mole_lookup_combine_grouped_workspace(1500, 16)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(mole.MoleError) as e:
        mole.mole_lookup_combine_grouped(dev(ids), dev(h), dev(Wr), dev(lut), workspace=ws)
    assert e.value.status == 4


@pytest.mark.parametrize("T,kind", [(16384, "zipf"), (16384, "uniform"), (4096, "zipf")])
def test_grouped_full_size_sampled(mole, oracle_mod, T, kind):
    shape = inputs.SHAPES["1b"]
    V, D, N = shape.V, shape.D, shape.N
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 5)
    lut = (torch.randn((V, N, D), generator=g, device="cuda", dtype=torch.float32) * 0.02).to(torch.bfloat16)
    rng = np.random.default_rng(shape.seed + T + 5)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    ids[0], ids[-1] = 0, V - 1
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    out = mole.mole_lookup_combine_grouped(dev(ids), dev(h), dev(Wr), lut)
    assert mole.mole_check() == 0
    plain = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), lut)
    assert mole.mole_check() == 0
    assert torch.equal(out, plain)
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 62)]))
    uniq, inv = np.unique(ids[sample], return_inverse=True)
    rows = host_bits(lut[torch.from_numpy(uniq.astype(np.int64)).cuda()])
    ref, _ = oracle_mod.combine(inv.astype(np.int32), h[sample], Wr, rows)
    assert_combine_close(out[torch.from_numpy(sample).cuda()].cpu().numpy(), ref)
    del lut, out, plain
    torch.cuda.empty_cache()


def test_token_groups_serve_every_layer(mole, oracle_mod):
    """One grouping of the batch, three layers (own table, router, hidden
    states, expert counts 16 / 16 / 8) combined with it."""
    V, D, T = 700, 256, 2500
    rng = np.random.default_rng(61)
    ids = inputs.draw_ids(rng, T, V, "zipf")
    groups = mole.mole_token_groups_build(dev(ids), V, 16)
    for layer, N in enumerate([16, 16, 8]):
        lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
        Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
        h = inputs.normal(rng, (T, D), 1.0, "bf16")
        got = mole.mole_lookup_combine_groups(dev(ids), groups, dev(h), dev(Wr), dev(lut))
        assert mole.mole_check() == 0
        plain = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), dev(lut))
        assert mole.mole_check() == 0
        assert torch.equal(got, plain), f"layer {layer}"
        ref, _ = oracle_mod.combine(ids, h, Wr, lut)
        assert_combine_close(got.cpu().numpy(), ref)


def test_token_groups_bad_ids_and_small_batches(mole, oracle_mod):
    V, D, N = 300, 128, 16
    for T in (1500, 200, 15000):  # grouped kernels (CTA-local, interleaved); below their threshold the plain ones
        ids, h, Wr, lut = _layer(62 + T, V, D, N, T, "zipf")
        ids[[1, T - 1]] = [V + 5, -2]
        groups = mole.mole_token_groups_build(dev(ids), V, N)
        out = mole.mole_lookup_combine_groups(dev(ids), groups, dev(h), dev(Wr), dev(lut))
        assert mole.mole_check() == 5
        got = out.cpu().numpy()
        bad = np.zeros(T, bool)
        bad[[1, T - 1]] = True
        assert np.isnan(got[bad]).all()
        ref, _ = oracle_mod.combine(ids, h, Wr, lut)
        assert_combine_close(got[~bad], ref[~bad])


def test_token_groups_buffer_too_small(mole):
    ids, h, Wr, lut = _layer(63, 300, 128, 16, 1500)
    need = mole.mole_token_groups_workspace(1500, 16)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mole.MoleError) as e:
        mole.mole_token_groups_build(dev(ids), 300, 16, groups=small)
    assert e.value.status == 4
    groups = mole.mole_token_groups_build(dev(ids), 300, 8)  # sized for 8 experts
    with pytest.raises(mole.MoleError) as e:
        mole.mole_lookup_combine_groups(dev(ids), groups, dev(h), dev(Wr), dev(lut))  # a 16-expert layer
    assert e.value.status == 4
