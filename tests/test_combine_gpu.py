"""Parity of mole_lookup_combine (CUDA, through the C ABI) against the fp64 oracle.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
训练阶段 (router on the hidden state, all routed experts active) and 推理阶段
(rows fetched from the table by token id).  Tolerance: per-token relative L2
error <= 1e-5; gather indices bit-exact via one-hot gates.
"""
import numpy as np
import pytest
import torch

from helpers import as_f64, assert_combine_close, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _layer(seed, V, D, N, T, dtype="bf16", ids_kind="uniform", lut_std=0.02):
    rng = np.random.default_rng(seed)
    lut = inputs.normal(rng, (V, N, D), lut_std, dtype)
    Wr = inputs.normal(rng, (D, N), 0.02, dtype)
    ids = inputs.draw_ids(rng, T, V, ids_kind)
    h = inputs.normal(rng, (T, D), 1.0, dtype)
    return ids, h, Wr, lut


def _run(mole, ids, h, Wr, lut):
    out = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), dev(lut))
    st = mole.mole_check()
    return out.cpu().numpy(), st


@pytest.mark.parametrize("V,D,N,T,kind", [
    (1000, 256, 16, 1000, "uniform"),
    (777, 768, 16, 333, "zipf"),
    (300, 64, 4, 50, "uniform"),
    (500, 128, 8, 97, "zipf"),
    (400, 32, 13, 71, "uniform"),
    (200, 16, 1, 17, "uniform"),
    (256, 96, 24, 40, "uniform"),
    (128, 48, 32, 33, "uniform"),
    (50304, 2048, 16, 300, "zipf"),
    (64, 2048, 32, 40, "uniform"),   # row block of 128 KB: register-gather kernel
    (96, 1024, 24, 77, "zipf"),      # 48 KB row blocks, padded expert count
    # >= 1024 tokens: router kernel + bulk-copy gather kernel
    (3000, 768, 16, 2000, "zipf"),   # two token groups per CTA
    (500, 256, 16, 1500, "uniform"),
    (300, 64, 8, 1100, "uniform"),
    (200, 128, 13, 1024, "zipf"),    # padded expert count
    (64, 2048, 32, 1030, "uniform"), # 128 KB row blocks: no ring fits, fused kernel
])
def test_combine_bf16_matches_oracle(mole, oracle_mod, V, D, N, T, kind):
    ids, h, Wr, lut = _layer(100 + D + N + T, V, D, N, T, ids_kind=kind)
    got, st = _run(mole, ids, h, Wr, lut)
    assert st == 0
    ref, nbad = oracle_mod.combine(ids, h, Wr, lut)
    assert nbad == 0
    assert_combine_close(got, ref)


@pytest.mark.parametrize("T", [1, 2, 3, 15, 16, 17, 31, 33, 255, 1024, 4097])
def test_combine_tile_boundaries(mole, oracle_mod, T):
    ids, h, Wr, lut = _layer(7 + T, 613, 128, 16, T)
    got, st = _run(mole, ids, h, Wr, lut)
    assert st == 0
    ref, _ = oracle_mod.combine(ids, h, Wr, lut)
    assert_combine_close(got, ref)


@pytest.mark.parametrize("V,D,N,T", [(512, 64, 4, 256), (100, 36, 7, 19), (64, 4, 1, 5)])
def test_combine_f32_matches_oracle(mole, oracle_mod, V, D, N, T):
    ids, h, Wr, lut = _layer(200 + T, V, D, N, T, dtype="f32")
    got, st = _run(mole, ids, h, Wr, lut)
    assert st == 0
    ref, _ = oracle_mod.combine(ids, h, Wr, lut)
    assert_combine_close(got, ref)


def test_combine_edges(mole, oracle_mod):
    V, D, N = 1000, 256, 16
    ids, h, Wr, lut = _layer(31, V, D, N, 8)
    ids[:] = [0, V - 1, 5, 5, 0, V - 1, 5, 999]
    h[3] = h[2]
    got, st = _run(mole, ids, h, Wr, lut)
    assert st == 0
    ref, _ = oracle_mod.combine(ids, h, Wr, lut)
    assert_combine_close(got, ref)
    np.testing.assert_array_equal(got[2], got[3])
    # T == 0 is a no-op that returns OK
    out = torch.full((0, D), 7.0, device="cuda")
    mole.mole_lookup_combine(torch.empty(0, dtype=torch.int32, device="cuda"), dev(h[:0]), dev(Wr), dev(lut), out=out)
    assert mole.mole_check() == 0


@pytest.mark.parametrize("T", [40, 1500])
def test_combine_bad_ids_give_nan_rows_and_index_error(mole, oracle_mod, T):
    V, D, N = 300, 128, 16
    ids, h, Wr, lut = _layer(32, V, D, N, T)
    ids[[3, 17, 39]] = [-1, V, 2 ** 31 - 1]
    got, st = _run(mole, ids, h, Wr, lut)
    assert st == 5  # MOLE_ERR_INDEX
    assert mole.mole_check() == 0  # the error word was cleared
    ref, nbad = oracle_mod.combine(ids, h, Wr, lut)
    assert nbad == 3
    bad = np.zeros(T, bool)
    bad[[3, 17, 39]] = True
    assert np.isnan(got[bad]).all()
    assert_combine_close(got[~bad], ref[~bad])


def _hash_bf16(V, N, D):
    """Distinct normal bf16 values per (v, j, d) from an integer hash."""
    i = np.arange(V * N * D, dtype=np.uint64)
    x = (i * np.uint64(2654435761) + np.uint64(12345)) & np.uint64(0xFFFF)
    f = (x.astype(np.float64) / 65536.0 - 0.5).astype(np.float32) + np.float32(0.001)
    return inputs.f32_to_bf16_bits(f.reshape(V, N, D))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gather_is_bit_exact_under_one_hot_gates(mole, dtype):
    """h[t] = e_{d_t}, Wr[d_t, j_t] = 200: gate j_t is exactly 1 in fp32 and
    the rest exactly 0, so out[t] must be the addressed row, bit for bit."""
    V, N, D, T = 257, 16, 256, 64
    lut = _hash_bf16(V, N, D)
    if dtype == "f32":
        lut = inputs.bf16_bits_to_f32(lut)
    rng = np.random.default_rng(5)
    ids = rng.integers(0, V, T).astype(np.int32)
    ids[:2] = [0, V - 1]
    outs = []
    for t in range(T):
        d_t, j_t = (7 * t) % D, (5 * t + 3) % N
        h = np.zeros((1, D), np.float32)
        h[0, d_t] = 1.0
        Wr = np.zeros((D, N), np.float32)
        Wr[d_t, j_t] = 200.0
        if dtype == "bf16":
            h, Wr = inputs.f32_to_bf16_bits(h), inputs.f32_to_bf16_bits(Wr)
        got, st = _run(mole, ids[t:t + 1], h, Wr, lut)
        assert st == 0
        outs.append((got[0], as_f64(lut[ids[t], j_t]).astype(np.float32)))
    for got, want in outs:
        np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# Full-size layers (the model shapes), checked on sampled tokens
# ---------------------------------------------------------------------------

FULL = [
    ("160m", 1, "zipf"), ("160m", 8, "zipf"), ("160m", 64, "zipf"),
    ("410m", 1, "zipf"), ("410m", 32, "zipf"), ("410m", 256, "zipf"),
    ("1b", 4096, "zipf"), ("1b", 4096, "uniform"), ("1b", 16384, "zipf"), ("1b", 16384, "uniform"),
]


@pytest.mark.parametrize("shape_name,T,kind", FULL)
def test_combine_full_size_sampled(mole, oracle_mod, shape_name, T, kind):
    shape = inputs.SHAPES[shape_name]
    V, D, N = shape.V, shape.D, shape.N
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed)
    lut = (torch.randn((V, N, D), generator=g, device="cuda", dtype=torch.float32) * 0.02).to(torch.bfloat16)
    rng = np.random.default_rng(shape.seed + T)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    ids[0], ids[-1] = 0, V - 1
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    out = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), lut)
    assert mole.mole_check() == 0
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 62)]))
    s_ids = ids[sample]
    uniq, inv = np.unique(s_ids, return_inverse=True)
    rows = host_bits(lut[torch.from_numpy(uniq.astype(np.int64)).cuda()])
    ref, _ = oracle_mod.combine(inv.astype(np.int32), h[sample], Wr, rows)
    got = out[torch.from_numpy(sample).cuda()].cpu().numpy()
    assert_combine_close(got, ref)
    # every output row is finite
    assert torch.isfinite(out).all().item()
    del lut, out
    torch.cuda.empty_cache()
