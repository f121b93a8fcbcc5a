"""Parity of the NF3 path (CUDA, through the C ABI) against the oracle: codes
and scales bit-exact, the fused dequant-gather-combine within 1e-5 per token.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
实验结果: the table keeps its quality when stored at 3 bits (e.g. NF3).
"""
import numpy as np
import pytest
import torch

from helpers import assert_combine_close, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _special_blocks(lut):
    """Overwrite a few blocks with edge cases: zeros, tiny values, values past
    the fp16 range (scale saturates), exact level multiples, one huge outlier."""
    f = inputs.bf16_bits_to_f32(lut).copy()
    V, N, D = f.shape
    f[0, 0, 0:64] = 0.0
    f[0, 0, 64:128] = np.float32(1e-30)
    if D >= 192:
        f[0, 0, 128:192] = np.linspace(-7e4, 7e4, 64, dtype=np.float32)
    f[1, 0, :64] = np.float32(3.0) * np.array([-1, -0.535, -0.247, 0, 0.1833, 0.382, 0.623, 1.0] * 8, np.float32)
    if N >= 2:
        f[1, 1, :64] = np.float32(1e-3)
        f[1, 1, 5] = np.float32(5.0)
    return inputs.f32_to_bf16_bits(f)


@pytest.mark.parametrize("V,N,D", [(64, 16, 256), (33, 5, 128), (7, 1, 64), (300, 16, 2048)])
def test_quantize_bit_exact(mole, oracle_mod, V, N, D):
    rng = np.random.default_rng(V * N + D)
    lut = _special_blocks(inputs.normal(rng, (V, N, D), 0.02, "bf16"))
    codes, scales = mole.mole_quantize_lut_nf3(dev(lut))
    ref_codes, ref_scales = oracle_mod.quantize_nf3(lut)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(host_bits(scales), ref_scales)


def _boundary_blocks(oracle_mod, n_blocks, seed):
    """Blocks whose elements sit on both sides of the decision boundaries:
    element 0 is the block's absmax A (a bf16 value inside the fp16 range, so
    the scale is A itself), the others the bf16 values nearest to m_k * A for
    each midpoint m_k -- the two neighbours and one more on each side -- so
    x / s lands within a few fp32 ulps of a midpoint, where a quantiser that
    does not compare exactly as the division rule would pick the other code."""
    rng = np.random.default_rng(seed)
    mids = oracle_mod.nf3_midpoints().astype(np.float64)
    blocks = np.zeros((n_blocks, 64), dtype=np.float32)
    for b in range(n_blocks):
        A = np.float32(inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(
            np.array([rng.choice([1.0, -1.0]) * np.exp(rng.uniform(np.log(1e-4), np.log(6e4)))], np.float32)))[0])
        vals = [A]
        for m in mids:
            target = np.float32(m * abs(A))
            u = int(inputs.f32_to_bf16_bits(np.array([target], np.float32))[0])
            for du in (-2, -1, 0, 1, 2):  # bf16 neighbours by bit pattern (same sign)
                bits = np.array([(u + du) & 0xffff], np.uint16)
                vals.append(float(inputs.bf16_bits_to_f32(bits)[0]))
        vals = [v for v in vals if abs(v) <= abs(A)]
        blocks[b, :len(vals[:64])] = vals[:64]
    return inputs.f32_to_bf16_bits(blocks)


def test_quantize_bit_exact_at_the_decision_boundaries(mole, oracle_mod):
    lut = _boundary_blocks(oracle_mod, 4096, 11).reshape(64, 16, 4 * 64)
    codes, scales = mole.mole_quantize_lut_nf3(dev(lut))
    ref_codes, ref_scales = oracle_mod.quantize_nf3(lut)
    np.testing.assert_array_equal(host_bits(scales), ref_scales)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)


@pytest.mark.parametrize("V,N,D,T,dtype", [
    (300, 16, 2048, 300, "bf16"), (100, 16, 128, 77, "bf16"), (50, 5, 64, 19, "bf16"),
    (64, 24, 256, 40, "bf16"), (80, 8, 192, 33, "f32"),
    (200, 16, 256, 1500, "bf16"), (300, 8, 2048, 1100, "bf16"),  # router + gather kernels
    (100, 5, 128, 1200, "bf16"),  # N*D/64 not a multiple of 8: fused kernel
])
def test_combine_nf3_matches_oracle(mole, oracle_mod, V, N, D, T, dtype):
    rng = np.random.default_rng(T + D)
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, dtype)
    h = inputs.normal(rng, (T, D), 1.0, dtype)
    ids = inputs.zipf_ids(rng, T, V)
    ids[0], ids[-1] = 0, V - 1
    codes, scales = oracle_mod.quantize_nf3(lut)  # the oracle's codes are the input here
    out = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), dev(codes),
                                       dev(scales).view(torch.float16))
    assert mole.mole_check() == 0
    ref, _ = oracle_mod.combine_nf3(ids, h, Wr, codes, scales)
    assert_combine_close(out.cpu().numpy(), ref)


@pytest.mark.parametrize("T", [20, 1200])
def test_combine_nf3_bad_ids(mole, oracle_mod, T):
    V, N, D = 40, 16, 128
    rng = np.random.default_rng(3)
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    ids = rng.integers(0, V, T).astype(np.int32)
    ids[[2, 9]] = [-5, V]
    codes, scales = oracle_mod.quantize_nf3(lut)
    out = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), dev(codes), dev(scales).view(torch.float16))
    assert mole.mole_check() == 5
    got = out.cpu().numpy()
    assert np.isnan(got[[2, 9]]).all()
    ref, nbad = oracle_mod.combine_nf3(ids, h, Wr, codes, scales)
    ok = np.ones(T, bool)
    ok[[2, 9]] = False
    assert_combine_close(got[ok], ref[ok])


@pytest.mark.parametrize("T,kind", [(1, "zipf"), (64, "zipf"), (4096, "zipf"), (16384, "zipf"), (16384, "uniform")])
def test_nf3_full_size_sampled(mole, oracle_mod, T, kind):
    """1B-shaped layer: quantise the full [50304, 16, 2048] table on the GPU,
    check sampled code blocks bit-exactly and sampled tokens of the fused
    combine against the oracle on the same codes."""
    shape = inputs.SHAPES["1b_nf3"]
    V, D, N = shape.V, shape.D, shape.N
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed)
    lut = (torch.randn((V, N, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    codes, scales = mole.mole_quantize_lut_nf3(lut)
    rng = np.random.default_rng(shape.seed + T)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    ids[0], ids[-1] = 0, V - 1
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    out = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), codes, scales)
    assert mole.mole_check() == 0
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 46)]))
    uniq, inv = np.unique(ids[sample], return_inverse=True)
    sel = torch.from_numpy(uniq.astype(np.int64)).cuda()
    rows = host_bits(lut[sel])
    # codes of the sampled rows are bit-exact
    ref_codes, ref_scales = oracle_mod.quantize_nf3(rows)
    np.testing.assert_array_equal(codes[sel].cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(host_bits(scales[sel]), ref_scales)
    ref, _ = oracle_mod.combine_nf3(inv.astype(np.int32), h[sample], Wr, ref_codes, ref_scales)
    got = out[torch.from_numpy(sample).cuda()].cpu().numpy()
    assert_combine_close(got, ref)
    del lut, codes, scales, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("V,N,D,T,kind", [
    (200, 16, 256, 1500, "zipf"), (300, 8, 2048, 1100, "uniform"), (50, 16, 128, 3000, "zipf"),
    (100, 13, 512, 1200, "zipf"),   # padded expert count (13 * 8 blocks = 104, a multiple of 8)
    (100, 5, 128, 1200, "zipf"),    # N * D/64 not a multiple of 8: ungrouped kernels
    (64, 16, 256, 300, "zipf"),     # below the grouping threshold: ungrouped kernels
    (3000, 16, 128, 15000, "zipf"),  # a prefill size: tensor-core router + grouped gather
    (2000, 8, 128, 40000, "zipf"),   # too many tokens per SM for the shares: mma.sync router + grouped gather
])
def test_combine_nf3_groups_matches_oracle_and_ungrouped(mole, oracle_mod, V, N, D, T, kind):
    rng = np.random.default_rng(T + D + N)
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    ids[0], ids[-1] = 0, V - 1
    codes, scales = oracle_mod.quantize_nf3(lut)
    c, s = dev(codes), dev(scales).view(torch.float16)
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    got = mole.mole_lookup_combine_nf3_groups(dev(ids), groups, dev(h), dev(Wr), c, s)
    assert mole.mole_check() == 0
    plain = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), c, s)
    assert mole.mole_check() == 0
    assert torch.equal(got, plain)
    ref, _ = oracle_mod.combine_nf3(ids, h, Wr, codes, scales)
    assert_combine_close(got.cpu().numpy(), ref)


def test_combine_nf3_groups_bad_ids(mole, oracle_mod):
    V, N, D, T = 40, 16, 128, 1500
    rng = np.random.default_rng(4)
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    ids = rng.integers(0, V, T).astype(np.int32)
    ids[[2, 900]] = [-5, V]
    codes, scales = oracle_mod.quantize_nf3(lut)
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    out = mole.mole_lookup_combine_nf3_groups(dev(ids), groups, dev(h), dev(Wr), dev(codes),
                                              dev(scales).view(torch.float16))
    assert mole.mole_check() == 5
    got = out.cpu().numpy()
    assert np.isnan(got[[2, 900]]).all()
    ref, _ = oracle_mod.combine_nf3(ids, h, Wr, codes, scales)
    ok = np.ones(T, bool)
    ok[[2, 900]] = False
    assert_combine_close(got[ok], ref[ok])


@pytest.mark.parametrize("kind", ["zipf", "uniform"])
def test_nf3_groups_full_size(mole, oracle_mod, kind):
    shape = inputs.SHAPES["1b_nf3"]
    V, D, N, T = shape.V, shape.D, shape.N, 16384
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 7)
    lut = (torch.randn((V, N, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    codes, scales = mole.mole_quantize_lut_nf3(lut)
    rng = np.random.default_rng(shape.seed + 11)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    got = mole.mole_lookup_combine_nf3_groups(dev(ids), groups, dev(h), dev(Wr), codes, scales)
    assert mole.mole_check() == 0
    plain = mole.mole_lookup_combine_nf3(dev(ids), dev(h), dev(Wr), codes, scales)
    assert mole.mole_check() == 0
    assert torch.equal(got, plain)
    sample = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 30)]))
    uniq, inv = np.unique(ids[sample], return_inverse=True)
    sel = torch.from_numpy(uniq.astype(np.int64)).cuda()
    ref, _ = oracle_mod.combine_nf3(inv.astype(np.int32), h[sample], Wr, codes[sel].cpu().numpy(),
                                    host_bits(scales[sel]))
    assert_combine_close(got[torch.from_numpy(sample).cuda()].cpu().numpy(), ref)
    del lut, codes, scales, got, plain
    torch.cuda.empty_cache()
