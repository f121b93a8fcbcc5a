"""Parity of mole_build_lut (CUDA, through the C ABI) against the fp64 oracle.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
推理阶段: LUT[v, j, :] = f_j(E[v]).  Tolerance: 2 bf16 ulps of the fp64 reference
(ulp at max(|ref|, 2^-8 rms of the row)); the oracle rounds the hidden
activation to bf16 where the bf16 build does.
"""
import numpy as np
import pytest
import torch

from helpers import BUILD_MAX_ULPS, as_f64, assert_combine_close, build_ulps, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _weights(V, D, N, Dr, dtype, seed):
    shape = inputs.small(V, D, N, Dr, dtype, seed)
    return inputs.expert_weights(shape)


def _check(lut_gpu, ref):
    ulps = build_ulps(host_bits(lut_gpu), ref)
    assert ulps.max() <= BUILD_MAX_ULPS, f"max {ulps.max():.2f} bf16 ulps"
    return ulps


@pytest.mark.parametrize("V,D,N,Dr,act", [
    (300, 128, 3, 256, "gelu"),      # ragged M, GEMM2 N=128 < one 256-wide tile
    (1000, 256, 2, 512, "gelu"),
    (129, 64, 4, 192, "relu"),       # partial N tile in GEMM1 (192 of 256)
    (256, 320, 2, 64, "identity"),   # K=64 single k-block, N=320 -> 2 tiles
    (200, 192, 2, 128, "silu"),
    (200, 128, 2, 128, "gelu_tanh"),
])
def test_build_bf16_tensor_core_matches_oracle(mole, oracle_mod, V, D, N, Dr, act):
    _, E, W1, W2 = _weights(V, D, N, Dr, "bf16", V + D + Dr)
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act=act)
    assert mole.mole_check() == 0
    ref = oracle_mod.build_lut(E, W1, W2, act_name=act, round_h=True)
    _check(lut, ref)


def test_build_workspace_groups_give_the_same_table(mole):
    V, D, N, Dr = 333, 128, 5, 256
    _, E, W1, W2 = _weights(V, D, N, Dr, "bf16", 9)
    a = mole.mole_build_lut(dev(E), dev(W1), dev(W2))
    for per_launch in (1, 2):
        ws = torch.empty(mole.mole_build_lut_workspace(V, D, N, Dr, torch.bfloat16, per_launch),
                         dtype=torch.uint8, device="cuda")
        b = mole.mole_build_lut(dev(E), dev(W1), dev(W2), workspace=ws)
        assert torch.equal(a, b)
    ws = torch.empty(mole.mole_build_lut_workspace(V, D, N, Dr, torch.bfloat16, 1) - 2, dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(mole.MoleError):
        mole.mole_build_lut(dev(E), dev(W1), dev(W2), workspace=ws)


def test_build_f32_tiny_layer_exhaustive(mole, oracle_mod):
    """The tiny fp32 layer: V=512, D=64, N=4, Dr=256, every element."""
    shape = inputs.SHAPES["tiny"]
    rng, E, W1, W2 = inputs.expert_weights(shape)
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2))
    assert mole.mole_check() == 0
    ref = oracle_mod.build_lut(E, W1, W2, act_name="gelu", round_h=False)
    _check(lut, ref)
    # and the combine over that table, against the oracle on the same table bytes
    Wr, ids, h = inputs.router_and_batch(rng, shape, T=256)
    out = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), lut)
    ref_out, _ = oracle_mod.combine(ids, h, Wr, lut.cpu().numpy())
    assert_combine_close(out.cpu().numpy(), ref_out)


def test_build_bf16_cuda_core_path(mole, oracle_mod):
    # D not a multiple of 64 -> the CUDA-core path
    V, D, N, Dr = 97, 48, 3, 80
    _, E, W1, W2 = _weights(V, D, N, Dr, "bf16", 21)
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2))
    ref = oracle_mod.build_lut(E, W1, W2, act_name="gelu", round_h=True)
    _check(lut, ref)


def test_reparameterisation_invariant_on_gpu(mole, oracle_mod):
    """Combining the GPU-built table equals evaluating the experts directly on
    the embedding rows (fp64, no rounding) and mixing with the same gates,
    within the bf16 storage error of the table."""
    V, D, N, Dr, T = 256, 128, 4, 256, 64
    shape = inputs.small(V, D, N, Dr, "bf16", 77)
    rng, E, W1, W2 = inputs.expert_weights(shape)
    Wr, ids, h = inputs.router_and_batch(rng, shape, T)
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2))
    out = mole.mole_lookup_combine(dev(ids), dev(h), dev(Wr), lut).cpu().numpy()
    direct = oracle_mod.build_lut(E, W1, W2, act_name="gelu", round_h=False, rows=ids)
    _, gates, _ = oracle_mod.combine(ids, h, Wr, host_bits(lut), return_gates=True)
    mix = np.einsum("tj,tjd->td", gates, direct)
    rel = np.linalg.norm(out - mix, axis=1) / np.linalg.norm(mix, axis=1)
    assert rel.max() < 2e-2  # bf16 table + bf16 hidden activation


@pytest.mark.parametrize("shape_name,n_rows", [("410m", 64), ("1b", 12), ("160m", 32)])
def test_build_full_size_sampled_rows(mole, oracle_mod, shape_name, n_rows):
    shape = inputs.SHAPES[shape_name]
    V, D, N, Dr = shape.V, shape.D, shape.N, shape.Dr
    # weights drawn on the device (seeded); the sampled rows are copied back
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed)
    E = (torch.randn((V, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    W1 = (torch.randn((N, D, Dr), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((N, Dr, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    lut = mole.mole_build_lut(E, W1, W2)
    assert mole.mole_check() == 0
    rng = np.random.default_rng(shape.seed)
    edges = [0, 1, 127, 128, 129, 255, 256, V - 129, V - 128, V - 2, V - 1]
    rows = np.unique(np.concatenate([edges, rng.integers(0, V, max(0, n_rows - len(edges)))]))
    E_rows = host_bits(E[torch.from_numpy(rows).cuda()])
    ref = oracle_mod.build_lut(E_rows, host_bits(W1), host_bits(W2), act_name="gelu", round_h=True)
    _check(lut[torch.from_numpy(rows).cuda()], ref)
    del E, W1, W2, lut
    torch.cuda.empty_cache()
