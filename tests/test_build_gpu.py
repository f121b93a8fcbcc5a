"""Parity of mole_build_lut (CUDA, through the C ABI) against the fp64 oracle.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
推理阶段: LUT[v, j, :] = f_j(E[v]).  Two kinds of checks:
  - bit-exact on dyadic data where every sum is exact in fp32 (identity / ReLU),
    so any mismatch is an indexing or pipeline fault, not rounding;
  - on N(0, 0.02) data with GELU-type activations: 2 bf16 ulps of the fp64
    reference, the ulp taken at max(|ref|, 2^-8 rms(row)), plus the oracle's
    allowance for hidden activations whose bf16 rounding is ambiguous, and row
    relative L2 <= 2^-8 (see helpers.py).
The oracle rounds the hidden activation to bf16 where the bf16 build does.
"""
import numpy as np
import pytest
import torch

from helpers import as_f64, assert_build_close, assert_combine_close, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _weights(V, D, N, Dr, dtype, seed):
    shape = inputs.small(V, D, N, Dr, dtype, seed)
    return inputs.expert_weights(shape)


def _check(lut_gpu, ref, allow=None):
    import os
    return assert_build_close(host_bits(lut_gpu), ref, allow, label=os.environ.get("PYTEST_CURRENT_TEST", ""))


def _dyadic(rng, shape):
    """Values in {-2, -1, 0, 1, 2} / 8 (exact in bf16 and fp32)."""
    return (rng.integers(-2, 3, size=shape) / 8.0).astype(np.float32)


@pytest.mark.parametrize("V,D,N,Dr,act", [
    (300, 128, 3, 256, "identity"),  # ragged M; GEMM2 N = 128 < one 256-wide tile
    (1000, 256, 2, 512, "relu"),
    (129, 64, 4, 192, "relu"),       # partial N tile in GEMM1 (192 of 256)
    (256, 320, 2, 64, "identity"),   # one k-block in GEMM2; N = 320 -> 2 tiles
    (200, 192, 2, 128, "relu"),
    (513, 448, 3, 320, "identity"),  # 5 k-blocks (ring wraps), N tails in both GEMMs
    (64, 512, 1, 512, "relu"),
])
def test_build_tensor_core_bit_exact_on_dyadic_data(mole, oracle_mod, V, D, N, Dr, act):
    """With entries in {0, +-1/8, +-1/4}, D, Dr <= 512, every product and every
    partial sum of both contractions is exact in fp32 (<= 21 significant bits),
    so the only roundings are the bf16 roundings of H and of the output, applied
    to the same exact values on both sides: the table must match bit for bit."""
    rng = np.random.default_rng(V + D + N + Dr)
    E = inputs.f32_to_bf16_bits(_dyadic(rng, (V, D)))
    W1 = inputs.f32_to_bf16_bits(_dyadic(rng, (N, D, Dr)))
    W2 = inputs.f32_to_bf16_bits(_dyadic(rng, (N, Dr, D)))
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act=act)
    assert mole.mole_check() == 0
    # the bf16 table is the exact value rounded to bf16 (ties to even)
    ref = oracle_mod.round_bf16_array(oracle_mod.build_lut(E, W1, W2, act_name=act, round_h=True))
    got = as_f64(host_bits(lut))
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} of {got.size} elements differ, first at {bad[:5].tolist()}"


@pytest.mark.parametrize("V,D,N,Dr,act", [
    (1000, 256, 2, 1024, "gelu"),
    (300, 128, 3, 2048, "silu"),
    (200, 192, 2, 1024, "gelu_tanh"),
    (257, 64, 2, 1536, "gelu"),
])
def test_build_bf16_tensor_core_matches_oracle(mole, oracle_mod, V, D, N, Dr, act):
    _, E, W1, W2 = _weights(V, D, N, Dr, "bf16", V + D + Dr)
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act=act)
    assert mole.mole_check() == 0
    ref, allow, _ = oracle_mod.build_lut(E, W1, W2, act_name=act, round_h=True, with_allowance=True)
    _check(lut, ref, allow)


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
    V, D, N, Dr = 97, 48, 3, 1040
    _, E, W1, W2 = _weights(V, D, N, Dr, "bf16", 21)
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2))
    ref, allow, _ = oracle_mod.build_lut(E, W1, W2, act_name="gelu", round_h=True, with_allowance=True)
    _check(lut, ref, allow)


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
    ref, allow, _ = oracle_mod.build_lut(E_rows, host_bits(W1), host_bits(W2), act_name="gelu", round_h=True,
                                         with_allowance=True)
    _check(lut[torch.from_numpy(rows).cuda()], ref, allow)
    del E, W1, W2, lut
    torch.cuda.empty_cache()


@pytest.mark.parametrize("V,D,N,Dr,act,per_launch", [
    (300, 128, 3, 256, "gelu", 0),     # ragged M; 2 blocks per row
    (1000, 256, 2, 512, "gelu", 1),    # one expert per launch
    (129, 64, 4, 192, "relu", 0),      # one block per row, partial N tile in GEMM1
    (513, 448, 3, 320, "gelu", 2),     # N tails; 7 blocks per row
    (256, 512, 2, 128, "silu", 0),
])
def test_build_nf3_equals_build_then_quantize(mole, oracle_mod, V, D, N, Dr, act, per_launch):
    """The quantising epilogue gives the codes and scales of mole_build_lut
    followed by mole_quantize_lut_nf3, bit for bit; the table it stands for
    still meets the build tolerance against the oracle once dequantised."""
    _, E, W1, W2 = _weights(V, D, N, Dr, "bf16", 40 + V)
    ws = torch.empty(mole.mole_build_lut_workspace(V, D, N, Dr, torch.bfloat16, per_launch), dtype=torch.uint8,
                     device="cuda")
    codes, scales = mole.mole_build_lut_nf3(dev(E), dev(W1), dev(W2), act, workspace=ws)
    assert mole.mole_check() == 0
    lut = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act)
    c2, s2 = mole.mole_quantize_lut_nf3(lut)
    assert mole.mole_check() == 0
    assert torch.equal(codes, c2)
    assert torch.equal(scales.view(torch.int16), s2.view(torch.int16))
    # the codes are also the oracle quantiser's of that table
    ref_codes, ref_scales = oracle_mod.quantize_nf3(host_bits(lut))
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(host_bits(scales), ref_scales)


def test_build_nf3_full_size_rows(mole, oracle_mod):
    """410M-shaped layer (V = 50304, D = 1024, N = 16, Dr = 4096): the fused
    NF3 build equals build + quantise on sampled rows, bit for bit."""
    shape = inputs.SHAPES["410m"]
    V, D, N, Dr = shape.V, shape.D, shape.N, shape.Dr
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 3)
    E = (torch.randn((V, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    W1 = (torch.randn((N, D, Dr), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((N, Dr, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    codes, scales = mole.mole_build_lut_nf3(E, W1, W2)
    assert mole.mole_check() == 0
    rows = torch.tensor([0, 1, 255, 256, 257, 12345, V - 2, V - 1], device="cuda")
    lut = mole.mole_build_lut(E, W1, W2)
    c2, s2 = mole.mole_quantize_lut_nf3(lut[rows].contiguous())
    assert torch.equal(codes[rows], c2)
    assert torch.equal(scales[rows].view(torch.int16), s2.view(torch.int16))
    del E, W1, W2, codes, scales, lut
    torch.cuda.empty_cache()
