"""FFN block (shared expert + routed-expert mixture + residual) against the
fp64 oracle.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
训练阶段 / 推理阶段: at inference the shared experts stay dense FFNs on the
previous layer's output and only the routed experts become the table.

Tolerance: per token, ||max(|gpu - ref| - allowance, 0)||_2 / ||ref||_2 <= 1e-5
(fp32 outputs; `allowance` covers hidden activations whose bf16 rounding is
ambiguous between the fp32 GPU sum and the fp64 oracle sum, as for the build).
"""
import numpy as np
import pytest
import torch

from helpers import dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu

RTOL = 1e-5


def assert_ffn_close(got, ref, allow):
    err = np.maximum(np.abs(got.astype(np.float64) - ref) - allow, 0.0)
    rel = np.linalg.norm(err, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert rel.max() <= RTOL, f"max rel {rel.max():.3e} at token {int(np.argmax(rel))}"


def _block(seed, T, D, Ds, N, V, kind="zipf", std_w=0.02):
    rng = np.random.default_rng(seed)
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    lut = inputs.normal(rng, (V, N, D), 0.02, "bf16")
    W1s = inputs.normal(rng, (D, Ds), std_w, "bf16")
    W2s = inputs.normal(rng, (Ds, D), std_w, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    res = rng.standard_normal((T, D)).astype(np.float32)
    return ids, h, Wr, lut, W1s, W2s, res


@pytest.mark.parametrize("T,D,Ds", [(300, 128, 256), (1500, 256, 512), (129, 64, 64), (257, 192, 320)])
def test_shared_ffn_matches_oracle(mole, oracle_mod, T, D, Ds):
    ids, h, Wr, lut, W1s, W2s, res = _block(800 + T + D, T, D, Ds, 4, 50)
    add = np.random.default_rng(T).standard_normal((T, D)).astype(np.float32)
    out = mole.mole_shared_ffn(dev(h), dev(W1s), dev(W2s), "gelu", add=dev(add), residual=dev(res))
    assert mole.mole_check() == 0
    shared, allow, _ = oracle_mod.build_lut(h, W1s.reshape(1, D, Ds), W2s.reshape(1, Ds, D), "gelu",
                                            with_allowance=True)
    ref = shared[:, 0, :] + add + res
    assert_ffn_close(out.cpu().numpy(), ref, allow[:, 0, :])
    # without the added terms
    out2 = mole.mole_shared_ffn(dev(h), dev(W1s), dev(W2s), "gelu")
    assert_ffn_close(out2.cpu().numpy(), shared[:, 0, :], allow[:, 0, :])


@pytest.mark.parametrize("T,D,Ds,N,V,kind", [
    (1500, 256, 512, 16, 400, "zipf"),   # grouped combine kernels
    (2000, 128, 256, 8, 900, "uniform"),
    (300, 128, 256, 16, 200, "zipf"),    # below the grouping threshold
])
def test_ffn_block_matches_oracle(mole, oracle_mod, T, D, Ds, N, V, kind):
    ids, h, Wr, lut, W1s, W2s, res = _block(900 + T + N, T, D, Ds, N, V, kind)
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    out = mole.mole_ffn_block(dev(ids), groups, dev(h), dev(Wr), dev(lut), dev(W1s), dev(W2s), "gelu",
                              residual=dev(res))
    assert mole.mole_check() == 0
    ref, allow, nbad = oracle_mod.ffn_block(ids, h, Wr, lut, W1s, W2s, "gelu", res)
    assert nbad == 0
    assert_ffn_close(out.cpu().numpy(), ref, allow)
    # in place on the residual stream: the same result
    r = dev(res)
    out2 = mole.mole_ffn_block(dev(ids), groups, dev(h), dev(Wr), dev(lut), dev(W1s), dev(W2s), "gelu",
                               residual=r, out=r)
    assert mole.mole_check() == 0
    assert torch.equal(out2, out)


def test_ffn_block_bad_ids(mole, oracle_mod):
    T, D, Ds, N, V = 1200, 128, 128, 16, 300
    ids, h, Wr, lut, W1s, W2s, res = _block(951, T, D, Ds, N, V)
    ids[[4, 700]] = [-3, V]
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    out = mole.mole_ffn_block(dev(ids), groups, dev(h), dev(Wr), dev(lut), dev(W1s), dev(W2s), "gelu",
                              residual=dev(res))
    assert mole.mole_check() == 5
    got = out.cpu().numpy()
    bad = np.zeros(T, bool)
    bad[[4, 700]] = True
    assert np.isnan(got[bad]).all()
    ref, allow, nbad = oracle_mod.ffn_block(ids, h, Wr, lut, W1s, W2s, "gelu", res)
    assert nbad == 2
    assert_ffn_close(got[~bad], ref[~bad], allow[~bad])


def test_ffn_block_full_size_sampled(mole, oracle_mod):
    """1B-shaped layer: D = 2048, one shared expert of width 8192, table
    [50304, 16, 2048], 4096 Zipf tokens; sampled tokens against the oracle."""
    shape = inputs.SHAPES["1b"]
    V, D, N, Ds, T = shape.V, shape.D, shape.N, shape.Dr, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 21)
    lut = (torch.randn((V, N, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    rng = np.random.default_rng(shape.seed + 23)
    Wr = inputs.normal(rng, (D, N), 0.02, "bf16")
    W1s = inputs.normal(rng, (D, Ds), 0.02, "bf16")
    W2s = inputs.normal(rng, (Ds, D), 0.02, "bf16")
    ids = inputs.draw_ids(rng, T, V, "zipf")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    res = rng.standard_normal((T, D)).astype(np.float32)
    groups = mole.mole_token_groups_build(dev(ids), V, N)
    out = mole.mole_ffn_block(dev(ids), groups, dev(h), dev(Wr), lut, dev(W1s), dev(W2s), "gelu", residual=dev(res))
    assert mole.mole_check() == 0
    sample = np.unique(np.concatenate([[0, 127, 128, 255, 256, T - 1], rng.integers(0, T, 18)]))
    uniq, inv = np.unique(ids[sample], return_inverse=True)
    rows = host_bits(lut[torch.from_numpy(uniq.astype(np.int64)).cuda()])
    ref, allow, _ = oracle_mod.ffn_block(inv.astype(np.int32), h[sample], Wr, rows, W1s, W2s, "gelu", res[sample])
    assert_ffn_close(out[torch.from_numpy(sample).cuda()].cpu().numpy(), ref, allow)
    del lut, out
    torch.cuda.empty_cache()
