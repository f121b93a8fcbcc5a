"""mole_prefetch_rows, the cross-layer row prefetch of a step (MoLE page,
推理阶段 / 复杂度分析: every layer indexes its table with the step's token ids,
so all layers' rows are known before the first layer runs).  A prefetch is a
hint: the layers' combines after it give the same bits as without it, bad
ids are skipped without a device error, and NF3 tables prefetch as their
code and scale arrays."""
import numpy as np
import pytest
import torch

from helpers import dev
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _layers(L, V, N, D, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    luts = [(torch.randn((V, N, D), generator=g, device="cuda") * 0.02).to(torch.bfloat16) for _ in range(L)]
    routers = [(torch.randn((D, N), generator=g, device="cuda") * 0.02).to(torch.bfloat16) for _ in range(L)]
    return g, luts, routers


@pytest.mark.parametrize("T", [1, 8, 64, 300])
def test_prefetch_then_layers_equal_layers_alone(mole, T):
    V, N, D, L = 5000, 16, 256, 6
    g, luts, routers = _layers(L, V, N, D, 600 + T)
    ids = dev(inputs.draw_ids(np.random.default_rng(T), T, V, "zipf"))
    hs = [torch.randn((T, D), generator=g, device="cuda").to(torch.bfloat16) for _ in range(L)]
    plain = [mole.mole_lookup_combine(ids, hs[l], routers[l], luts[l]) for l in range(L)]
    mole.mole_prefetch_rows(ids, luts)
    pref = [mole.mole_lookup_combine(ids, hs[l], routers[l], luts[l]) for l in range(L)]
    assert mole.mole_check() == 0
    for a, b in zip(plain, pref):
        assert torch.equal(a, b)


def test_prefetch_nf3_tables_and_bad_ids(mole):
    V, N, D, L, T = 3000, 8, 128, 3, 40
    g, luts, routers = _layers(L, V, N, D, 77)
    q = [mole.mole_quantize_lut_nf3(x) for x in luts]
    ids_np = inputs.draw_ids(np.random.default_rng(5), T, V, "uniform")
    ids_np[[0, 7]] = [-3, V + 11]  # skipped by the prefetch
    ids = dev(ids_np)
    h = torch.randn((T, D), generator=g, device="cuda").to(torch.bfloat16)
    good = dev(np.where((ids_np >= 0) & (ids_np < V), ids_np, 0).astype(np.int32))
    ref = mole.mole_lookup_combine_nf3(good, h, routers[0], *q[0])
    assert mole.mole_check() == 0
    mole.mole_prefetch_rows(ids, [c for c, _ in q])
    mole.mole_prefetch_rows(ids, [s for _, s in q])
    assert mole.mole_check() == 0  # the prefetch itself reports nothing
    out = mole.mole_lookup_combine_nf3(good, h, routers[0], *q[0])
    assert mole.mole_check() == 0
    assert torch.equal(out, ref)


def test_prefetch_of_a_full_size_layer_stack(mole):
    """160M-shaped decode step: 12 layer tables [50304, 16, 768] bf16, 64 Zipf
    tokens; then the 12 combines, equal to those without the prefetch."""
    shape = inputs.SHAPES["160m"]
    V, N, D, L, T = shape.V, shape.N, shape.D, shape.layers, 64
    g, luts, routers = _layers(L, V, N, D, shape.seed)
    ids = dev(inputs.draw_ids(np.random.default_rng(shape.seed), T, V, "zipf"))
    hs = [torch.randn((T, D), generator=g, device="cuda").to(torch.bfloat16) for _ in range(L)]
    plain = [mole.mole_lookup_combine(ids, hs[l], routers[l], luts[l]) for l in range(L)]
    torch.cuda.synchronize()
    mole.mole_prefetch_rows(ids, luts)
    pref = [mole.mole_lookup_combine(ids, hs[l], routers[l], luts[l]) for l in range(L)]
    assert mole.mole_check() == 0
    for a, b in zip(plain, pref):
        assert torch.equal(a, b)
    del luts
    torch.cuda.empty_cache()
