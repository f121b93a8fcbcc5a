"""Training step of one MoLE layer (forward + backward) against the fp64 oracle.

MoLE page ("ICML 2025 Spotlight | 华为诺亚提出端侧大模型新架构MoLE...", zejuncao.github.io),
训练阶段: routed experts on the token's embedding row, all N active, mixed by
the router on the previous layer's output.

Forward: equal to the inference path (mole_build_lut, then
mole_lookup_combine on the same ids) -- the same kernels on the same rows; the
expert GEMM may take its single-CTA or CTA-pair form depending on the row
count, so the comparison allows fp32 rounding (2e-6 relative) -- and per
token within FWD_RTOL of the oracle's output on its bf16-rounded expert rows
(an expert row element that fp32 and fp64 round to neighbouring bf16 values
moves a token's output by about 2^-8 / sqrt(D) relative).
Backward: the oracle rounds where the device rounds (hidden activation,
expert rows, dL/dY and dL/dpre: the bf16 operands of the backward GEMMs), so
what remains is fp32 accumulation and the rare bf16 rounding of a value that
fp32 and fp64 put on different sides of a rounding boundary (one bf16 ulp of
that element).  Per gradient tensor ||gpu - ref||_2 / ||ref||_2 within
GRAD_RTOL (expert gradients) or ROUTER_RTOL (dh, dWr: fp32 arithmetic on the
same bf16 rows).
"""
import numpy as np
import pytest
import torch

import os

from helpers import ERR_DIAG, dev
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu

GRAD_RTOL = 1e-3
ROUTER_RTOL = 5e-4
FWD_RTOL = 4e-3


def _layer(seed, T, V, D, N, Dr, kind="zipf"):
    rng = np.random.default_rng(seed)
    E = inputs.normal(rng, (V, D), 0.5, "bf16")
    W1 = inputs.normal(rng, (N, D, Dr), 0.05, "bf16")
    W2 = inputs.normal(rng, (N, Dr, D), 0.05, "bf16")
    Wr = inputs.normal(rng, (D, N), 0.05, "bf16")
    h = inputs.normal(rng, (T, D), 1.0, "bf16")
    ids = inputs.draw_ids(rng, T, V, kind)
    dout = rng.standard_normal((T, D)).astype(np.float32)
    return ids, h, Wr, E, W1, W2, dout


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _grads(mole, ids, groups, h, Wr, E, W1, W2, dout, cache, U, act):
    T, D = h.shape
    V = E.shape[0]
    N, _, Dr = W1.shape
    z = lambda *s: torch.zeros(s, dtype=torch.float32, device="cuda")
    g = dict(dh=z(T, D), dWr=z(D, N), dE=z(V, D), dW1=z(N, D, Dr), dW2=z(N, Dr, D))
    mole.mole_train_backward(ids, groups, h, Wr, E, W1, W2, dout, cache, U, act, **g)
    return g


@pytest.mark.parametrize("T,V,D,N,Dr,act,kind", [
    (300, 400, 128, 4, 256, "gelu", "zipf"),    # below the grouping threshold (ungrouped combine)
    (1500, 500, 256, 16, 512, "gelu", "zipf"),  # grouped combine; ids repeat
    (1100, 3000, 128, 8, 192, "silu", "uniform"),
    (64, 40, 64, 2, 64, "relu", "uniform"),     # more tokens than ids
])
def test_train_step_matches_inference_and_oracle(mole, oracle_mod, T, V, D, N, Dr, act, kind):
    ids, h, Wr, E, W1, W2, dout = _layer(1000 + T + N, T, V, D, N, Dr, kind)
    dids, dh_, dWr_, dE_, dW1_, dW2_ = dev(ids), dev(h), dev(Wr), dev(E), dev(W1), dev(W2)
    groups = mole.mole_token_groups_build(dids, V, N)
    out, cache, U = mole.mole_train_forward(dids, groups, dh_, dWr_, dE_, dW1_, dW2_, act)
    assert mole.mole_check() == 0
    assert U == len(np.unique(ids))
    # forward = the inference path on a built table
    lut = mole.mole_build_lut(dE_, dW1_, dW2_, act)
    ref_out = mole.mole_lookup_combine(dids, dh_, dWr_, lut)
    assert mole.mole_check() == 0
    torch.testing.assert_close(out, ref_out, rtol=2e-6, atol=1e-8)
    # backward (and forward) against the oracle at the device's precision points
    g = _grads(mole, dids, groups, dh_, dWr_, dE_, dW1_, dW2_, dev(dout), cache, U, act)
    assert mole.mole_check() == 0
    ref_o, ref = oracle_mod.train_step(ids, h, Wr, E, W1, W2, act, dout, round_ops=True)
    here = os.environ.get("PYTEST_CURRENT_TEST", "").split("::")[-1]
    fwd = float((np.linalg.norm(out.cpu().numpy() - ref_o, axis=1) / np.linalg.norm(ref_o, axis=1)).max())
    ERR_DIAG.append((f"{here} out (max token rel L2)", fwd))
    assert fwd <= FWD_RTOL
    for name, tol in [("dh", ROUTER_RTOL), ("dWr", ROUTER_RTOL), ("dE", GRAD_RTOL), ("dW1", GRAD_RTOL),
                      ("dW2", GRAD_RTOL)]:
        got = g[name].cpu().numpy()
        assert np.isfinite(got).all(), name
        ERR_DIAG.append((f"{here} {name} (rel L2)", _rel(got, ref[name])))
        assert _rel(got, ref[name]) <= tol, (name, _rel(got, ref[name]))
    # dE touches only the batch's rows
    untouched = np.setdiff1d(np.arange(V), ids)
    assert not g["dE"][torch.from_numpy(untouched).cuda()].any()


def test_train_backward_accumulates_and_skips_absent_gradients(mole):
    T, V, D, N, Dr = 1200, 300, 128, 16, 128
    ids, h, Wr, E, W1, W2, dout = _layer(1101, T, V, D, N, Dr)
    dids, dh_, dWr_, dE_, dW1_, dW2_ = dev(ids), dev(h), dev(Wr), dev(E), dev(W1), dev(W2)
    groups = mole.mole_token_groups_build(dids, V, N)
    _, cache, U = mole.mole_train_forward(dids, groups, dh_, dWr_, dE_, dW1_, dW2_)
    once = _grads(mole, dids, groups, dh_, dWr_, dE_, dW1_, dW2_, dev(dout), cache, U, "gelu")
    twice = {k: v.clone() for k, v in once.items()}
    mole.mole_train_backward(dids, groups, dh_, dWr_, dE_, dW1_, dW2_, dev(dout), cache, U, "gelu", **twice)
    assert mole.mole_check() == 0
    # the backward is deterministic (no atomics): a second call adds exactly
    # the same values
    for k in once:
        assert torch.equal(twice[k], 2 * once[k]), k
    # only dW2 requested: the others stay untouched
    dW2 = torch.zeros_like(once["dW2"])
    mole.mole_train_backward(dids, groups, dh_, dWr_, dE_, dW1_, dW2_, dev(dout), cache, U, "gelu", dW2=dW2)
    assert mole.mole_check() == 0
    assert torch.equal(dW2, once["dW2"])


def test_train_bad_ids(mole, oracle_mod):
    T, V, D, N, Dr = 1100, 200, 128, 8, 128
    ids, h, Wr, E, W1, W2, dout = _layer(1102, T, V, D, N, Dr)
    bad = np.zeros(T, bool)
    bad[[3, 600]] = True
    ids_bad = ids.copy()
    ids_bad[[3, 600]] = [-1, V + 2]
    dids = dev(ids_bad)
    dh_, dWr_, dE_, dW1_, dW2_ = dev(h), dev(Wr), dev(E), dev(W1), dev(W2)
    groups = mole.mole_token_groups_build(dids, V, N)
    out, cache, U = mole.mole_train_forward(dids, groups, dh_, dWr_, dE_, dW1_, dW2_)
    assert mole.mole_check() == 5
    assert torch.isnan(out[torch.from_numpy(np.flatnonzero(bad)).cuda()]).all()
    g = _grads(mole, dids, groups, dh_, dWr_, dE_, dW1_, dW2_, dev(dout), cache, U, "gelu")
    assert mole.mole_check() == 0
    # the oracle on the good tokens only (a bad token contributes nothing)
    _, ref = oracle_mod.train_step(ids[~bad], h[~bad], Wr, E, W1, W2, "gelu", dout[~bad], round_ops=True)
    assert not g["dh"][torch.from_numpy(np.flatnonzero(bad)).cuda()].any()
    assert _rel(g["dh"].cpu().numpy()[~bad], ref["dh"]) <= ROUTER_RTOL
    for name in ("dE", "dW1", "dW2"):
        assert _rel(g[name].cpu().numpy(), ref[name]) <= GRAD_RTOL, name


def test_train_full_size_properties(mole):
    """1B-shaped layer (V = 50304, D = 2048, N = 16, Dr = 8192), 4096 Zipf
    tokens: the forward equals the inference path on the sampled tokens' table
    rows; the gradients are finite and dE touches only the batch's rows."""
    shape = inputs.SHAPES["1b"]
    V, D, N, Dr, T = shape.V, shape.D, shape.N, shape.Dr, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(shape.seed + 31)
    rnd = lambda *s, sd=0.02: (torch.randn(s, generator=g, device="cuda") * sd).to(torch.bfloat16)
    E, W1, W2, Wr, h = rnd(V, D), rnd(N, D, Dr), rnd(N, Dr, D), rnd(D, N), rnd(T, D, sd=1.0)
    rng = np.random.default_rng(shape.seed + 33)
    ids = inputs.draw_ids(rng, T, V, "zipf")
    dids = dev(ids)
    groups = mole.mole_token_groups_build(dids, V, N)
    out, cache, U = mole.mole_train_forward(dids, groups, h, Wr, E, W1, W2)
    assert mole.mole_check() == 0
    assert U == len(np.unique(ids))
    sample = torch.from_numpy(np.unique(rng.integers(0, T, 24))).cuda()
    sids = dids[sample].contiguous()
    uniq = torch.unique(sids)
    lut_rows = mole.mole_build_lut(E[uniq].contiguous(), W1, W2)
    remap = torch.searchsorted(uniq, sids).to(torch.int32)
    ref = mole.mole_lookup_combine(remap, h[sample].contiguous(), Wr, lut_rows)
    torch.testing.assert_close(out[sample], ref, rtol=2e-6, atol=1e-8)
    dout = torch.randn((T, D), generator=g, device="cuda")
    dE = torch.zeros((V, D), dtype=torch.float32, device="cuda")
    dW1 = torch.zeros((N, D, Dr), dtype=torch.float32, device="cuda")
    dh = torch.zeros((T, D), dtype=torch.float32, device="cuda")
    mole.mole_train_backward(dids, groups, h, Wr, E, W1, W2, dout, cache, U, dh=dh, dE=dE, dW1=dW1)
    assert mole.mole_check() == 0
    assert torch.isfinite(dh).all() and torch.isfinite(dE).all() and torch.isfinite(dW1).all()
    touched = dE.abs().sum(dim=1) > 0
    mask = torch.zeros(V, dtype=torch.bool, device="cuda")
    mask[dids.long()] = True
    assert not touched[~mask].any()
    del E, W1, W2, cache, dE, dW1
    torch.cuda.empty_cache()
