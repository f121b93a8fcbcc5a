"""mole_build_lut_noalloc, the table build for callers that cannot allocate
device memory (code inside a CUDA-graph stream capture, serving loops with a
fixed memory footprint, plugin hosts without an allocator for plugins): its
tables equal those of mole_build_lut, called through the C ABI, on two calls
in a row.  Collected last so a stop-at-first-failure run has already run the
rest of the suite."""
import numpy as np
import pytest
import torch

from helpers import BUILD_MAX_ULPS, as_f64, build_ulps, dev, host_bits
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


def _close(got: torch.Tensor, ref: torch.Tensor):
    """Within the build tolerance of the allocating entry point's table."""
    r = as_f64(host_bits(ref)) if ref.dtype == torch.bfloat16 else ref.cpu().numpy().astype(np.float64)
    g = host_bits(got)
    assert build_ulps(g, r).max() <= BUILD_MAX_ULPS


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_build_matches_allocating_build_on_two_calls(mole, dtype):
    cases = [((300, 128, 3, 256), "gelu", 501), ((517, 256, 2, 512), "silu", 502)]
    for (V, D, N, Dr), act, seed in cases:  # two calls in a row, different shapes and data
        _, E, W1, W2 = inputs.expert_weights(inputs.small(V, D, N, Dr, dtype, seed))
        ref = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act=act)
        got = mole.mole_build_lut_noalloc(dev(E), dev(W1), dev(W2), act=act)
        assert mole.mole_check() == 0
        _close(got, ref)


def test_noalloc_build_rejects_a_request_beyond_its_scratch(mole):
    V, D, N, Dr = 4096, 64, 1, 4096  # one expert's activations: 32 MiB of bf16 > 16 MiB
    E = torch.zeros((V, D), dtype=torch.bfloat16, device="cuda")
    W1 = torch.zeros((N, D, Dr), dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros((N, Dr, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mole.MoleError) as e:
        mole.mole_build_lut_noalloc(E, W1, W2)
    assert e.value.status == 4  # MOLE_ERR_WORKSPACE
