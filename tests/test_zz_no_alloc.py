"""mole_build_lut_noalloc, the table build for callers that cannot allocate
device memory (serving loops whose memory footprint is fixed at start-up,
plugin hosts that give plugins no allocator): its tables equal those of
mole_build_lut bit for bit, called through the C ABI, on two calls in a row.
Both entry points run the same kernels and a table does not depend on how
experts are grouped per launch, so any difference is a fault in the fixed
scratch.  Collected last so a stop-at-first-failure run has already run the
rest of the suite."""
import pytest
import torch

from helpers import dev
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_build_matches_allocating_build_on_two_calls(mole, dtype):
    cases = [((300, 128, 3, 256), "gelu", 501), ((517, 256, 2, 512), "silu", 502)]
    for (V, D, N, Dr), act, seed in cases:  # two calls in a row, different shapes and data
        _, E, W1, W2 = inputs.expert_weights(inputs.small(V, D, N, Dr, dtype, seed))
        ref = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act=act)
        got = mole.mole_build_lut_noalloc(dev(E), dev(W1), dev(W2), act=act)
        assert mole.mole_check() == 0
        assert torch.equal(got, ref)


def test_noalloc_build_loops_over_expert_groups(mole):
    """8 MiB of bf16 activations per expert: two experts per pass through the
    16 MiB scratch, three passes for six experts; two calls in a row."""
    V, D, N, Dr = 4096, 128, 6, 1024
    for seed in (503, 504):
        _, E, W1, W2 = inputs.expert_weights(inputs.small(V, D, N, Dr, "bf16", seed))
        ref = mole.mole_build_lut(dev(E), dev(W1), dev(W2), act="gelu")
        got = mole.mole_build_lut_noalloc(dev(E), dev(W1), dev(W2), act="gelu")
        assert mole.mole_check() == 0
        assert torch.equal(got, ref)


def test_noalloc_build_rejects_a_request_beyond_its_scratch(mole):
    V, D, N, Dr = 4096, 64, 1, 4096  # one expert's activations: 32 MiB of bf16 > 16 MiB
    E = torch.zeros((V, D), dtype=torch.bfloat16, device="cuda")
    W1 = torch.zeros((N, D, Dr), dtype=torch.bfloat16, device="cuda")
    W2 = torch.zeros((N, Dr, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mole.MoleError) as e:
        mole.mole_build_lut_noalloc(E, W1, W2)
    assert e.value.status == 4  # MOLE_ERR_WORKSPACE
