"""mole_gather_plan (CUDA, through the C ABI) is bit-exact with the oracle's
sort + unique (MoLE page, 复杂度分析: a batch moves only its tokens' rows)."""
import numpy as np
import pytest

from helpers import dev
from mixture_lookup_experts_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,V,kind", [
    (1, 50304, "zipf"), (7, 10, "uniform"), (4096, 50304, "zipf"), (16384, 50304, "uniform"),
    (16384, 50304, "zipf"), (3000, 524288, "uniform"), (5000, 33, "uniform"),
])
def test_gather_plan_bit_exact(mole, oracle_mod, T, V, kind):
    rng = np.random.default_rng(T + V)
    ids = inputs.draw_ids(rng, T, V, kind)
    uniq, slot = mole.mole_gather_plan(dev(ids), V)
    assert mole.mole_check() == 0
    ru, rslot = oracle_mod.gather_plan(ids, V)
    np.testing.assert_array_equal(uniq.cpu().numpy(), ru)
    np.testing.assert_array_equal(slot.cpu().numpy(), rslot)


def test_gather_plan_bad_ids_and_limits(mole, oracle_mod):
    ids = np.array([3, -1, 9, 3, 10], np.int32)
    uniq, slot = mole.mole_gather_plan(dev(ids), 10)
    assert mole.mole_check() == 5
    np.testing.assert_array_equal(uniq.cpu().numpy(), [3, 9])
    np.testing.assert_array_equal(slot.cpu().numpy(), [0, -1, 1, 0, -1])
    with pytest.raises(mole.MoleError):
        mole.mole_gather_plan(dev(ids), 524289)
