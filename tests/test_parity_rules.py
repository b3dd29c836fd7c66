"""The comparison rules of tests/parity.py on the CPU, with mistakes planted
in copies of the oracle's own outputs (no GPU)."""
import numpy as np
import pytest

import lmoe_inputs as li
import oracle
from parity import compare, rel_err, row_rel_err


@pytest.fixture(scope="module")
def case():
    w = li.custom("rules", 64, 128, 64, 128, 16, 4, 128, dtype="f32", seed=61)
    x, W = li.tokens(w), li.weights(w)
    return w, x, W, oracle.forward(x, W, w.k)


def _as_gpu(ora):
    return {k: ora[k].copy() for k in ("output", "selected_experts", "mixture_weights", "latent_routed_aggregate")}


def test_identical_outputs_pass(case):
    w, x, W, ora = case
    errs = compare(_as_gpu(ora), ora, W["b"].numpy(), 1e-4)
    assert errs["output"] == 0.0 and errs["output_rows"] == 0.0


def test_a_defect_in_one_small_row_fails_the_row_check(case):
    """One row scaled down a thousandfold and then off by 50 %: the per-tensor
    normwise error stays under the tolerance, the per-row error does not."""
    w, x, W, ora = case
    ora2 = {k: v.copy() for k, v in ora.items()}
    ora2["latent_routed_aggregate"][5] *= 1e-3
    gpu = _as_gpu(ora2)
    gpu["latent_routed_aggregate"][5] *= 1.5
    assert rel_err(gpu["latent_routed_aggregate"], ora2["latent_routed_aggregate"]) < 2e-2
    assert row_rel_err(gpu["latent_routed_aggregate"], ora2["latent_routed_aggregate"]) == pytest.approx(0.5)
    with pytest.raises(AssertionError, match="latent_routed_aggregate_rows"):
        compare(gpu, ora2, W["b"].numpy(), 2e-2)


def test_swapped_mixture_weights_fail(case):
    w, x, W, ora = case
    gpu = _as_gpu(ora)
    gpu["mixture_weights"][3, [0, 1]] = gpu["mixture_weights"][3, [1, 0]]
    if abs(ora["mixture_weights"][3, 0] - ora["mixture_weights"][3, 1]) < 1e-3:
        pytest.skip("the two weights are too close to tell apart")
    with pytest.raises(AssertionError):
        compare(gpu, ora, W["b"].numpy(), 1e-4)


def test_a_wrong_expert_on_a_clear_row_fails(case):
    w, x, W, ora = case
    gpu = _as_gpu(ora)
    t = int(np.argmax(ora["gap"]))                    # the clearest selection
    unchosen = sorted(set(range(w.E)) - set(ora["selected_experts"][t].tolist()))
    gpu["selected_experts"][t, -1] = unchosen[0]
    with pytest.raises(AssertionError, match="selection differs"):
        compare(gpu, ora, W["b"].numpy(), 1e-4)
