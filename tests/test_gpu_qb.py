"""Quantile-Balancing statistics on B200 against the oracle (cooking-agi
LatentMoE page, section "Quantile Balancing: measure now, use next step").

The cutoff (each token's (k+1)-th biased score) and the margin bins are
integer-like decisions taken from fp32 scores, so the oracle takes them from
the GPU's own fp32 router scores in fp32 (the scores themselves are compared
with the fp64 oracle in test_gpu_parity) and both must agree bit for bit; the
bias update is compared to the oracle's fp64 estimate to fp32 rounding.
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as li
import oracle

pytestmark = pytest.mark.gpu


def _layer(w, W):
    import latent_space_routed_b200 as lm
    return lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in W.items()})


@pytest.mark.parametrize("shape", [
    (1000, 512, 256, 256, 32, 6, 256),   # tensor-core router, top 6 of 32
    (7, 256, 128, 128, 16, 4, 128),      # few tokens: CUDA-core router
    (96, 256, 128, 128, 8, 8, 128),      # k = E: nothing is left unselected
])
def test_quantile_balancing_statistics_match_the_oracle(shape):
    w = li.custom("qb", *shape, dtype="bf16", seed=41)
    W = li.weights(w)
    T, E, k = w.T, w.E, w.k
    layer = _layer(w, W)
    layer(li.tokens(w).cuda())
    torch.cuda.synchronize()
    r = layer.region(T, "scores", torch.float32, (T, E)).cpu().numpy()
    cut = layer.region(T, "cutoff", torch.float32, (T,)).cpu().numpy()
    b = W["b"].numpy().astype(np.float32)
    s = (r + b[None, :]).astype(np.float32)          # the kernel's fp32 add
    np.testing.assert_array_equal(cut, oracle.qb_cutoff(s, k))

    bins, lo, hi = 48, -0.5, 0.5
    hist = torch.zeros(E, bins, dtype=torch.int32, device="cuda")
    layer.qb_histogram(T, hist, bins, lo, hi)
    layer.qb_histogram(T, hist, bins, lo, hi)        # a second batch accumulates
    ref = 2 * oracle.qb_margin_histogram(s, cut, bins, lo, hi)
    np.testing.assert_array_equal(hist.cpu().numpy(), ref)
    if k == E:
        assert np.all(ref[:, -1] == 2 * T)           # every margin is +inf

    target = 2 * T * k // E
    nb = layer.qb_bias_update(hist, bins, lo, hi, target).cpu().numpy()
    q = oracle.qb_quantile_from_histogram(ref, target, lo, hi)
    np.testing.assert_allclose(nb, b.astype(np.float64) - q, rtol=0, atol=2e-6)
    layer.close()


def test_quantile_balancing_bias_moves_load_towards_the_target():
    """Measure now, use next step: with a strongly skewed bias, one update from
    the margin histogram brings the busiest expert's load much closer to the
    average, and the bias only changes selection (the page: mixture weights
    still use raw affinities)."""
    w = li.custom("qb_skew", 2048, 256, 128, 128, 16, 2, 128, dtype="bf16", bias="zipf", seed=43)
    W = li.weights(w)
    T, E, k = w.T, w.E, w.k
    layer = _layer(w, W)
    x = li.tokens(w).cuda()
    out0 = layer(x)
    torch.cuda.synchronize()
    load0 = np.bincount(out0["selected_experts"].cpu().numpy().ravel(), minlength=E)
    bins, lo, hi = 256, -1.0, 1.0
    hist = torch.zeros(E, bins, dtype=torch.int32, device="cuda")
    layer.qb_histogram(T, hist, bins, lo, hi)
    layer.set_bias(layer.qb_bias_update(hist, bins, lo, hi, T * k // E))
    out1 = layer(x)
    torch.cuda.synchronize()
    load1 = np.bincount(out1["selected_experts"].cpu().numpy().ravel(), minlength=E)
    avg = T * k / E
    assert load0.max() > 3 * avg
    assert load1.max() < 0.6 * load0.max()
    # raw-score weights: p is r of the chosen experts over their sum, whatever the bias
    r1 = layer.region(T, "scores", torch.float32, (T, E)).cpu().numpy().astype(np.float64)
    sel1 = out1["selected_experts"].cpu().numpy()
    p = np.take_along_axis(r1, sel1, axis=1)
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(out1["mixture_weights"].float().cpu().numpy(), p, atol=1e-2)
    layer.close()
