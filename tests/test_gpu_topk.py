"""Biased top-k of every routing path on B200 against the oracle's top-k
("Stable LatentMoE", equation for T_k(x): TopK(r + b, k), equal scores to the
lower expert index as in the cooking-agi LatentMoE page's routed_example; the
cutoff of the same page's section "Quantile Balancing: measure now, use next
step").

Three routing paths choose the experts: the CUDA-core routing launch (up to 8
tokens), the fused tensor-core router + top-k (E <= 256, a cluster per token
tile) and the router GEMM followed by the one-warp-per-token top-k kernel
(larger E, or more token tiles than leave a cluster each); each runs the radix
selection for 9 <= k <= 32 and the tournament otherwise.

Two kinds of cases:
- exact scores: with W_r = 0 every router score is sigmoid(0) = 1/2 exactly in
  fp32 and fp64, and b holds multiples of 2^-6, so 1/2 + b is exact on both
  sides and the selection, its order and the cutoff are fixed by b alone
  (drawn from a few values: the cut falls inside groups of equal scores); they
  must equal the oracle's on every row.
- router scores: the selection is an integer decision taken from fp32 scores,
  so the oracle takes it from the GPU's own fp32 scores r + b (the scores are
  compared with the fp64 oracle in test_gpu_parity) and both must agree bit for
  bit, order and cutoff included.
"""
import numpy as np
import pytest
import torch

import lmoe_inputs as li
import oracle

pytestmark = pytest.mark.gpu

# (T, d, l, f, E, k, f_s): the path each shape takes is in its comment
SHAPES = [
    (7, 256, 128, 128, 64, 12, 128),      # CUDA-core routing launch, radix, 2 experts per lane
    (5, 256, 128, 128, 320, 32, 128),     # CUDA-core routing launch, radix, 16 per lane (6 padding)
    (8, 256, 128, 128, 48, 6, 128),       # CUDA-core routing launch, tournament
    (1000, 512, 256, 256, 64, 24, 256),   # fused router, clusters of 8 CTAs, radix
    (600, 256, 128, 128, 256, 32, 128),   # fused router, clusters of 4, radix, k = 32
    (300, 256, 128, 128, 96, 9, 128),     # fused router, radix at its smallest k
    (700, 256, 128, 128, 96, 8, 128),     # fused router, tournament at its largest k
    (300, 256, 128, 128, 320, 20, 128),   # router GEMM + top-k kernel (E > 256), radix
    (20000, 256, 128, 128, 64, 16, 128),  # router GEMM + top-k kernel (one cluster per tile), radix
]


def _layer(w, W):
    import latent_space_routed_b200 as lm
    return lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in W.items()})


def _run(w, W, x):
    layer = _layer(w, W)
    out = layer(x.cuda())
    torch.cuda.synchronize()
    layer.check_device(w.T)
    r = layer.region(w.T, "scores", torch.float32, (w.T, w.E)).cpu().numpy()
    cut = layer.region(w.T, "cutoff", torch.float32, (w.T,)).cpu().numpy()
    sel = out["selected_experts"].cpu().numpy()
    p = layer.region(w.T, "p32", torch.float32, (w.T, w.k)).cpu().numpy()
    layer.close()
    return sel, cut, r, p


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s[0]}_E{s[4]}_k{s[5]}")
def test_exact_scores_with_ties(shape):
    w = li.custom("topk_exact", *shape, dtype="bf16", seed=61)
    W = dict(li.weights(w))
    W["W_r"] = torch.zeros_like(W["W_r"])
    rng = np.random.default_rng(shape[4] * 100 + shape[5])
    for b in (rng.integers(-6, 7, w.E), np.zeros(w.E, np.int64)):   # groups of equal scores; all equal
        W["b"] = torch.from_numpy((b * 2.0 ** -6).astype(np.float32))
        sel, cut, r, p = _run(w, W, li.tokens(w))
        assert np.all(r == np.float32(0.5))
        s = 0.5 + W["b"].numpy().astype(np.float64)           # exact on both sides
        want_sel, _ = oracle.topk(s[None, :], w.k)
        want_cut = oracle.qb_cutoff(s[None, :], w.k)[0]
        np.testing.assert_array_equal(sel, np.broadcast_to(want_sel, sel.shape))
        np.testing.assert_array_equal(cut, np.full(w.T, want_cut, np.float32))
        np.testing.assert_allclose(p, 1.0 / w.k, rtol=1e-6)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s[0]}_E{s[4]}_k{s[5]}")
def test_router_scores(shape):
    w = li.custom("topk_router", *shape, dtype="bf16", seed=62)
    W = li.weights(w)
    sel, cut, r, p = _run(w, W, li.tokens(w))
    s = (r + W["b"].numpy()[None, :]).astype(np.float32) + np.float32(0.0)   # the kernel's fp32 add, -0 as +0
    want_sel, _ = oracle.topk(s.astype(np.float64), w.k)
    np.testing.assert_array_equal(sel, want_sel)
    np.testing.assert_array_equal(cut, oracle.qb_cutoff(s, w.k))
    rs = np.take_along_axis(r, want_sel.astype(np.int64), axis=1).astype(np.float64)
    np.testing.assert_allclose(p, rs / rs.sum(axis=1, keepdims=True), rtol=1e-5)
