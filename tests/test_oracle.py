"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test names the passage it follows.  None of them compares the oracle
with itself or with a retyped copy of its formula: they use values printed on
the pages, brute force, library routines for special cases, and invariants.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import lmoe_inputs as li
from conftest import GOLDEN


def _f32(a):
    return np.asarray(a, dtype=np.float32)


def _weights(**kw):
    return {k: _f32(v) for k, v in kw.items()}


# --------------------------------------------------------------------------
# "Stable LatentMoE", section Examples
# --------------------------------------------------------------------------

def _stable_example():
    with open(os.path.join(GOLDEN, "stable_latentmoe_example.json")) as fh:
        return json.load(fh)


def test_stable_latentmoe_worked_example():
    g = _stable_example()
    i = g["inputs"]
    w = _weights(W_r=i["router_projection"], b=i["current_bias"], W_down=i["latent_down_projection"],
                 W_up=i["latent_up_projection"], G=i["routed_gate_weights"], U=i["routed_up_weights"],
                 D=i["routed_down_weights"], Gs=i["shared_gate_weights"], Us=i["shared_up_weights"],
                 Ds=i["shared_down_weights"])
    out = oracle.forward(_f32(i["tokens"]), w, i["selected_count"], eps=i["eps"], act="situ",
                         gate_cap=i["gate_cap"], up_cap=i["up_cap"])
    e = g["expected"]
    assert out["selected_experts"].tolist() == e["selected_experts"]
    assert out["mixture_weights"].tolist() == e["mixture_weights"]
    # 16 printed digits; allow a few ulp for the order of fp64 operations.
    np.testing.assert_allclose(out["output"], e["output"], rtol=4e-16 * 4, atol=0)
    np.testing.assert_allclose(out["latent_routed_aggregate"], e["latent_routed_aggregate"], rtol=4e-16 * 4,
                               atol=0)
    # The router's raw scores are sigmoid(+1), sigmoid(-1) for router_projection [[1], [-1]].
    np.testing.assert_allclose(out["scores"][0], [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1))], rtol=1e-15)


def test_stable_latentmoe_example_rejects_other_gate_readings():
    """The same inputs under plain SwiGLU miss the printed output by far more
    than rounding: the example really fixes the capped (SiTU) gate."""
    g = _stable_example()
    i = g["inputs"]
    w = _weights(W_r=i["router_projection"], b=i["current_bias"], W_down=i["latent_down_projection"],
                 W_up=i["latent_up_projection"], G=i["routed_gate_weights"], U=i["routed_up_weights"],
                 D=i["routed_down_weights"], Gs=i["shared_gate_weights"], Us=i["shared_up_weights"],
                 Ds=i["shared_down_weights"])
    out = oracle.forward(_f32(i["tokens"]), w, 1, eps=i["eps"], act="swiglu")
    assert abs(out["latent_routed_aggregate"][0, 0] - g["expected"]["latent_routed_aggregate"][0][0]) > 1e-3


@pytest.mark.parametrize("case", [0, 1])
def test_stable_latentmoe_shape_examples(case):
    ex = _stable_example()["shape_examples"][case]
    T, d, l, E, k = ex["T"], ex["d"], ex["l"], ex["E"], ex["k"]
    f = fs = 3
    rng = np.random.default_rng(7)
    w = _weights(W_r=rng.standard_normal((E, d)), b=np.zeros(E), W_down=rng.standard_normal((l, d)),
                 W_up=rng.standard_normal((d, l)), G=rng.standard_normal((E, f, l)),
                 U=rng.standard_normal((E, f, l)), D=rng.standard_normal((E, l, f)),
                 Gs=rng.standard_normal((2, fs, d)), Us=rng.standard_normal((2, fs, d)),
                 Ds=rng.standard_normal((2, d, fs)))
    out = oracle.forward(_f32(rng.standard_normal((T, d))), w, k)
    for key, shp in ex["shapes"].items():
        assert list(out[key].shape) == shp
    # "Selected mixture weights sum to one per token" (Requirements)
    np.testing.assert_allclose(out["mixture_weights"].sum(1), 1.0, rtol=1e-14)


# --------------------------------------------------------------------------
# cooking-agi LatentMoE page
# --------------------------------------------------------------------------

def _agi():
    with open(os.path.join(GOLDEN, "cooking_agi_latentmoe.json")) as fh:
        return json.load(fh)


def test_routed_example_router_reads_full_width_input():
    """Section "Does the same latent vector imply the same output?": both
    inputs share the latent z = 1 but route differently, so outputs differ.
    Built in the oracle's own terms: W_down keeps the first coordinate, the
    router scores are monotone in the coordinates (sigmoid of the identity),
    k = 1, linear experts A(z) = 2z, B(z) = -z, W_up copies into both
    coordinates, no norm, shared experts contribute zero."""
    ex = _agi()["routed_example"]
    w = _weights(W_r=np.eye(2), b=np.zeros(2), W_down=[[1, 0]], W_up=[[1], [1]],
                 G=[[[2]], [[-1]]], U=[[[0]], [[0]]], D=[[[1]], [[1]]],
                 Gs=np.zeros((2, 1, 2)), Us=np.zeros((2, 1, 2)), Ds=np.zeros((2, 2, 1)))
    for c in ex["cases"]:
        out = oracle.forward(_f32([c["vector"]]), w, 1, act="linear", use_norm=False)
        assert out["selected_experts"][0, 0] == c["selected"]
        np.testing.assert_array_equal(out["latent_routed_aggregate"][0] / (2 if c["selected"] == 0 else -1),
                                      [c["latent"]])
        np.testing.assert_array_equal(out["output"][0], c["output"])


def test_equal_scores_go_to_the_lower_index():
    """routed_example selects index 0 when v0 >= v1."""
    w = _weights(W_r=np.eye(2), b=np.zeros(2), W_down=[[1, 0]], W_up=[[1], [1]],
                 G=[[[2]], [[-1]]], U=[[[0]], [[0]]], D=[[[1]], [[1]]],
                 Gs=np.zeros((2, 1, 2)), Us=np.zeros((2, 1, 2)), Ds=np.zeros((2, 2, 1)))
    out = oracle.forward(_f32([[1, 1], [3, 3]]), w, 1, act="linear", use_norm=False)
    assert out["selected_experts"][:, 0].tolist() == [0, 0]
    assert out["gap"].tolist() == [0.0, 0.0]


def test_norm_applies_to_the_sum():
    """Section "Why the normalization cannot simply move": RMSNorm of
    0.5 [2, 0] + 0.5 [0, 1] keeps the 2:1 direction ([1.2649, 0.6325])."""
    ex = _agi()["norm_order"]
    # two experts, both selected with equal raw scores (p = 0.5 each);
    # linear experts D_i (G_i z) with z = x = [1, 1] produce [2, 0] and [0, 1].
    w = _weights(W_r=[[0.0, 0.0], [0.0, 0.0]], b=np.zeros(2), W_down=np.eye(2), W_up=np.eye(2),
                 G=[[[1, 0]], [[1, 0]]], U=np.zeros((2, 1, 2)), D=[[[2], [0]], [[0], [1]]],
                 Gs=np.zeros((2, 1, 2)), Us=np.zeros((2, 1, 2)), Ds=np.zeros((2, 2, 1)))
    out = oracle.forward(_f32([[1, 1]]), w, 2, act="linear", eps=0.0)
    np.testing.assert_allclose(out["mixture_weights"][0], ex["weights"], rtol=0)
    np.testing.assert_allclose(out["latent_routed_aggregate"][0], [1.0, 0.5], rtol=0)
    np.testing.assert_allclose(np.round(out["output"][0], ex["digits"]), ex["rmsnorm_of_sum"], rtol=0)
    # and it is not the sum of the normalised outputs
    assert not np.allclose(np.round(out["output"][0], ex["digits"]), ex["sum_of_rmsnorms"])


def test_latent_budget_rows():
    b = _agi()["latent_budget"]
    rows = [oracle.latent_budget(*r["args"]) for r in b["rows"]]
    for got, r in zip(rows, b["rows"]):
        assert got == {"parameters": r["parameters"], "mac_per_token": r["mac_per_token"],
                       "slot_bytes": r["slot_bytes"]}
    # prose: parameters +2.1 %, MACs +8.3 % (third row against the first)
    assert round(rows[2]["parameters"] / rows[0]["parameters"] - 1, 3) == 0.021
    assert round(rows[2]["mac_per_token"] / rows[0]["mac_per_token"] - 1, 3) == 0.083


@pytest.mark.parametrize("args", [(0, 64, 256, 8, 2, 32, 2), (128, 256, 256, 8, 2, 32, 2),
                                  (128, 64, 256, 8, 9, 32, 2), (128.0, 64, 256, 8, 2, 32, 2)])
def test_latent_budget_rejects(args):
    with pytest.raises(ValueError):
        oracle.latent_budget(*args)


def test_fixed_cutoff_bias():
    q = _agi()["fixed_cutoff_bias"]
    bias = oracle.fixed_cutoff_bias(q["margins"], q["target"])
    assert sum(m + bias > 0 for m in q["margins"]) == q["positive_after_bias"]
    with pytest.raises(ValueError):
        oracle.fixed_cutoff_bias(q["margins"], 0)
    with pytest.raises(ValueError):
        oracle.fixed_cutoff_bias([0.1, float("nan")], 1)


# --------------------------------------------------------------------------
# Quantile Balancing statistics (cooking-agi page, "Quantile Balancing:
# measure now, use next step")
# --------------------------------------------------------------------------

@pytest.mark.parametrize("E,k", [(2, 1), (5, 2), (8, 3), (10, 9), (6, 6)])
def test_qb_cutoff_is_the_next_score_after_the_top_k(E, k):
    rng = np.random.default_rng(7 * E + k)
    s = rng.standard_normal((100, E))
    c = oracle.qb_cutoff(s, k)
    for t in range(s.shape[0]):
        ranked = sorted(s[t].tolist(), reverse=True)
        assert c[t] == (ranked[k] if k < E else -math.inf)
    # exactly the k selected experts have a positive margin (distinct scores)
    if k < E:
        assert np.all(((s - c[:, None]) > 0).sum(axis=1) == k)


def test_qb_margin_histogram_matches_a_count_over_bin_intervals():
    rng = np.random.default_rng(3)
    T, E, bins, lo, hi = 300, 7, 16, -0.5, 0.5
    s = rng.uniform(-0.9, 0.9, (T, E))
    c = rng.uniform(-0.2, 0.2, T)
    hist = oracle.qb_margin_histogram(s, c, bins, lo, hi)
    w = (hi - lo) / bins
    m = s - c[:, None]
    for e in range(E):
        for j in range(bins):
            a, b = lo + j * w, lo + (j + 1) * w
            inside = (m[:, e] >= a) & (m[:, e] < b)
            if j == 0:
                inside |= m[:, e] < lo
            if j == bins - 1:
                inside |= m[:, e] >= hi
            assert hist[e, j] == int(inside.sum())
    assert np.all(hist.sum(axis=1) == T)


def test_qb_histogram_quantile_reproduces_the_fixed_cutoff_example():
    """The page's margins [0.31, 0.16, 0.07, -0.08, -0.19, -0.34] with target 2:
    the histogram estimate of the quantile lies within one bin of the exact
    0.07, and the bias it gives leaves exactly two margins positive, as the
    page's assertion does."""
    q = _agi()["fixed_cutoff_bias"]
    margins, target = q["margins"], q["target"]
    lo, hi, bins = -1.0, 1.0, 200
    hist = oracle.qb_margin_histogram(np.asarray(margins)[:, None], np.zeros(len(margins)), bins, lo, hi)
    est = oracle.qb_quantile_from_histogram(hist, target, lo, hi)[0]
    exact = -oracle.fixed_cutoff_bias(margins, target)
    assert abs(est - exact) <= (hi - lo) / bins
    assert sum(m - est > 0 for m in margins) == q["positive_after_bias"]


@pytest.mark.parametrize("target", [0, 1, 17, 250, 499])
def test_qb_histogram_quantile_within_one_bin_of_the_exact_one(target):
    rng = np.random.default_rng(11 + target)
    margins = rng.uniform(-0.8, 0.8, 500)
    lo, hi, bins = -1.0, 1.0, 64
    hist = oracle.qb_margin_histogram(margins[:, None], np.zeros(500), bins, lo, hi)
    est = oracle.qb_quantile_from_histogram(hist, target, lo, hi)[0]
    exact = sorted(margins.tolist(), reverse=True)[target]
    assert abs(est - exact) <= (hi - lo) / bins


def test_qb_six_tokens_three_experts_top1():
    """The page's setting: six tokens, three experts, top-1, so six assignments
    and a target of two per expert.  Per expert, the margins against the
    current cutoff (the second score of each token) and the fixed-cutoff rule
    leave exactly two positive margins each; the histogram estimate agrees
    with it to one bin."""
    s = np.array([[0.9, 0.2, 0.1], [0.8, 0.3, 0.0], [0.7, 0.6, 0.2],
                  [0.1, 0.5, 0.4], [0.2, 0.1, 0.65], [0.3, 0.35, 0.05]])
    k, E = 1, 3
    target = s.shape[0] * k // E
    assert target == 2
    c = oracle.qb_cutoff(s, k)
    m = s - c[:, None]
    hist = oracle.qb_margin_histogram(s, c, 400, -1.0, 1.0)
    est = oracle.qb_quantile_from_histogram(hist, target, -1.0, 1.0)
    for e in range(E):
        bias = oracle.fixed_cutoff_bias(m[:, e].tolist(), target)
        assert int((m[:, e] + bias > 0).sum()) == target
        assert abs(est[e] + bias) <= 2.0 / 400


def test_oracle_parameter_count_matches_budget():
    """Count the weights the oracle consumes for the page's third budget row
    (d=128, l=64, f=256, 16 experts) and compare with the closed form."""
    w = li.weights(li.custom("budget", 1, 128, 64, 256, 16, 4, 8, dtype="f32"))
    routed = sum(w[n].numel() for n in ("G", "U", "D"))
    proj = w["W_down"].numel() + w["W_up"].numel()
    assert routed + proj == oracle.latent_budget(128, 64, 256, 16, 4, 32, 2)["parameters"]


# --------------------------------------------------------------------------
# Top-k by brute force
# --------------------------------------------------------------------------

@pytest.mark.parametrize("E,k", [(1, 1), (4, 2), (6, 3), (8, 4), (10, 4), (10, 1), (5, 5)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 31 + k)
    s = rng.standard_normal((200, E))
    sel, gap = oracle.topk(s, k)
    for i in range(s.shape[0]):
        best = max(itertools.combinations(range(E), k), key=lambda c: sum(s[i, j] for j in c))
        assert sorted(sel[i].tolist()) == sorted(best)
        # order: scores descending
        assert all(s[i, sel[i, j]] >= s[i, sel[i, j + 1]] for j in range(k - 1))
        rest = sorted((s[i, j] for j in range(E) if j not in best), reverse=True)
        expect_gap = math.inf if k == E else min(s[i, j] for j in best) - rest[0]
        assert gap[i] == expect_gap


def test_topk_ties():
    s = np.array([[0.5, 0.7, 0.7, 0.1], [0.2, 0.2, 0.2, 0.2], [0.3, 0.9, 0.3, 0.3]])
    sel, gap = oracle.topk(s, 2)
    assert sel.tolist() == [[1, 2], [0, 1], [1, 0]]
    sel1, _ = oracle.topk(s, 1)
    assert sel1[:, 0].tolist() == [1, 0, 1]
    assert gap.tolist()[1] == 0.0


# --------------------------------------------------------------------------
# Special cases that reduce to library routines
# --------------------------------------------------------------------------

def test_single_expert_is_a_dense_swiglu_mlp_between_two_linear_maps():
    """E = k = 1 makes p = 1, so the routed path is the dense composition
    Linear(d->l), SwiGLU MLP (l->f->l), RMSNorm, Linear(l->d), plus the two
    shared SwiGLU MLPs on x.  Checked against torch's own linear, silu and
    rms_norm in fp64; every matrix is non-square and non-symmetric, so a
    transposed or swapped operand fails."""
    rng = np.random.default_rng(3)
    d, l, f, fs = 7, 4, 5, 3
    F = torch.nn.functional
    W_down, W_up = rng.standard_normal((l, d)), rng.standard_normal((d, l))
    G, U, D = rng.standard_normal((1, f, l)), rng.standard_normal((1, f, l)), rng.standard_normal((1, l, f))
    Gs, Us, Ds = rng.standard_normal((2, fs, d)), rng.standard_normal((2, fs, d)), rng.standard_normal((2, d, fs))
    x = rng.standard_normal((4, d))
    w = _weights(W_r=rng.standard_normal((1, d)), b=np.zeros(1), W_down=W_down, W_up=W_up,
                 G=G, U=U, D=D, Gs=Gs, Us=Us, Ds=Ds)
    out = oracle.forward(_f32(x), w, 1, eps=1e-6)
    t = lambda a: torch.tensor(_f32(a), dtype=torch.float64)
    X = t(x)
    z = F.linear(X, t(W_down))
    u = F.linear(F.silu(F.linear(z, t(G)[0])) * F.linear(z, t(U)[0]), t(D)[0])
    y = F.linear(F.rms_norm(u, (l,), eps=1e-6), t(W_up))
    for j in range(2):
        y = y + F.linear(F.silu(F.linear(X, t(Gs)[j])) * F.linear(X, t(Us)[j]), t(Ds)[j])
    np.testing.assert_allclose(out["latent_routed_aggregate"], u.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["output"], y.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(out["mixture_weights"], 1.0)


def test_identity_projections_without_norm_are_the_standard_moe():
    """The standard-MoE form the library offers (cooking-agi page: a standard
    MoE routes and computes its experts at the model width) is the oracle's
    layer with W_down = W_up = I and no norm.  Checked against torch's topk,
    linear and silu at width d: r = sigmoid(W_r x), the top k of r + b,
    p = r_sel / sum r_sel, y = sum_j p_j E_j(x) + S_1(x) + S_2(x)."""
    rng = np.random.default_rng(8)
    d, f, fs, E, k, T = 6, 5, 3, 5, 2, 9
    F = torch.nn.functional
    Wr, b = rng.standard_normal((E, d)), rng.uniform(-0.05, 0.05, E)
    G, U, D = rng.standard_normal((E, f, d)), rng.standard_normal((E, f, d)), rng.standard_normal((E, d, f))
    Gs, Us, Ds = rng.standard_normal((2, fs, d)), rng.standard_normal((2, fs, d)), rng.standard_normal((2, d, fs))
    x = rng.standard_normal((T, d))
    w = _weights(W_r=Wr, b=b, W_down=np.eye(d), W_up=np.eye(d), G=G, U=U, D=D, Gs=Gs, Us=Us, Ds=Ds)
    out = oracle.forward(_f32(x), w, k, use_norm=False)
    t = lambda a: torch.tensor(_f32(a), dtype=torch.float64)
    X = t(x)
    r = torch.sigmoid(F.linear(X, t(Wr)))
    sel = torch.topk(r + t(b), k, dim=1).indices
    y = torch.zeros(T, d, dtype=torch.float64)
    u = torch.zeros(T, d, dtype=torch.float64)
    for i in range(T):
        rs = r[i, sel[i]]
        for j in range(k):
            e = int(sel[i, j])
            h = F.silu(F.linear(X[i], t(G)[e])) * F.linear(X[i], t(U)[e])
            u[i] += rs[j] / rs.sum() * F.linear(h, t(D)[e])
    y += u
    for j in range(2):
        y = y + F.linear(F.silu(F.linear(X, t(Gs)[j])) * F.linear(X, t(Us)[j]), t(Ds)[j])
    np.testing.assert_array_equal(out["selected_experts"], sel.numpy())
    np.testing.assert_allclose(out["latent_routed_aggregate"], u.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["output"], y.numpy(), rtol=1e-12, atol=1e-12)


def test_shared_only_is_two_swiglu_mlps():
    """Routed path zeroed (D = 0, so u = 0 and RMSNorm(0) = 0): y is the sum of
    the two shared SwiGLU experts, each on the full-width x (Hint 2)."""
    rng = np.random.default_rng(4)
    d, l, fs, E = 5, 2, 3, 3
    Gs, Us, Ds = rng.standard_normal((2, fs, d)), rng.standard_normal((2, fs, d)), rng.standard_normal((2, d, fs))
    x = rng.standard_normal((3, d))
    w = _weights(W_r=rng.standard_normal((E, d)), b=np.zeros(E), W_down=rng.standard_normal((l, d)),
                 W_up=rng.standard_normal((d, l)), G=rng.standard_normal((E, 4, l)),
                 U=rng.standard_normal((E, 4, l)), D=np.zeros((E, l, 4)), Gs=Gs, Us=Us, Ds=Ds)
    out = oracle.forward(_f32(x), w, 2)
    X = torch.tensor(_f32(x), dtype=torch.float64)
    y = 0
    for j in range(2):
        g, v, dd = (torch.tensor(_f32(a)[j], dtype=torch.float64) for a in (Gs, Us, Ds))
        y = y + (torch.nn.functional.silu(X @ g.T) * (X @ v.T)) @ dd.T
    np.testing.assert_allclose(out["output"], y.numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Invariants on a small random layer
# --------------------------------------------------------------------------

def _small(seed=11, T=24, d=16, l=8, f=12, E=7, k=3, fs=10):
    wl = li.custom("inv", T, d, l, f, E, k, fs, dtype="f32", seed=seed)
    return wl, li.tokens(wl), li.weights(wl)


def test_mixture_weights_sum_to_one_and_use_raw_scores():
    wl, x, w = _small()
    out = oracle.forward(x, w, wl.k)
    np.testing.assert_allclose(out["mixture_weights"].sum(1), 1.0, rtol=1e-14)
    r = out["scores"]
    sel = out["selected_experts"]
    raw = np.take_along_axis(r, sel.astype(np.int64), 1)
    np.testing.assert_allclose(out["mixture_weights"], raw / raw.sum(1, keepdims=True), rtol=1e-14)


def test_k_equals_E_gives_all_experts_and_bias_is_irrelevant():
    wl, x, w = _small(E=5, k=5)
    out = oracle.forward(x, w, 5)
    w2 = dict(w)
    w2["b"] = torch.tensor([0.4, -0.3, 0.2, 0.0, -0.1], dtype=torch.float32)
    out2 = oracle.forward(x, w2, 5)
    assert (np.sort(out["selected_experts"], 1) == np.arange(5)).all()
    r = out["scores"]
    order = np.argsort(out["selected_experts"], 1)
    p_sorted = np.take_along_axis(out["mixture_weights"], order, 1)
    np.testing.assert_allclose(p_sorted, r / r.sum(1, keepdims=True), rtol=1e-14)
    np.testing.assert_allclose(out2["output"], out["output"], rtol=1e-12, atol=1e-13)


def test_adding_a_constant_to_the_bias_changes_nothing():
    wl, x, w = _small()
    out = oracle.forward(x, w, wl.k)
    w2 = dict(w)
    w2["b"] = w["b"] + 0.25
    out2 = oracle.forward(x, w2, wl.k)
    # the constant is exact in fp32 for these magnitudes only up to rounding of b,
    # so compare selections where the gap is clear and everything else exactly
    clear = out["gap"] > 1e-6
    np.testing.assert_array_equal(np.sort(out["selected_experts"][clear], 1),
                                  np.sort(out2["selected_experts"][clear], 1))
    np.testing.assert_allclose(out2["output"][clear], out["output"][clear], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(out2["mixture_weights"][clear], out["mixture_weights"][clear], rtol=1e-13)


def test_scaling_routed_down_weights_scales_u_but_not_y():
    wl, x, w = _small()
    out = oracle.forward(x, w, wl.k, eps=0.0)
    w2 = dict(w)
    w2["D"] = w["D"] * 4.0           # exact in fp32
    out2 = oracle.forward(x, w2, wl.k, eps=0.0)
    np.testing.assert_allclose(out2["latent_routed_aggregate"], 4.0 * out["latent_routed_aggregate"], rtol=1e-13)
    np.testing.assert_allclose(out2["output"], out["output"], rtol=1e-12, atol=1e-12)


def test_rows_are_independent():
    wl, x, w = _small()
    full = oracle.forward(x, w, wl.k)
    perm = np.random.default_rng(5).permutation(wl.T)
    out = oracle.forward(x[perm], w, wl.k)
    for key in ("output", "mixture_weights", "latent_routed_aggregate", "selected_experts"):
        np.testing.assert_array_equal(out[key], full[key][perm])
    sub = oracle.forward(x, w, wl.k, rows=[5, 0, 17])
    for key in ("output", "latent_routed_aggregate"):
        np.testing.assert_array_equal(sub[key], full[key][[5, 0, 17]])


def test_two_shared_experts_equal_one_stacked_expert():
    wl, x, w = _small()
    out = oracle.forward(x, w, wl.k)
    w2 = dict(w)
    w2["Gs"] = w["Gs"].reshape(1, 2 * wl.f_s, wl.d)
    w2["Us"] = w["Us"].reshape(1, 2 * wl.f_s, wl.d)
    w2["Ds"] = torch.cat([w["Ds"][0], w["Ds"][1]], dim=1).unsqueeze(0)
    out2 = oracle.forward(x, w2, wl.k)
    np.testing.assert_allclose(out2["output"], out["output"], rtol=1e-12, atol=1e-13)


def test_situ_tends_to_swiglu_for_large_caps():
    wl, x, w = _small()
    a = oracle.forward(x, w, wl.k, act="swiglu")
    b = oracle.forward(x, w, wl.k, act="situ", gate_cap=1e6, up_cap=1e6)
    np.testing.assert_allclose(b["output"], a["output"], rtol=1e-9, atol=1e-10)


def test_given_selection_reproduces_top_k():
    wl, x, w = _small()
    a = oracle.forward(x, w, wl.k)
    b = oracle.forward(x, w, wl.k, sel=a["selected_experts"][:, ::-1].copy())
    np.testing.assert_allclose(b["output"], a["output"], rtol=1e-13, atol=1e-14)


def test_bf16_inputs_widen_exactly():
    wl = li.custom("bf", 8, 32, 16, 32, 6, 2, 16, dtype="bf16", seed=9)
    x, w = li.tokens(wl), li.weights(wl)
    a = oracle.forward(x, w, wl.k)
    w32 = {k: (v.float() if v.dtype == torch.bfloat16 else v) for k, v in w.items()}
    b = oracle.forward(x.float(), w32, wl.k)
    for key in ("output", "latent_routed_aggregate", "mixture_weights"):
        np.testing.assert_array_equal(a[key], b[key])


def test_bad_arguments():
    wl, x, w = _small()
    with pytest.raises(ValueError):
        oracle.forward(x, w, 0)
    with pytest.raises(ValueError):
        oracle.forward(x, w, wl.E + 1)
    with pytest.raises(ValueError):
        oracle.forward(x, w, wl.k, rows=[wl.T])
