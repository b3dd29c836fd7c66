"""The benchmark's algorithmic model against the cooking-agi LatentMoE page.

bench.py turns its measured times into roofline fractions with per-token FLOP
and byte counts.  Their routed and projection parts must be the page's closed
form (section "Does the saving pay for more experts?": k * 3 l f + 2 d l MACs
per token, no projections when l = d, two FLOPs per MAC), and the per-stage
model must add up to the layer total, for every workload the bench runs.
"""
import pytest

import bench
import lmoe_inputs as li
import oracle


@pytest.mark.parametrize("name", sorted(li.WORKLOADS))
def test_layer_flops_follow_the_latent_budget(name):
    w = li.WORKLOADS[name]
    T = 7
    budget = oracle.latent_budget(w.d, w.l, w.f, w.E, w.k, T, w.item_bytes)
    router = 2 * w.d * w.E * T
    shared = 2 * 3 * w.d * (2 * w.f_s) * T          # two SwiGLU experts of width f_s at width d
    assert bench.layer_flops(w, T) - router - shared == 2 * budget["mac_per_token"] * T


@pytest.mark.parametrize("name", sorted(li.WORKLOADS))
def test_stage_model_adds_up_to_the_layer(name):
    w = li.WORKLOADS[name]
    T, touched = 5, min(w.E, 5 * w.k)
    stages = bench.stage_model(w, T, touched)
    assert sum(f for f, _ in stages.values()) == bench.layer_flops(w, T)
    if w.standard:
        assert stages["down_proj"] == (0, 0)


@pytest.mark.parametrize("name", sorted(li.WORKLOADS))
def test_layer_weight_bytes_follow_the_parameter_count(name):
    w = li.WORKLOADS[name]
    T, touched = 3, min(w.E, 3 * w.k)
    B = w.item_bytes
    budget = oracle.latent_budget(w.d, w.l, w.f, touched, min(w.k, touched), T, B)
    weights = budget["parameters"] * B + 6 * w.d * w.f_s * B + 4 * w.d * w.E
    io = T * w.d * B * 2 + T * w.k * (4 + B) + T * w.l * B
    assert bench.layer_bytes(w, T, touched) == weights + io
