"""Failure detection without a GPU fault.

The tensor-core GEMM bounds every wait; a test hook makes one GEMM's MMA warp
wait on a barrier that nothing signals, so that wait runs out.  The forward
must report LMOE_ERR_DEVICE_TIMEOUT through the device status word, and the
context must stay usable: the next forward is correct.  An injected
allocation failure in lmoe_create must return LMOE_ERR_OOM and leave the
process able to create layers.
"""
import pytest
import torch

import lmoe_inputs as li
from parity import rel_err

pytestmark = pytest.mark.gpu

W = li.custom("failure", 256, 256, 128, 256, 16, 4, 256, dtype="bf16", seed=41)


def test_bounded_wait_runs_out_and_is_reported():
    import latent_space_routed_b200 as lm
    weights = {k: v.cuda() for k, v in li.weights(W).items()}
    layer = lm.LatentMoE(lm.config_for(W), weights)
    x = li.tokens(W).cuda()
    ref = {k: v.clone() for k, v in layer(x).items()}
    torch.cuda.synchronize()
    layer.check_device(W.T)

    lm.lmoe_debug_inject(lm.LMOE_INJECT_STALL_NEXT_GEMM)
    layer(x)
    with pytest.raises(lm.LmoeError) as ei:
        layer.check_device(W.T)
    assert ei.value.status == lm.LMOE_ERR_DEVICE_TIMEOUT

    out = layer(x)                       # the context is still usable
    torch.cuda.synchronize()
    layer.check_device(W.T)
    assert torch.equal(out["selected_experts"], ref["selected_experts"])
    for key in ("output", "mixture_weights", "latent_routed_aggregate"):
        assert rel_err(out[key].float().cpu().numpy(), ref[key].float().cpu().numpy()) == 0.0
    layer.close()


def test_bounded_wait_in_the_fused_router_is_reported():
    """The fused router + top-k launch (a cluster of 8 CTAs per 128 tokens at
    E = 32, T = 256) runs first when stage events put every stage on one
    stream in order; the stall hook makes its MMA thread's wait run out.  Every
    CTA of each cluster still passes both cluster barriers, the status word
    reports it, and the next forward is bit-identical to a clean one."""
    import ctypes
    import latent_space_routed_b200 as lm
    w = li.custom("failure_router", 256, 512, 128, 256, 32, 4, 256, dtype="bf16", seed=43)
    layer = lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in li.weights(w).items()})
    x = li.tokens(w).cuda()
    ns = lm.LMOE_NUM_STAGES + 1
    events = [torch.cuda.Event(enable_timing=True) for _ in range(ns)]
    for e in events:   # materialise the events before taking their handles
        e.record()
    torch.cuda.synchronize()
    arr = (ctypes.c_void_p * ns)(*[e.cuda_event for e in events])
    lm.lmoe_set_stage_events(layer.handle, arr, ns)
    ref = {k: v.clone() for k, v in layer(x).items()}
    torch.cuda.synchronize()
    layer.check_device(w.T)

    lm.lmoe_debug_inject(lm.LMOE_INJECT_STALL_NEXT_GEMM)
    layer(x)
    with pytest.raises(lm.LmoeError) as ei:
        layer.check_device(w.T)
    assert ei.value.status == lm.LMOE_ERR_DEVICE_TIMEOUT

    out = layer(x)                       # the context is still usable
    torch.cuda.synchronize()
    layer.check_device(w.T)
    lm.lmoe_set_stage_events(layer.handle, None, 0)
    for key in ref:
        assert torch.equal(out[key], ref[key]), key
    layer.close()


@pytest.mark.parametrize("T", [256, 4200])
def test_bounded_wait_is_reported_through_the_host_entry(T):
    """lmoe_forward_host (at 4200 tokens cut into two pipelined chunks): a wait
    that runs out in the first chunk stays in the status word through the
    later chunks, and lmoe_check_device_host reports it."""
    import latent_space_routed_b200 as lm
    w = li.custom("failure_host", T, 256, 128, 256, 16, 6, 256, dtype="bf16", seed=42)
    layer = lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in li.weights(w).items()})
    xh = li.tokens(w).pin_memory()
    ref = layer.empty_outputs(T, device="cpu", pin=True)
    layer.forward_host(xh, ref)
    torch.cuda.synchronize()
    layer.check_device_host(T)

    lm.lmoe_debug_inject(lm.LMOE_INJECT_STALL_NEXT_GEMM)
    out = layer.empty_outputs(T, device="cpu", pin=True)
    layer.forward_host(xh, out)
    with pytest.raises(lm.LmoeError) as ei:
        layer.check_device_host(T)
    assert ei.value.status == lm.LMOE_ERR_DEVICE_TIMEOUT

    layer.forward_host(xh, out)                  # the context is still usable
    torch.cuda.synchronize()
    layer.check_device_host(T)
    for key in ref:
        assert torch.equal(out[key], ref[key]), key
    layer.close()


@pytest.mark.parametrize("which", [1, 3, 7])
def test_injected_allocation_failure(which):
    import latent_space_routed_b200 as lm
    weights = {k: v.cuda() for k, v in li.weights(W).items()}
    free0 = torch.cuda.mem_get_info()[0]
    lm.lmoe_debug_inject(lm.LMOE_INJECT_FAIL_ALLOC, which)
    with pytest.raises(lm.LmoeError) as ei:
        lm.LatentMoE(lm.config_for(W), weights)
    assert ei.value.status == lm.LMOE_ERR_OOM
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0 - (8 << 20)   # nothing of note leaked
    layer = lm.LatentMoE(lm.config_for(W), weights)            # and creation works again
    layer.close()
