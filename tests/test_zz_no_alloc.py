"""lmoe_forward_noalloc: the forward on the library's built-in scratch area.

This entry point exists for callers that cannot allocate device memory where
they run the layer (a stream capture that must not allocate, an allocator
owned by another runtime, a path that must not take allocator locks).  The
test drives it through the C ABI and checks, on two calls in a row (the
second finds the first call's data still in the shared area), that it returns
what lmoe_forward with a caller workspace returns.  Both run the same kernels
on the same inputs, whose results do not depend on timing, so the outputs must
be equal bit for bit (which is within any tolerance the parity tests use): data
that an earlier call left in the area would show up as a difference.  It also
checks that the size limit is enforced before any work, and that a bounded
wait which gives up inside this entry point is reported by lmoe_check_device
with a NULL workspace.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test.
"""
import pytest
import torch

import lmoe_inputs as li

pytestmark = pytest.mark.gpu


def test_noalloc_matches_the_workspace_entry_point_twice():
    import latent_space_routed_b200 as lm
    w = li.custom("noalloc", 300, 512, 256, 256, 32, 6, 256, dtype="bf16", seed=31)
    W = li.weights(w)
    layer = lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in W.items()})
    T = w.T
    assert lm.lmoe_workspace_size(layer.handle, T) <= lm.LMOE_NOALLOC_WORKSPACE_BYTES
    x = li.tokens(w).cuda()
    ref = layer.forward_into(x, layer.empty_outputs(T))
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in ref.items()}

    x2 = li.tokens(w, seed=77).cuda()        # a different batch in between
    for xb in (x, x2, x):
        out = layer.empty_outputs(T)
        lm.lmoe_forward_noalloc(layer.handle, xb, T, out["output"], out["selected_experts"],
                                out["mixture_weights"], out["latent_routed_aggregate"])
        torch.cuda.synchronize()
        lm.lmoe_check_device(layer.handle, T, None)     # the area's status word: clean
        if xb is x:
            for key in ref:
                assert torch.equal(out[key], ref[key]), key

    # too many tokens for the built-in area: rejected with a clear status
    big = 1
    while lm.lmoe_workspace_size(layer.handle, big) <= lm.LMOE_NOALLOC_WORKSPACE_BYTES:
        big *= 2
    xb = torch.zeros(big, w.d, dtype=torch.bfloat16, device="cuda")
    out = layer.empty_outputs(big)
    with pytest.raises(lm.LmoeError) as ei:
        lm.lmoe_forward_noalloc(layer.handle, xb, big, out["output"], out["selected_experts"],
                                out["mixture_weights"], out["latent_routed_aggregate"])
    assert ei.value.status == lm.LMOE_ERR_WORKSPACE
    assert "64 MiB" in str(ei.value)
    layer.close()


def test_noalloc_reports_a_bounded_wait_that_gave_up():
    """A GEMM wait that runs out inside lmoe_forward_noalloc (test hook, no
    fault) is visible through lmoe_check_device with a NULL workspace, and the
    next call on the area is correct again."""
    import latent_space_routed_b200 as lm
    w = li.custom("noalloc_stall", 256, 256, 128, 256, 16, 4, 256, dtype="bf16", seed=43)
    layer = lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in li.weights(w).items()})
    T = w.T
    x = li.tokens(w).cuda()
    ref = {k: v.clone() for k, v in layer(x).items()}
    out = layer.empty_outputs(T)

    def call():
        lm.lmoe_forward_noalloc(layer.handle, x, T, out["output"], out["selected_experts"],
                                out["mixture_weights"], out["latent_routed_aggregate"])

    lm.lmoe_debug_inject(lm.LMOE_INJECT_STALL_NEXT_GEMM)
    call()
    with pytest.raises(lm.LmoeError) as ei:
        lm.lmoe_check_device(layer.handle, T, None)
    assert ei.value.status == lm.LMOE_ERR_DEVICE_TIMEOUT
    call()
    torch.cuda.synchronize()
    lm.lmoe_check_device(layer.handle, T, None)
    for key in ref:
        assert torch.equal(out[key], ref[key]), key
    layer.close()
