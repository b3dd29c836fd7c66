"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on B200.

Sizes: small cases span several 128 x 256 tiles with ragged tails and are
compared element by element on every row; the full-size workloads run the
whole batch on the GPU (the launch configuration the benchmark times) and are
compared on a seeded sample of token rows that the oracle computes one by one.
"""
import functools

import numpy as np
import pytest
import torch

import lmoe_inputs as li
import oracle
from parity import compare, SEL_GAP

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _lm():
    import latent_space_routed_b200 as lm
    return lm


@functools.lru_cache(maxsize=2)
def _weights(w):
    return li.weights(w)


def _layer(w, gemm=0, act=0, W=None):
    lm = _lm()
    W = _weights(w) if W is None else W
    return lm.LatentMoE(lm.config_for(w, gemm=gemm, act=act), {k: v.cuda() for k, v in W.items()})


def run_parity(w, T=None, gemm=0, act="swiglu", n_rows=None, seed=0, expert_tails=False, bias=None):
    """Whole batch on the GPU; oracle on every row, or on n_rows seeded rows
    (always with the last row, and with expert_tails also every token that
    holds an expert's last slot row, where a tile's ragged edge falls).
    bias replaces the workload's selection bias on both sides."""
    lm = _lm()
    T = w.T if T is None else T
    W = _weights(w)
    if bias is not None:
        W["b"] = bias
    x = li.tokens(w, T)
    layer = _layer(w, gemm, lm.LMOE_ACT_SITU if act == "situ" else lm.LMOE_ACT_SWIGLU, W=W)
    out = layer(x.cuda())
    torch.cuda.synchronize()
    layer.check_device(T)
    rows = None
    if n_rows is not None and n_rows < T:
        rng = np.random.default_rng(1234 + seed)
        rows = np.sort(rng.choice(T, size=n_rows, replace=False))
        rows[-1] = T - 1   # always include the ragged tail
        if expert_tails:
            offsets = layer.region(T, "offsets", torch.int32, (w.E + 1,)).cpu().numpy().astype(np.int64)
            perm = layer.region(T, "perm_tok", torch.int32, (T * w.k,)).cpu().numpy()
            last = offsets[1:][offsets[1:] > offsets[:-1]] - 1      # each non-empty expert's last slot row
            rows = np.concatenate([rows, perm[last]])
        rows = np.unique(rows)
    # a standard workload carries identity projections: with no norm, the
    # oracle's layer formula is then the standard MoE
    norm = not w.standard
    ora = oracle.forward(x, W, w.k, act=act, rows=rows, eps=w.eps, use_norm=norm)

    def rerun(idx, sel):
        r = idx if rows is None else rows[idx]
        return oracle.forward(x, W, w.k, act=act, rows=r, sel=sel, eps=w.eps, use_norm=norm)

    errs = compare({k: v.cpu() for k, v in out.items()}, ora, W["b"].numpy(), TOL[w.dtype], rerun, rows)
    layer.close()
    return errs, out


# ---------------------------------------------------------------- small, all rows
MULTI = li.custom("multi_tile_ragged", 1000, 512, 256, 256, 32, 6, 256, dtype="bf16", seed=21)


def test_tiny_fp32_all_rows():
    errs, _ = run_parity(li.WORKLOADS["tiny_fp32"])
    assert errs["output"] < 1e-4


def test_tiny_fp32_situ_gate():
    run_parity(li.WORKLOADS["tiny_fp32"], act="situ")


@pytest.mark.parametrize("gemm", [0, 1], ids=["tensor_cores", "cuda_cores"])
def test_bf16_multi_tile_ragged(gemm):
    run_parity(MULTI, gemm=gemm)


def test_bf16_situ_tensor_cores():
    run_parity(MULTI, act="situ")


@pytest.mark.parametrize("T", [1, 2, 3, 6, 8, 9, 127, 129, 333])
def test_bf16_token_counts(T):
    """Token counts across the few-token plans (one CUDA-core routing launch up
    to 8 tokens, weight-streaming GEMVs up to 2, split-K tensor-core GEMMs
    above) and ragged tiles."""
    run_parity(MULTI, T=T)


@pytest.mark.parametrize("T", [6000, 2500, 200])
def test_fused_router_cluster_sizes(T):
    """The fused router + top-k launch with clusters of 2, 4 and 8 CTAs per
    128-token tile (47, 20 and 2 tiles of the multi-tile case): the split
    logits are summed over the cluster's shared memory in rank order."""
    run_parity(MULTI, T=T)


ODD = li.custom("odd_k_blocks", 1100, 448, 192, 256, 32, 6, 256, dtype="bf16", seed=23)


@pytest.mark.parametrize("act", ["swiglu", "situ"])
def test_odd_k_block_counts(act):
    """K of 7 (down-projection, shared gate/up), 3 (routed gate/up) and 11
    (final GEMM) 64-wide k-blocks on CTA-pair tiles: the last ring stage holds
    one k-block, whose partner is read past the end of K (zero fill) and not
    multiplied.  Both gates, on CTA-pair tiles with half tiles."""
    run_parity(ODD, act=act)


@pytest.mark.parametrize("T", [1088, 1152, 1153, 1280, 1281])
def test_expert_row_counts_at_tile_edges(T):
    """A selection bias far above every score sends all T tokens to the same
    six experts, so each routed GEMM sees six experts of exactly T slot rows
    on CTA-pair tiles: last m-tiles of 64, 128, 129, 0 and 1 rows (the first
    two and the last run as half tiles, M = 128; 129 rows take a full tile)."""
    b = torch.zeros(MULTI.E, dtype=torch.float32)
    b[[3, 7, 11, 15, 19, 23]] = 10.0
    errs, out = run_parity(MULTI, T=T, bias=b)
    sel = out["selected_experts"].cpu()
    assert set(sel.unique().tolist()) == {3, 7, 11, 15, 19, 23}


@pytest.mark.parametrize("E,k", [(8, 8), (64, 1), (40, 17)])
def test_bf16_selection_extremes(E, k):
    w = li.custom(f"sel_{E}_{k}", 300, 256, 128, 256, E, k, 256, dtype="bf16", seed=22)
    run_parity(w)


def test_bf16_many_rows_per_expert():
    """About 400 slot rows per expert (the grouped GEMMs' larger-tile regime,
    with ragged expert ends inside tiles); every row is compared."""
    w = li.custom("many_rows", 1600, 256, 128, 256, 16, 4, 256, dtype="bf16", seed=24)
    run_parity(w)


@pytest.mark.parametrize("shape", [
    (1536, 512, 512, 128, 8, 2, 128),    # K = l = 512: eight A k-blocks, one n-tile per expert
    (1200, 256, 64, 384, 16, 4, 128),    # K = 64: one A k-block, three n-tiles
])
def test_bf16_pair_tiles_edge_shapes(shape):
    """Enough slot rows per expert for CTA-pair tiles, with the routed GEMMs'
    K and n-tile counts at their edges (eight k-blocks and one n-tile; one
    k-block and three n-tiles); every row is compared."""
    w = li.custom("pair_edges", *shape, dtype="bf16", seed=25)
    errs, _ = run_parity(w)
    assert errs["output"] <= TOL["bf16"]


def test_bf16_latent_rows_above_8_kb():
    """l = 4160 (8320-byte bf16 rows): the permute stores each z row to its
    slot rows in two pieces; every row is compared."""
    w = li.custom("wide_latent", 40, 4160, 4160, 128, 16, 4, 128, dtype="bf16", seed=46)
    errs, _ = run_parity(w)
    assert errs["output"] <= TOL["bf16"]


@pytest.mark.parametrize("dtype,gemm", [("bf16", 0), ("bf16", 1), ("f32", 0)])
def test_standard_moe_form(dtype, gemm):
    """config.standard: experts at the model width on x itself, no projections
    or norm, y = shared + sum_j p_j E_j(x) (the final GEMM adds u in its
    epilogue); every row against the oracle run with identity projections and
    no norm."""
    w = li.custom("standard", 600, 256, 256, 256, 16, 3, 256, dtype=dtype, seed=27, standard=True)
    run_parity(w, gemm=gemm)


@pytest.mark.parametrize("T", [2, 5, 100])
def test_standard_moe_form_few_tokens(T):
    """Few tokens: CUDA-core router and split-K final GEMM, whose reduction
    adds u."""
    w = li.custom("standard_few", T, 512, 512, 256, 32, 4, 256, dtype="bf16", seed=28, standard=True)
    run_parity(w)


@pytest.mark.parametrize("bias", ["zipf", "uniform"])
def test_bf16_pair_tiles_skewed_expert_loads(bias):
    """CTA-pair tiles for the grouped GEMMs; a Zipf bias gives experts from a
    handful of slot rows to thousands (empty and ragged m-tiles next to long
    runs of full ones); every row compared."""
    w = li.custom("skew_" + bias, 1500, 256, 256, 256, 16, 4, 256, dtype="bf16", bias=bias, seed=26)
    run_parity(w)


@pytest.mark.parametrize("T", [2, 4])
def test_bf16_few_slot_rows_per_expert(T):
    """Fewer slot rows than experts (S <= E, the decode regime at a small
    size): single-CTA tiles with one or two real rows each; every row compared."""
    w = li.custom("grouped_split", 4, 512, 512, 512, 64, 4, 256, dtype="bf16", seed=45)
    run_parity(w, T=T)


def test_fp32_multi_tile_ragged():
    w = li.custom("multi_f32", 333, 256, 128, 128, 24, 5, 192, dtype="f32", seed=23)
    run_parity(w)


def test_equal_scores_go_to_the_lower_expert_index():
    """Router rows repeated in groups of four (zero bias) give exactly equal
    scores inside each group, so every row's top 6 is one whole group plus two
    experts of the next one: the selection and its order must be the oracle's
    (score descending, equal scores to the lower index), on rows whose distinct
    score values near the cut are more than 1e-5 apart (fp32 vs fp64)."""
    lm = _lm()
    w = li.custom("ties", 256, 256, 128, 128, 64, 6, 128, dtype="bf16", seed=29)
    W = dict(li.weights(w))
    Wr = W["W_r"].clone()
    for g in range(w.E // 4):
        Wr[4 * g + 1:4 * g + 4] = Wr[4 * g]
    W["W_r"] = Wr
    W["b"] = torch.zeros_like(W["b"])
    x = li.tokens(w)
    layer = lm.LatentMoE(lm.config_for(w), {k: v.cuda() for k, v in W.items()})
    for T in (5, w.T):                       # CUDA-core router, tensor-core router
        out = layer(x[:T].cuda())
        torch.cuda.synchronize()
        ora = oracle.forward(x[:T], W, w.k, eps=w.eps)
        sel_g = out["selected_experts"].cpu().numpy()
        checked = 0
        for t in range(T):
            vals = np.unique(ora["scores"][t])[::-1][:4]     # distinct group scores, descending
            if np.min(-np.diff(vals)) <= 1e-5:
                continue
            np.testing.assert_array_equal(sel_g[t], ora["selected_experts"][t])
            assert sel_g[t][4] % 4 == 0 and sel_g[t][5] % 4 == 1   # the next group's two lowest
            checked += 1
        assert checked >= 0.9 * T
    layer.close()


# ---------------------------------------------------------------- stages
def test_router_scores_and_dispatch_are_exact():
    """Scores r match the fp64 oracle to fp32 rounding; counts, offsets, slot
    positions and the slot -> token map equal a host stable counting sort of the
    GPU's own selection, bit for bit."""
    w = MULTI
    T = w.T
    W = _weights(w)
    x = li.tokens(w)
    layer = _layer(w)
    out = layer(x.cuda())
    torch.cuda.synchronize()
    r_gpu = layer.region(T, "scores", torch.float32, (T, w.E)).cpu().numpy().astype(np.float64)
    ora = oracle.forward(x, W, w.k, rows=np.arange(64))
    assert np.abs(r_gpu[:64] - ora["scores"]).max() < 2e-6
    sel = out["selected_experts"].cpu().numpy().astype(np.int64)
    counts = np.bincount(sel.ravel(), minlength=w.E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    slot_expected = np.zeros_like(sel)
    perm_expected = np.zeros(T * w.k, np.int64)
    fill = offsets[:-1].copy()
    for t in range(T):
        for j in range(w.k):
            e = sel[t, j]
            slot_expected[t, j] = fill[e]
            perm_expected[fill[e]] = t
            fill[e] += 1
    np.testing.assert_array_equal(layer.region(T, "counts", torch.int32, (w.E,)).cpu().numpy(), counts)
    np.testing.assert_array_equal(layer.region(T, "offsets", torch.int32, (w.E + 1,)).cpu().numpy(), offsets)
    np.testing.assert_array_equal(layer.region(T, "slot_of", torch.int32, (T, w.k)).cpu().numpy(), slot_expected)
    np.testing.assert_array_equal(layer.region(T, "perm_tok", torch.int32, (T * w.k,)).cpu().numpy(), perm_expected)
    # the latent z = W_down x of every token (bf16-rounded) in each of its k
    # expert-sorted slot rows, which the routed gate/up GEMM reads
    zp = layer.region(T, "Zp", torch.bfloat16, (T * w.k, w.l)).float().cpu()
    slots = torch.from_numpy(slot_expected.astype(np.int64))
    ref = (x.double() @ W["W_down"].double().T)
    got = zp[slots.reshape(-1)].reshape(T, w.k, w.l).double()
    assert ((got - ref[:, None, :]).abs().max() / ref.abs().max()).item() < 1e-2
    layer.close()


def test_deterministic_and_host_entry_matches():
    w = MULTI
    lm = _lm()
    x = li.tokens(w)
    layer = _layer(w)
    a = {k: v.clone() for k, v in layer(x.cuda()).items()}
    b = layer(x.cuda())
    for key in a:
        assert torch.equal(a[key], b[key]), key
    xh = x.pin_memory()
    oh = layer.empty_outputs(w.T, device="cpu", pin=True)
    layer.forward_host(xh, oh)
    torch.cuda.synchronize()
    for key in a:
        assert torch.equal(a[key].cpu(), oh[key]), key
    assert layer.launch_count(w.T) > 0
    layer.close()


def test_side_stream_order_and_graph_capture_match_one_stream():
    """T >= 256 runs the shared gate/up GEMM on the handle's side stream; with
    stage events set every stage runs on the caller's stream.  Both orders, on
    the default and on another stream, and a CUDA-graph replay of the forward
    return the same bits."""
    import ctypes
    lm = _lm()
    w = MULTI
    x = li.tokens(w).cuda()
    layer = _layer(w)
    ref = {k: v.clone() for k, v in layer(x).items()}
    ns = lm.LMOE_NUM_STAGES + 1
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(ns)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    arr = (ctypes.c_void_p * ns)(*[e.cuda_event for e in evs])
    lm.lmoe_set_stage_events(layer.handle, arr, ns)
    one = {k: v.clone() for k, v in layer(x).items()}
    torch.cuda.synchronize()
    lm.lmoe_set_stage_events(layer.handle, None, 0)
    for key in ref:
        assert torch.equal(ref[key], one[key]), key

    other = torch.cuda.Stream()
    out = layer.empty_outputs(w.T)
    layer.workspace(w.T)
    other.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(other):
        layer.forward_into(x, out, stream=other)
    torch.cuda.current_stream().wait_stream(other)
    torch.cuda.synchronize()
    for key in ref:
        assert torch.equal(ref[key], out[key]), key

    gout = layer.empty_outputs(w.T)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.forward_into(x, gout, stream=torch.cuda.current_stream())
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for key in ref:
        assert torch.equal(ref[key], gout[key]), key
    del graph
    layer.close()


def test_host_entry_pipelines_chunks():
    """Enough tokens for lmoe_forward_host to cut the batch into chunks whose
    copies overlap the compute: each row equals lmoe_forward on the chunk that
    holds it, bit for bit, and the whole batch matches the oracle."""
    lm = _lm()
    w = li.custom("host_chunks", 4200, 256, 128, 256, 16, 6, 256, dtype="bf16", seed=44)
    x = li.tokens(w)
    layer = _layer(w)
    xh = x.pin_memory()
    oh = layer.empty_outputs(w.T, device="cpu", pin=True)
    layer.forward_host(xh, oh)
    torch.cuda.synchronize()
    layer.check_device_host(w.T)
    Tc = (w.T + 1) // 2                      # max(2048, 192 E / k) = 2048 -> two chunks
    for t0 in (0, Tc):
        part = layer(x[t0:t0 + Tc].cuda())
        torch.cuda.synchronize()
        for key in part:
            assert torch.equal(part[key].cpu(), oh[key][t0:t0 + Tc]), key
    ora = oracle.forward(x, _weights(w), w.k, eps=w.eps)
    compare(oh, ora, _weights(w)["b"].numpy(), TOL["bf16"],
            lambda idx, sel: oracle.forward(x, _weights(w), w.k, rows=idx, sel=sel, eps=w.eps))
    layer.close()


def test_launch_count_matches_the_kernels_launched():
    """lmoe_launch_count (the bench's gpu_launches) against the library
    kernels a CUDA activity trace sees in one forward, for the one-or-two-token
    plan and for the two-stream plan."""
    from torch.profiler import profile, ProfilerActivity
    w = MULTI
    x = li.tokens(w).cuda()
    layer = _layer(w)
    layer(x)
    torch.cuda.synchronize()
    for T in (2, w.T):
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            layer(x[:T])
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if str(e.device_type).endswith("CUDA")]
        if not names:
            pytest.skip("no CUDA activity trace on this machine")
        ours = [n for n in names if "lmoe" in n]
        assert len(ours) == layer.launch_count(T), sorted(set(ours))
    layer.close()


def test_zero_tokens_is_a_noop_and_errors_are_reported():
    lm = _lm()
    w = MULTI
    layer = _layer(w)
    x = torch.empty(0, w.d, dtype=torch.bfloat16, device="cuda")
    lm.lmoe_forward(layer.handle, x, 0, None, None, None, None, None, 0)
    x = li.tokens(w, 16).cuda()
    out = layer.empty_outputs(16)
    with pytest.raises(lm.LmoeError) as ei:
        lm.lmoe_forward(layer.handle, x, 16, out["output"], out["selected_experts"], out["mixture_weights"],
                        out["latent_routed_aggregate"], layer.workspace(16), 64)
    assert ei.value.status == lm.LMOE_ERR_WORKSPACE
    ws = layer.workspace(16)
    xm = torch.empty(16 * w.d + 1, dtype=torch.bfloat16, device="cuda")[1:].view(16, w.d)
    with pytest.raises(lm.LmoeError) as ei:
        lm.lmoe_forward(layer.handle, xm, 16, out["output"], out["selected_experts"], out["mixture_weights"],
                        out["latent_routed_aggregate"], ws, ws.numel())
    assert ei.value.status == lm.LMOE_ERR_UNSUPPORTED
    layer.close()


# ---------------------------------------------------------------- full-size workloads
@pytest.mark.parametrize("name", ["acc_d2048", "eff_zipf_d2048"])
def test_full_size_every_row(name):
    """The whole batch in the benchmark's launch configuration, every row
    against the oracle."""
    errs, _ = run_parity(li.WORKLOADS[name])
    assert errs["rows_compared"] == li.WORKLOADS[name].T
    print(name, errs)


def test_standard_full_size_sampled_rows():
    errs, _ = run_parity(li.WORKLOADS["std_d2048"], n_rows=256, expert_tails=True)
    print("std_d2048", errs)


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_decode_sweep(T):
    """Every row of each decode batch."""
    w = li.WORKLOADS["decode_d7168"]
    errs, _ = run_parity(w, T=T)
    assert errs["rows_compared"] == T
    print("decode", T, errs)


def test_large_sampled_rows():
    """512 seeded rows plus every token holding an expert's last slot row (the
    grouped GEMMs' ragged tile edges): about a thousand rows of 32768."""
    errs, _ = run_parity(li.WORKLOADS["large_d4096"], n_rows=512, expert_tails=True)
    assert errs["rows_compared"] >= 512
    print("large", errs)
