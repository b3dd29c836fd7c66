#!/usr/bin/env python
"""LatentMoE layer-forward benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME [--T T]]
    python bench.py --impl reference ...

One step = one whole layer forward (router, top-k, dispatch, down-projection,
routed experts, combine, RMSNorm, shared experts, up-projection) over the
workload's batch, inputs resident in HBM.  Prints one JSON line (rank 0).

With no --workload the headline is large_d4096 (T 32768, d 4096, 512 experts,
top 24), the largest single-GPU workload; the same run also measures
acc_d2048, eff_zipf_d2048, std_d2048 and the decode_d7168 sweep (T = 1, 8,
32, 128, also replayed from a CUDA graph) and reports them under
``workloads``.  ``--save DIR`` writes each workload's full line to
DIR/bench_<workload>[_T<T>].json.

N > 1 runs N independent replicas, one per GPU, each on its own batch: the
layer's rows are independent and there is no exchange step, so there is no
data-path collective (weak scaling).  The process group is used only for the
barrier and the max over ranks of the timed region.  Launched without
torch.distributed.run (no WORLD_SIZE in the environment), ``--gpus N`` starts
the N ranks itself through torch.distributed.run on 127.0.0.1.

``--impl reference`` times the fp64 CPU oracle (the only reference this
layer has) on the host cores, each step a bounded sample of token rows.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import socket
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LatentMoE layer fwd tokens/s on 1 B200; % of tensor-core or HBM roofline"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
HEADLINE = "large_d4096"
OTHERS = (("acc_d2048", None), ("eff_zipf_d2048", None), ("std_d2048", None),
          ("decode_d7168", 1), ("decode_d7168", 8), ("decode_d7168", 32), ("decode_d7168", 128))
# B200 datasheet figures (dense bf16 tensor, HBM3e), beside the measured peaks
SPEC_TFLOPS, SPEC_GBS = 2250.0, 7700.0


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default=None, help="one workload only (default: the headline and the others)")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--gemm", type=int, default=0, help="0 tensor cores, 1 CUDA cores")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--graph", action="store_true", help="also time the forward replayed from a CUDA graph")
    ap.add_argument("--save", default=None, help="directory for one JSON file per workload line")
    ap.add_argument("--launch-check", action="store_true",
                    help="CPU only: start the ranks, time a trivial step per rank over gloo and print the line "
                         "(checks the multi-rank launch and aggregation without a GPU)")
    return ap.parse_args(argv)


def source_hash():
    """Hash of the GEMM and planner sources a traffic capture was taken from."""
    import hashlib
    h = hashlib.sha256()
    for f in ("latent_space_routed_b200/csrc/gemm_tc.cu", "latent_space_routed_b200/csrc/lmoe_api.cu"):
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload, T, kernel):
    """DRAM bytes per launch of `kernel` at T tokens from profiles/traffic.json
    (ncu dram__bytes_read.sum + dram__bytes_write.sum), or None when no entry
    matches or the kernel sources changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
            entries = json.load(fh)["entries"]
    except (OSError, ValueError, KeyError):
        return None
    sha = source_hash()
    for e in entries:
        if e["workload"] == workload and e["T"] == T and e["kernel"] == kernel:
            return int(e["bytes_per_launch"]) if e["sources"] == sha else None
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- algorithmic model
def layer_flops(w, T):
    """2dE + 4dl + 6klf + 12 d f_s per token (router, projections, routed, shared);
    no projection term for the standard MoE (l = d, no W_down / W_up)."""
    proj = 0 if w.standard else 4 * w.d * w.l
    return T * (2 * w.d * w.E + proj + 6 * w.k * w.l * w.f + 12 * w.d * w.f_s)


def layer_bytes(w, T, touched):
    B = w.item_bytes
    proj = 0 if w.standard else 2 * w.d * w.l * B
    weights = touched * 3 * w.l * w.f * B + 6 * w.d * w.f_s * B + proj + 4 * w.d * w.E
    io = T * w.d * B * 2 + T * w.k * (4 + B) + T * w.l * B
    return weights + io


def stage_model(w, T, touched):
    """Per-kernel algorithmic (flops, bytes): operands read once, results written once."""
    B, S = w.item_bytes, T * w.k
    kf = 2 * w.f_s + (0 if w.standard else w.l)     # final GEMM's K ([h_s | n], or h_s + u added)
    return {
        "router": (2 * T * w.d * w.E, T * w.d * B + 4 * w.d * w.E + 4 * T * w.E),
        "topk": (0, 4 * T * w.E + T * w.k * (8 + B)),
        "scan": (0, 0),
        "dispatch": (0, T * w.k * 16),
        "down_proj": (0, 0) if w.standard else (2 * T * w.d * w.l, T * w.d * B + w.l * w.d * B + T * w.l * B),
        "permute": (0, T * w.l * B + S * w.l * B + S * 4),
        "gate_up": (2 * S * 2 * w.f * w.l, touched * 2 * w.f * w.l * B + S * w.l * B + S * w.f * B),
        "down_combine": (2 * S * w.l * w.f, touched * w.l * w.f * B + S * w.f * B + S * w.l * B),
        "combine_norm": (0, S * w.l * B + (1 if w.standard else 2) * T * w.l * B),
        "shared_gate_up": (2 * T * w.d * 4 * w.f_s, T * w.d * B + 4 * w.f_s * w.d * B + T * 2 * w.f_s * B),
        "final": (2 * T * w.d * kf,
                  T * kf * B + w.d * kf * B + T * w.d * B + (T * w.d * B if w.standard else 0)),
    }


# ---------------------------------------------------------------- ranks
def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank float over the process group (the job's time is its
    slowest rank's); the value itself when there is no group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, T: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own T-token batch per step."""
    return world * T / (ms_per_step / 1e3)


def replica_seed(w, rank: int) -> int:
    """Each replica draws its own token batch (same weights)."""
    return w.seed + 1000 * rank


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launcher_cmd(argv, gpus: int, port: int):
    """torch.distributed.run command that starts `gpus` ranks of this script."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


# ---------------------------------------------------------------- clocks
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(gpu_id), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle timing
def time_oracle(w, x, W, seconds, max_rows=None):
    """Time the fp64 oracle on a bounded, seeded sample of token rows."""
    import numpy as np
    import oracle
    cores = len(os.sched_getaffinity(0))
    T = x.shape[0]
    rng = np.random.default_rng(7)
    n0 = min(cores, T)
    t0 = time.perf_counter()
    oracle.forward(x, W, w.k, rows=rng.choice(T, n0, replace=False), eps=w.eps, use_norm=not w.standard)
    dt0 = time.perf_counter() - t0
    n = int(max(n0, min(T if max_rows is None else max_rows, n0 * seconds / max(dt0, 1e-6))))
    rows = rng.choice(T, n, replace=False)
    t1 = time.perf_counter()
    oracle.forward(x, W, w.k, rows=rows, eps=w.eps, use_norm=not w.standard)
    dt = time.perf_counter() - t1
    return n / dt, n, dt, cores


def run_reference(args, rank, world):
    if rank != 0:
        return
    import lmoe_inputs as li
    w = li.WORKLOADS[args.workload or HEADLINE]
    T = args.T or w.T
    x, W = li.tokens(w, T), li.weights(w)
    # one step = the oracle on a bounded sample of rows, sized to ~4 s
    _, n, _, cores = time_oracle(w, x, W, 4.0)
    import numpy as np
    import oracle
    rng = np.random.default_rng(11)
    times = []
    for i in range(args.warmup + args.steps):
        rows = rng.choice(T, n, replace=False)
        t0 = time.perf_counter()
        oracle.forward(x, W, w.k, rows=rows, eps=w.eps, use_norm=not w.standard)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = n / per_step
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "T": T, "d": w.d, "l": w.l, "f": w.f, "E": w.E, "k": w.k,
                       "f_shared": w.f_s, "sample_rows_per_step": n},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{n} seeded token rows of {T} per step (fp64 C oracle, threads over rows)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- own arm
def _roofline(fl, by, ms, hbm, tf):
    """Roofline object of `ms` per launch for fl FLOPs and by bytes."""
    t_s = ms / 1e3
    if fl / (tf * 1e12) >= by / (hbm * 1e9):
        r = {"bound": "tensor", "achieved": fl / t_s / 1e12, "peak": tf, "unit": "TFLOP/s",
             "frac_of_spec": fl / t_s / 1e12 / SPEC_TFLOPS}
    else:
        r = {"bound": "hbm", "achieved": by / t_s / 1e9, "peak": hbm, "unit": "GB/s",
             "frac_of_spec": by / t_s / 1e9 / SPEC_GBS}
    r["frac"] = r["achieved"] / r["peak"]
    return r


def measure(args, w, T, layer, x_cpu, W, rank, world, dev, *, headline):
    """Time one workload at T tokens on an existing layer; returns the full line."""
    import torch
    import latent_space_routed_b200 as lm

    x = x_cpu.to(dev)
    out = layer.empty_outputs(T)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    # warm-up (also yields the realised touched-expert count)
    for _ in range(max(args.warmup, 3)):
        layer.forward_into(x, out)
    torch.cuda.synchronize()
    layer.check_device(T)
    counts = layer.region(T, "counts", torch.int32, (w.E,)).cpu().numpy()
    touched = int((counts > 0).sum())
    # host cost of one call (enqueue only): tells whether small batches starve the GPU
    torch.cuda.synchronize()
    t_h = time.perf_counter()
    for _ in range(10):
        layer.forward_into(x, out)
    host_us = (time.perf_counter() - t_h) / 10 * 1e6
    torch.cuda.synchronize()

    ns = lm.LMOE_NUM_STAGES + 1
    ev_stage = [[torch.cuda.Event(enable_timing=True) for _ in range(ns)] for _ in range(args.steps)]
    for evs in ev_stage:   # materialise the events on this device before taking their handles
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    arrays = [(ctypes.c_void_p * ns)(*[e.cuda_event for e in evs]) for evs in ev_stage]
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = dev.index
    clocks = Clocks(gpu_id)
    time.sleep(0.5)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))                      # evict L2 between timed steps (untimed)
        ev_a[i].record(stream)
        layer.forward_into(x, out)
        ev_b[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    layer.check_device(T)
    step_ms = [a.elapsed_time(b) for a, b in zip(ev_a, ev_b)]
    total_ms = max_over_ranks(sum(step_ms), dev)

    # Per-stage breakdown: the same steps again with stage events set, under
    # which the library runs every stage on one stream in order (no overlap).
    for i in range(args.steps):
        flush.fill_(float(i))
        lm.lmoe_set_stage_events(layer.handle, arrays[i], ns)
        layer.forward_into(x, out)
    torch.cuda.synchronize()
    lm.lmoe_set_stage_events(layer.handle, None, 0)
    layer.check_device(T)
    stage_ms = {}
    for si, name in enumerate(lm.STAGE_NAMES):
        stage_ms[name] = sum(ev_stage[i][si].elapsed_time(ev_stage[i][si + 1]) for i in range(args.steps)) / args.steps
    serial_ms = sum(ev_stage[i][0].elapsed_time(ev_stage[i][ns - 1]) for i in range(args.steps)) / args.steps

    graph_ms = None
    if args.graph or T <= 128:
        # the same forward captured once into a CUDA graph and replayed (no host launch gaps)
        layer.workspace(T)
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            layer.forward_into(x, out, stream=side)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.forward_into(x, out, stream=torch.cuda.current_stream())
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        g_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        g_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        for i in range(args.steps):
            flush.fill_(float(i))
            g_a[i].record(stream)
            graph.replay()
            g_b[i].record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(g_a, g_b)), dev) / args.steps
        del graph
        layer.check_device(T)

    # end to end through the public API: pinned host x in, host outputs back, copies inside the timing
    x_host = x_cpu.pin_memory()
    out_host = layer.empty_outputs(T, device="cpu", pin=True)
    for _ in range(2):
        layer.forward_host(x_host, out_host)
    torch.cuda.synchronize()
    e_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    for i in range(args.steps):
        flush.fill_(float(i))
        e_a[i].record(stream)
        layer.forward_host(x_host, out_host)
        e_b[i].record(stream)
    torch.cuda.synchronize()
    layer.check_device_host(T)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e_a, e_b)), dev)
    B = w.item_bytes
    h2d = T * w.d * B
    d2h = T * w.d * B + T * w.k * 4 + T * w.k * B + T * w.l * B
    del x, out, flush, x_host, out_host

    if rank != 0:
        return None

    hbm, tf_burst, tf_sus, peak_src = peaks()
    ms = total_ms / args.steps
    value = job_tokens_per_s(world, T, ms)
    model = stage_model(w, T, touched)
    dom = max(stage_ms, key=lambda k: stage_ms[k])
    fl, by = model[dom]
    roof = _roofline(fl, by, stage_ms[dom], hbm, tf_burst)
    roof["traffic"] = measured_traffic(w.name, T, dom)
    roof["kernel"] = dom
    roof["per_launch"] = {"flops": fl, "bytes": by, "ms": stage_ms[dom]}
    roof["peak_source"] = (f"{peak_src} (MEASURED_PEAKS.json burst bf16 / copy bandwidth); "
                           f"frac_of_spec against the B200 datasheet {SPEC_TFLOPS:.0f} TFLOP/s / {SPEC_GBS:.0f} GB/s")
    Lf, Lb = layer_flops(w, T), layer_bytes(w, T, touched)
    t_roof = max(Lf / (tf_burst * 1e12), Lb / (hbm * 1e9))
    bound = "tensor" if Lf / (tf_burst * 1e12) >= Lb / (hbm * 1e9) else "hbm"
    layer_roof = {"flops": Lf, "bytes": Lb, "roofline_ms": t_roof * 1e3, "frac": t_roof / (ms / 1e3),
                  "bound": bound, "achieved_tflops": Lf / (ms / 1e3) / 1e12, "achieved_gbs": Lb / (ms / 1e3) / 1e9,
                  "frac_of_sustained_tensor": (Lf / (tf_sus * 1e12)) / (ms / 1e3) if tf_sus else None,
                  "frac_of_spec": max(Lf / (SPEC_TFLOPS * 1e12), Lb / (SPEC_GBS * 1e9)) / (ms / 1e3)}
    # the two routed expert GEMMs together: the touched experts' weights (the
    # decode workload's figure of merit) and all their algorithmic bytes
    r_ms = stage_ms["gate_up"] + stage_ms["down_combine"]
    r_weights = touched * 3 * w.l * w.f * w.item_bytes
    r_bytes = model["gate_up"][1] + model["down_combine"][1]
    routed = {"ms": r_ms, "touched_experts": touched, "weight_bytes": r_weights, "bytes": r_bytes,
              "weight_gbs": r_weights / (r_ms / 1e3) / 1e9, "all_gbs": r_bytes / (r_ms / 1e3) / 1e9,
              "weight_frac_of_hbm": r_weights / (r_ms / 1e3) / 1e9 / hbm}

    cpu = None
    if headline and not args.no_cpu_baseline and world == 1:
        v, n, dt, cores = time_oracle(w, x_cpu, W, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n} seeded token rows of the {T}-token batch in {dt:.1f} s (fp64 C oracle)"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,1) tokens, N(0,1/fan_in) weights)",
            "config": {"workload": w.name, "T": T, "d": w.d, "l": w.l, "f": w.f, "E": w.E, "k": w.k,
                       "f_shared": w.f_s, "touched_experts": touched,
                       "gemm": "tcgen05" if (args.gemm == 0 and w.dtype == "bf16") else "cuda-cores",
                       "l2": "flushed between timed steps (256 MiB write, untimed)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": roof, "layer_roofline": layer_roof, "routed": routed,
            "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "stages_note": "stages timed in a second pass with stage events set (one stream, no overlap)",
            "serial_ms_per_step": round(serial_ms, 4),
            "cpu_baseline": cpu,
            "e2e": {"value": job_tokens_per_s(world, T, e2e_ms / args.steps), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": layer.launch_count(T) * args.steps, "clocks": clk,
            "host_us_per_call": host_us}
    if graph_ms is not None:
        line["graph"] = {"ms_per_step": graph_ms, "value": world * T / (graph_ms / 1e3), "unit": UNIT,
                         "layer_frac": t_roof / (graph_ms / 1e3)}
    return line


def summary(line):
    """The per-workload entry of the headline line's `workloads` object."""
    s = {"T": line["config"]["T"], "ms_per_step": line["ms_per_step"], "tokens_per_s": line["value"],
         "layer_frac": line["layer_roofline"]["frac"], "layer_bound": line["layer_roofline"]["bound"],
         "dominant_kernel": line["roofline"]["kernel"], "dominant_kernel_frac": line["roofline"]["frac"],
         "routed_weight_gbs": line["routed"]["weight_gbs"],
         "routed_weight_frac_of_hbm": line["routed"]["weight_frac_of_hbm"],
         "e2e_tokens_per_s": line["e2e"]["value"], "clocks": line["clocks"]}
    if "graph" in line:
        s["graph_ms_per_step"] = line["graph"]["ms_per_step"]
        s["graph_layer_frac"] = line["graph"]["layer_frac"]
    return s


def _save(args, line):
    if not args.save:
        return
    os.makedirs(args.save, exist_ok=True)
    c = line["config"]
    name = f"bench_{c['workload']}" + (f"_T{c['T']}" if c["workload"] == "decode_d7168" else "") + ".json"
    with open(os.path.join(args.save, name), "w") as fh:
        json.dump(line, fh, indent=1)


def run_own(args, rank, world, local_rank):
    import torch
    import lmoe_inputs as li
    import latent_space_routed_b200 as lm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.workload:
        plan = [(args.workload, [args.T])]
        headline = args.workload
    else:
        plan = [(HEADLINE, [None])]
        for name, T in OTHERS:
            if plan[-1][0] == name:
                plan[-1][1].append(T)
            else:
                plan.append((name, [T]))
        headline = HEADLINE
    lines = []
    for name, Ts in plan:
        w = li.WORKLOADS[name]
        W = li.weights(w)
        layer = lm.LatentMoE(lm.config_for(w, gemm=args.gemm), {k: v.to(dev) for k, v in W.items()})
        torch.cuda.empty_cache()   # the caller-side weight copies are no longer needed (the handle repacked them)
        for T in Ts:
            T = T or w.T
            x_cpu = li.tokens(w, T, seed=replica_seed(w, rank))
            line = measure(args, w, T, layer, x_cpu, W, rank, world, dev, headline=(name == headline and not lines))
            if line is not None:
                _save(args, line)
                lines.append(line)
        layer.close()
        del layer, W
        torch.cuda.empty_cache()
    if rank != 0:
        return
    head = lines[0]
    if len(lines) > 1:
        head["workloads"] = {}
        for ln in lines[1:]:
            c = ln["config"]
            key = c["workload"] + (f"_T{c['T']}" if c["workload"] == "decode_d7168" else "")
            head["workloads"][key] = summary(ln)
    print(json.dumps(head), flush=True)


def run_launch_check(args, rank, world):
    """The multi-rank plumbing on CPU ranks over gloo: barrier, a trivial timed
    step per rank, max over ranks, the whole-job aggregate."""
    import datetime
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        T = 1024
        if world > 1:
            dist.barrier()
        t0 = time.perf_counter()
        a = torch.ones(256, 256)
        for _ in range(args.steps):
            a = a @ a * 1e-3
        per_rank_ms = (time.perf_counter() - t0) * 1e3 + 5.0 * rank
        job_ms = max_over_ranks(per_rank_ms, "cpu")
        if rank == 0:
            print(json.dumps({"metric": METRIC, "launch_check": True, "n_gpus": world, "rank_ms": per_rank_ms,
                              "job_ms": job_ms, "value": job_tokens_per_s(world, T, job_ms / args.steps),
                              "unit": UNIT, "steps": args.steps, "warmup": args.warmup}), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse(argv)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # started as a plain script with --gpus N: start the N ranks here
        r = subprocess.run(launcher_cmd(argv, args.gpus, _free_port()))
        sys.exit(r.returncode)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.launch_check:
        run_launch_check(args, rank, world)
        return
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import datetime
    import torch
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_own(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
