"""Rates behind the tensor-core GEMM's tile shapes, measured on the B200.

``tests/gpu_rates.cu`` (a standalone program) times tcgen05.mma for the
kind::f16 shapes of both CTA groups with one, two or four independent
accumulators in flight (each k-step to every accumulator in turn, or all
k-steps of a slice to one accumulator before the next), and with a commit and
a barrier wait after every 4, 8 or 16 MMAs (the GEMM's per-stage pattern),
and the copy engine's
global -> shared bandwidth (1D bulk and tiled tensor copies) over an
L2-resident and an HBM-sized buffer, with one or two issuing threads and
barrier waits of CTA or cluster scope.  The test builds it with nvcc,
runs it once, prints its JSON lines (``pytest -s`` shows them) and checks that
every bounded wait completed and that the numbers are physically sensible:
the largest shape issues at a rate near the tensor pipe's per-SM peak,
L2-resident copies are at least as fast as HBM-bound ones, and copies waited
for with CTA-scope barrier waits run as fast as with cluster-scope ones
(within 10 %).
"""
import json
import os
import subprocess
import tempfile

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _run_probe():
    src = os.path.join(ROOT, "tests", "gpu_rates.cu")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "gpu_rates")
        subprocess.run([NVCC, "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-o", exe, src],
                       check=True, capture_output=True, text=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    lines = [json.loads(s) for s in r.stdout.splitlines() if s.startswith("{")]
    return r.returncode, lines, r.stderr


def test_mma_and_bulk_copy_rates():
    rc, lines, err = _run_probe()
    for ln in lines:
        print(json.dumps(ln))
    assert rc == 0, err
    done = [ln for ln in lines if ln["probe"] == "done"]
    assert done and done[0]["status"] == 0
    mma = {(ln["cta_group"], ln["M"], ln["N"], ln["nacc"], ln["order"]): ln for ln in lines
           if ln["probe"] == "mma" and ln["commit_every"] == 0}
    # the pair shape the routed GEMMs use: within a factor two of 8192 FLOP
    # per clock per SM (the tensor pipe's nominal dense bf16 rate: 2.25
    # PFLOP/s over 148 SMs near 1.9 GHz)
    best = mma[(2, 256, 256, 1, "interleaved")]["flop_per_clk_per_sm"]
    assert 4096 < best < 8192 * 1.1, best
    bulk = [ln for ln in lines if ln["probe"] == "bulk"]
    l2 = max(ln["GBps"] for ln in bulk if ln["span_bytes"] <= (48 << 20))
    hbm = max(ln["GBps"] for ln in bulk if ln["span_bytes"] > (1 << 30))
    assert l2 >= 0.9 * hbm, (l2, hbm)
    # the GEMM waits on its barriers with CTA-scope acquire semantics: on the
    # same copies that is as fast as cluster-scope waits, within 10 %
    tile = {(ln["wait_scope"], ln["chunk"], ln["stages"], ln["issuers"]): ln["GBps"] for ln in lines
            if ln["probe"] == "tile" and ln["span_bytes"] <= (48 << 20)}
    for key in [k for k in tile if k[0] == "cta"]:
        assert tile[key] >= 0.9 * tile[("cluster",) + key[1:]], (key, tile)
