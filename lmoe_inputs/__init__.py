"""Seeded synthetic inputs for the LatentMoE layer forward.

This module is shared by the fp64 oracle (``oracle/``) and the CUDA path
(``latent_space_routed_b200``).  It holds none of the layer's arithmetic: it
only draws random numbers, rounds them once to the storage dtype, and names the
workloads.  Both sides consume exactly the tensors returned here, so the
comparison between them carries no input-quantisation error.

Workloads (shapes from the LatentMoE description, "Stable LatentMoE" problem
and the PyPI ``latent_moe`` README configuration block):

* ``tiny_fp32``      T=256,   d=128,  l=64,   f=256,  E=16,  k=4,  f_s=256,  fp32
* ``acc_d2048``      T=4096,  d=2048, l=512,  f=1408, E=256, k=24, f_s=1408, bf16
  (README defaults d=2048, m=1408, N=64, K=6, alpha=4, variant "acc":
  E = alpha*N = 256, k = alpha*K = 24)
* ``eff_zipf_d2048`` T=16384, same dims, k=6 (variant "eff"), Zipf-skewed bias
* ``large_d4096``    T=32768, d=4096, l=1024, f=2688, E=512, k=24, f_s=2688, bf16
* ``decode_d7168``   T in {1, 8, 32, 128}, d=7168, l=1792, f=2048, E=384, k=32,
  f_s=2048, bf16, zero bias

Value recipe: tokens ~ N(0, 1); every weight ~ N(0, 1/fan_in) with fan_in its
input width (d for W_r, W_down, shared gate/up; l for routed gate/up and
W_up; f for routed down; f_s for shared down); selection bias
b ~ U(-0.05, 0.05), or b_i = 0.3 / rank_i over a seeded random permutation of
the experts (Zipf skew), or zero.  The router weight W_r and the bias are
always fp32 ("fp32 router"); the rest use the workload dtype, rounded
round-to-nearest-even from fp32 draws.

Every tensor (and every expert slice of the expert stacks) draws from its own
``torch.Generator`` seeded from (workload seed, tensor id, slice index), so any
subset can be regenerated independently and in any order.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    l: int
    f: int
    E: int
    k: int
    f_s: int
    dtype: str          # "f32" or "bf16": token and expert-weight storage
    bias: str           # "uniform" | "zipf" | "zero"
    seed: int
    n_shared: int = 2
    eps: float = 1e-6
    T_sweep: Sequence[int] = ()
    standard: bool = False  # the standard MoE (l = d, no projections, no norm)

    def with_T(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def item_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS: Dict[str, Workload] = {
    "tiny_fp32": Workload("tiny_fp32", 256, 128, 64, 256, 16, 4, 256, "f32", "uniform", 0),
    "acc_d2048": Workload("acc_d2048", 4096, 2048, 512, 1408, 256, 24, 1408, "bf16", "uniform", 1),
    "eff_zipf_d2048": Workload("eff_zipf_d2048", 16384, 2048, 512, 1408, 256, 6, 1408, "bf16", "zipf", 2),
    "large_d4096": Workload("large_d4096", 32768, 4096, 1024, 2688, 512, 24, 2688, "bf16", "uniform", 3),
    "decode_d7168": Workload("decode_d7168", 128, 7168, 1792, 2048, 384, 32, 2048, "bf16", "zero", 4,
                             T_sweep=(1, 8, 32, 128)),
    # the standard MoE that acc_d2048 is derived from (alpha = 4: 64 experts,
    # top 6, experts at the model width): the comparison the pages make
    "std_d2048": Workload("std_d2048", 4096, 2048, 2048, 1408, 64, 6, 1408, "bf16", "uniform", 5,
                          standard=True),
}


def custom(name: str, T: int, d: int, l: int, f: int, E: int, k: int, f_s: int,
           dtype: str = "bf16", bias: str = "uniform", seed: int = 100, standard: bool = False) -> Workload:
    """A workload with arbitrary sizes (used for multi-tile / ragged tests)."""
    return Workload(name, T, d, l, f, E, k, f_s, dtype, bias, seed, standard=standard)


# Tensor ids: fixed forever so that stored expected values stay valid.
_TID = {"x": 1, "W_r": 2, "b": 3, "W_down": 4, "W_up": 5, "G": 6, "U": 7, "D": 8,
        "Gs": 9, "Us": 10, "Ds": 11, "b_perm": 12}


def _gen(seed: int, tid: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed((seed * 1_000_003 + tid * 10_007 + sub) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, std: float, g: torch.Generator, dtype: torch.dtype) -> torch.Tensor:
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _stack(n: int, shape, std: float, seed: int, tid: int, dtype: torch.dtype) -> torch.Tensor:
    """n slices, each from its own generator; slices are drawn on a thread pool
    (torch releases the GIL), which leaves every value unchanged."""
    import concurrent.futures as cf
    import os

    out = torch.empty((n,) + tuple(shape), dtype=dtype)

    def one(i):
        out[i] = _normal(shape, std, _gen(seed, tid, i), dtype)

    def worker(i):
        torch.set_num_threads(1)      # in the worker thread: no nested intra-op pools
        one(i)

    workers = min(n, len(os.sched_getaffinity(0)), 32)
    if workers <= 1 or n * math.prod(shape) < (1 << 22):
        for i in range(n):
            one(i)
        return out
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(worker, range(n)))
    return out


def tokens(w: Workload, T: Optional[int] = None, seed: Optional[int] = None) -> torch.Tensor:
    """x [T, d] ~ N(0, 1) in the workload dtype (CPU)."""
    T = w.T if T is None else T
    s = w.seed if seed is None else seed
    return _normal((T, w.d), 1.0, _gen(s, _TID["x"], T), w.torch_dtype)


def bias(w: Workload) -> torch.Tensor:
    """Selection bias b [E] fp32."""
    if w.bias == "zero":
        return torch.zeros(w.E, dtype=torch.float32)
    if w.bias == "uniform":
        g = _gen(w.seed, _TID["b"])
        return (torch.rand(w.E, generator=g, dtype=torch.float64) * 0.1 - 0.05).to(torch.float32)
    if w.bias == "zipf":
        g = _gen(w.seed, _TID["b_perm"])
        perm = torch.randperm(w.E, generator=g)
        ranks = torch.arange(1, w.E + 1, dtype=torch.float64)
        b = torch.empty(w.E, dtype=torch.float64)
        b[perm] = 0.3 / ranks
        return b.to(torch.float32)
    raise ValueError(f"unknown bias recipe {w.bias!r}")


def weights(w: Workload) -> Dict[str, torch.Tensor]:
    """All layer weights on the CPU, in the layouts the library takes.

    Layout is "out x in" (row-major, as in W @ x):
    W_r [E, d] fp32, b [E] fp32, W_down [l, d], W_up [d, l],
    G, U [E, f, l], D [E, l, f], Gs, Us [2, f_s, d], Ds [2, d, f_s].
    A standard workload (l = d) carries identity W_down and W_up: the layer
    formula with identity projections and no norm is the standard MoE, so a
    reference can run it as is, while the library skips them.
    """
    dt = w.torch_dtype
    s = w.seed
    if w.standard:
        if w.l != w.d:
            raise ValueError("a standard workload needs l = d")
        eye = torch.eye(w.d, dtype=dt)
        out = weights(dataclasses.replace(w, standard=False, l=1))
        out["W_down"], out["W_up"] = eye, eye.clone()
        out["G"] = _stack(w.E, (w.f, w.l), 1.0 / math.sqrt(w.l), s, _TID["G"], dt)
        out["U"] = _stack(w.E, (w.f, w.l), 1.0 / math.sqrt(w.l), s, _TID["U"], dt)
        out["D"] = _stack(w.E, (w.l, w.f), 1.0 / math.sqrt(w.f), s, _TID["D"], dt)
        return out
    return {
        "W_r": _normal((w.E, w.d), 1.0 / math.sqrt(w.d), _gen(s, _TID["W_r"]), torch.float32),
        "b": bias(w),
        "W_down": _normal((w.l, w.d), 1.0 / math.sqrt(w.d), _gen(s, _TID["W_down"]), dt),
        "W_up": _normal((w.d, w.l), 1.0 / math.sqrt(w.l), _gen(s, _TID["W_up"]), dt),
        "G": _stack(w.E, (w.f, w.l), 1.0 / math.sqrt(w.l), s, _TID["G"], dt),
        "U": _stack(w.E, (w.f, w.l), 1.0 / math.sqrt(w.l), s, _TID["U"], dt),
        "D": _stack(w.E, (w.l, w.f), 1.0 / math.sqrt(w.f), s, _TID["D"], dt),
        "Gs": _stack(w.n_shared, (w.f_s, w.d), 1.0 / math.sqrt(w.d), s, _TID["Gs"], dt),
        "Us": _stack(w.n_shared, (w.f_s, w.d), 1.0 / math.sqrt(w.d), s, _TID["Us"], dt),
        "Ds": _stack(w.n_shared, (w.d, w.f_s), 1.0 / math.sqrt(w.f_s), s, _TID["Ds"], dt),
    }


WEIGHT_NAMES = ("W_r", "b", "W_down", "W_up", "G", "U", "D", "Gs", "Us", "Ds")
