"""fp64 CPU oracle for the LatentMoE layer forward (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``latent_space_routed_b200``) never does, and this package never imports the
product: the two share nothing but the seeded input generator ``lmoe_inputs``.

The arithmetic lives in ``lmoe_oracle.c`` (plain fp64 loops, threads over
token rows); this module builds it with gcc, marshals numpy/torch CPU arrays
into it, and adds two closed forms written out from the cooking-agi LatentMoE
page:

* ``latent_budget`` -- section "Does the saving pay for more experts?":
  parameters = E * 3 l f + 2 d l (no projections when l == d),
  MACs per token = k * 3 l f + 2 d l, slot bytes = 2 T k l B.
* ``fixed_cutoff_bias`` -- section "Quantile Balancing: measure now, use next
  step": the bias that leaves exactly ``target`` positive margins is minus the
  target-th largest margin (0-based after a descending sort).
* ``qb_cutoff``, ``qb_margin_histogram``, ``qb_quantile_from_histogram`` --
  the same section's statistics: the (k+1)-th biased score per token as the
  cutoff, per-expert margin histograms, and the histogram estimate of the
  quantile that fixed_cutoff_bias takes exactly.

Pins (tests/test_oracle.py): the worked example and the shape examples of
"Stable LatentMoE"; routed_example, the norm-order example, the latent_budget
and fixed_cutoff_bias assertions of the cooking-agi page; brute-force top-k
and cutoffs; margin histograms against a direct count, and their quantile
estimate within one bin of fixed_cutoff_bias;
invariants (sum p = 1, k = E, bias shift, D scaling, row permutation,
stacked shared experts, SiTU -> SwiGLU as the caps grow).  Nothing here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lmoe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liblmoe_oracle.so")

ACT = {"swiglu": 0, "situ": 1, "linear": 2}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) into oracle/_build."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int), ("l", ctypes.c_int), ("f", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("fs", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("eps", ctypes.c_double), ("act", ctypes.c_int), ("gate_cap", ctypes.c_double),
                ("up_cap", ctypes.c_double), ("use_norm", ctypes.c_int), ("n_threads", ctypes.c_int)]


class _Inputs(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("x_dt", ctypes.c_int), ("W_r", ctypes.c_void_p),
                ("b", ctypes.c_void_p), ("W_down", ctypes.c_void_p), ("W_up", ctypes.c_void_p),
                ("G", ctypes.c_void_p), ("U", ctypes.c_void_p), ("D", ctypes.c_void_p),
                ("Gs", ctypes.c_void_p), ("Us", ctypes.c_void_p), ("Ds", ctypes.c_void_p),
                ("w_dt", ctypes.c_int)]


class _Outputs(ctypes.Structure):
    _fields_ = [("y", ctypes.c_void_p), ("sel", ctypes.c_void_p), ("p", ctypes.c_void_p),
                ("u", ctypes.c_void_p), ("r", ctypes.c_void_p), ("gap", ctypes.c_void_p)]


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build())
        lib.ora_forward.restype = ctypes.c_int
        lib.ora_forward.argtypes = [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), ctypes.POINTER(_Outputs),
                                    ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        lib.ora_topk.restype = None
        lib.ora_topk.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p]
        _lib_handle = lib
    return _lib_handle


def _as_storage(a, name):
    """Return (contiguous numpy array, dtype code): fp32 -> 0, bf16 bits -> 1.

    Accepts numpy float32 arrays, or torch CPU tensors of float32 / bfloat16
    (bf16 is passed as its raw 16-bit patterns, widened exactly in C).
    """
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), 1
            if a.dtype == torch.float32:
                return a.numpy(), 0
            raise TypeError(f"{name}: unsupported torch dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.float64:
        # Only exact fp32 values are accepted, so the oracle sees what the GPU sees.
        a32 = a.astype(np.float32)
        if not np.array_equal(a32.astype(np.float64), a):
            raise ValueError(f"{name}: float64 input is not exactly representable in fp32")
        return a32, 0
    if a.dtype == np.uint16:
        return a, 1
    raise TypeError(f"{name}: unsupported dtype {a.dtype}")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def forward(x, w: Dict, k: int, *, eps: float = 1e-6, act: str = "swiglu", gate_cap: float = 4.0,
            up_cap: float = 25.0, use_norm: bool = True, rows: Optional[Sequence[int]] = None,
            sel: Optional[np.ndarray] = None, threads: int = 0) -> Dict[str, np.ndarray]:
    """Run the oracle.

    x [T, d]; w holds W_r [E, d] fp32, b [E] fp32, W_down [l, d], W_up [d, l],
    G, U [E, f, l], D [E, l, f], Gs, Us [n_shared, f_s, d], Ds [n_shared, d, f_s]
    (all weights other than W_r and b in one dtype).  ``rows`` restricts the
    evaluation to those token rows (outputs are compact, in that order);
    ``sel`` [n, k] replaces the top-k selection.  Returns fp64 arrays
    ``output``, ``mixture_weights``, ``latent_routed_aggregate``, ``scores``
    (raw r), ``gap`` (s_(k) - s_(k+1)) and int32 ``selected_experts``.
    """
    lib = _lib()
    xs, x_dt = _as_storage(x, "x")
    T, d = xs.shape
    W_r, _ = _as_storage(w["W_r"], "W_r")
    b, _ = _as_storage(w["b"], "b")
    if W_r.dtype != np.float32 or b.dtype != np.float32:
        raise TypeError("W_r and b must be fp32")
    arrs = {}
    w_dt = None
    for name in ("W_down", "W_up", "G", "U", "D", "Gs", "Us", "Ds"):
        arrs[name], dt = _as_storage(w[name], name)
        if w_dt is None:
            w_dt = dt
        elif dt != w_dt:
            raise TypeError("all expert/projection weights must share one dtype")
    E = W_r.shape[0]
    l = arrs["W_down"].shape[0]
    f = arrs["G"].shape[1]
    n_shared, fs = arrs["Gs"].shape[0], arrs["Gs"].shape[1]
    shapes = {"W_r": (E, d), "b": (E,), "W_down": (l, d), "W_up": (d, l), "G": (E, f, l), "U": (E, f, l),
              "D": (E, l, f), "Gs": (n_shared, fs, d), "Us": (n_shared, fs, d), "Ds": (n_shared, d, fs)}
    for name, shp in shapes.items():
        got = (W_r if name == "W_r" else b if name == "b" else arrs[name]).shape
        if tuple(got) != shp:
            raise ValueError(f"{name}: shape {tuple(got)} != {shp}")
    if not (1 <= k <= E):
        raise ValueError("k must satisfy 1 <= k <= E")

    rows_arr = None
    n = T
    if rows is not None:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n = rows_arr.shape[0]
    sel_arr = None
    if sel is not None:
        sel_arr = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
        if sel_arr.shape != (n, k):
            raise ValueError("sel must be [n, k]")
        if sel_arr.size and (sel_arr.min() < 0 or sel_arr.max() >= E):
            raise ValueError("sel out of range")

    dims = _Dims(T, d, l, f, E, k, fs, n_shared, eps, ACT[act], gate_cap, up_cap, int(use_norm), threads)
    ins = _Inputs(_ptr(xs).value, x_dt, _ptr(W_r).value, _ptr(b).value, _ptr(arrs["W_down"]).value,
                  _ptr(arrs["W_up"]).value, _ptr(arrs["G"]).value, _ptr(arrs["U"]).value,
                  _ptr(arrs["D"]).value, _ptr(arrs["Gs"]).value, _ptr(arrs["Us"]).value,
                  _ptr(arrs["Ds"]).value, w_dt)
    y = np.zeros((n, d), np.float64)
    sel_out = np.zeros((n, k), np.int32)
    p = np.zeros((n, k), np.float64)
    u = np.zeros((n, l), np.float64)
    r = np.zeros((n, E), np.float64)
    gap = np.zeros((n,), np.float64)
    outs = _Outputs(_ptr(y).value, _ptr(sel_out).value, _ptr(p).value, _ptr(u).value, _ptr(r).value,
                    _ptr(gap).value)
    rc = lib.ora_forward(ctypes.byref(dims), ctypes.byref(ins), ctypes.byref(outs),
                         None if rows_arr is None else _ptr(rows_arr), n,
                         None if sel_arr is None else _ptr(sel_arr))
    if rc != 0:
        raise ValueError("ora_forward rejected its arguments")
    return {"output": y, "selected_experts": sel_out, "mixture_weights": p, "latent_routed_aggregate": u,
            "scores": r, "gap": gap}


def topk(s: np.ndarray, k: int):
    """Top-k of each row of s [n, E] (fp64): indices in selection order
    (score descending, equal scores to the lower index) and s_(k) - s_(k+1)."""
    s = np.ascontiguousarray(np.asarray(s, dtype=np.float64))
    n, E = s.shape
    if not (1 <= k <= E):
        raise ValueError("k must satisfy 1 <= k <= E")
    sel = np.zeros((n, k), np.int32)
    gap = np.zeros((n,), np.float64)
    _lib().ora_topk(n, E, k, _ptr(s), _ptr(sel), _ptr(gap))
    return sel, gap


def latent_budget(width, latent, intermediate, experts, top_k, tokens, item_bytes):
    """Closed-form budget of the cooking-agi LatentMoE page, section "Does the
    saving pay for more experts?".  Each SwiGLU expert l -> f -> l holds 3 l f
    weights; the two projections hold 2 d l unless l == d (standard MoE)."""
    values = (width, latent, intermediate, experts, top_k, tokens, item_bytes)
    for v in values:
        if type(v) is not int or v < 1:
            raise ValueError("dimensions and counts must be positive integers")
    if latent > width or top_k > experts:
        raise ValueError("latent must not exceed width and top_k must not exceed experts")
    proj = 0 if latent == width else 2 * width * latent
    expert = 3 * latent * intermediate
    return {"parameters": experts * expert + proj,
            "mac_per_token": top_k * expert + proj,
            "slot_bytes": 2 * tokens * top_k * latent * item_bytes}


def qb_cutoff(s, k: int) -> np.ndarray:
    """Quantile-Balancing cutoff per token (cooking-agi LatentMoE page, section
    "Quantile Balancing: measure now, use next step"): the (k+1)-th largest
    biased score s = r + b of each row of s [T, E]; -inf when k = E (nothing is
    left unselected).  Works in s's own dtype (the selection is exact)."""
    s = np.asarray(s)
    T, E = s.shape
    if not 1 <= k <= E:
        raise ValueError("k must satisfy 1 <= k <= E")
    if k == E:
        return np.full(T, -np.inf, dtype=s.dtype)
    return -np.partition(-s, k, axis=1)[:, k]


def qb_margin_histogram(s, cutoff, bins: int, lo: float, hi: float) -> np.ndarray:
    """Per-expert histogram [E, bins] (int64) of the margins m[t, e] = s[t, e] -
    cutoff[t] (the page: expert-wise score margins against the current cutoff,
    "global quantiles are approximated with histograms").  Bin j covers
    [lo + j w, lo + (j + 1) w), w = (hi - lo) / bins; margins below lo count in
    bin 0 and margins at or above hi in bin bins - 1.  The bin of a margin is
    floor((m - lo) * (bins / (hi - lo))), each operation rounded in s's dtype
    (pass fp32 scores to take the decision in fp32)."""
    s = np.asarray(s)
    dt = s.dtype.type
    if bins < 1 or not hi > lo:
        raise ValueError("need bins >= 1 and hi > lo")
    T, E = s.shape
    inv_w = dt(dt(bins) / (dt(hi) - dt(lo)))
    hist = np.zeros((E, bins), np.int64)
    for t in range(T):
        for e in range(E):
            m = dt(s[t, e] - dt(cutoff[t]))
            x = dt(dt(m - dt(lo)) * inv_w)
            j = 0 if x < 0 else (bins - 1 if x >= bins else int(np.floor(x)))
            hist[e, j] += 1
    return hist


def qb_quantile_from_histogram(hist, target: int, lo: float, hi: float) -> np.ndarray:
    """Per expert, the histogram estimate of the target-th largest margin
    (0-based, the value fixed_cutoff_bias takes from sorted margins): scanning
    bins from the top with C the count in the bins above bin j, the value lies
    in the bin j with C <= target < C + h_j, and is placed at the upper edge of
    that bin minus (target - C + 1/2) / h_j of its width (the centre of its
    rank inside the bin).  Experts whose total count is <= target get lo.  The
    next step's bias is b - q (fp64)."""
    hist = np.asarray(hist, dtype=np.int64)
    E, bins = hist.shape
    w = (hi - lo) / bins
    q = np.full(E, float(lo))
    for e in range(E):
        above = 0
        for j in range(bins - 1, -1, -1):
            h = int(hist[e, j])
            if above <= target < above + h:
                q[e] = lo + (j + 1) * w - w * (target - above + 0.5) / h
                break
            above += h
    return q


def fixed_cutoff_bias(margins, target):
    """Quantile-Balancing bias from fixed margins (cooking-agi LatentMoE page,
    "Quantile Balancing: measure now, use next step"): with the margins sorted
    descending, the bias is minus the margin at 0-based position ``target``,
    so exactly ``target`` margins stay positive when they are distinct."""
    import math
    if not margins or any(not math.isfinite(float(m)) for m in margins):
        raise ValueError("margins must be finite and non-empty")
    if type(target) is not int or not 0 < target < len(margins):
        raise ValueError("target must be an integer strictly between 0 and len(margins)")
    return -sorted(margins, reverse=True)[target]
