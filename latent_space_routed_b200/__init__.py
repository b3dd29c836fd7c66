"""Python binding of liblmoe, the sm_100a LatentMoE layer-forward library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels (include/lmoe.h).  PyTorch supplies device memory and streams.  The
functions keep the C names; ``LatentMoE`` is a small convenience wrapper that
owns a handle and a cached workspace and returns the four outputs of the
"Stable LatentMoE" contract as a dict.

Importing fails loudly (ImportError) when the library has not been built:
``python latent_space_routed_b200/build.py``.  There is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "liblmoe.so")

LMOE_OK, LMOE_ERR_INVALID_ARG, LMOE_ERR_UNSUPPORTED, LMOE_ERR_OOM, LMOE_ERR_CUDA, LMOE_ERR_DEVICE_TIMEOUT, \
    LMOE_ERR_WORKSPACE = range(7)
LMOE_F32, LMOE_BF16 = 0, 1
LMOE_ACT_SWIGLU, LMOE_ACT_SITU = 0, 1

STATUS_NAMES = {0: "LMOE_OK", 1: "LMOE_ERR_INVALID_ARG", 2: "LMOE_ERR_UNSUPPORTED", 3: "LMOE_ERR_OOM",
                4: "LMOE_ERR_CUDA", 5: "LMOE_ERR_DEVICE_TIMEOUT", 6: "LMOE_ERR_WORKSPACE"}

# lmoe_workspace_region ids
REGION = {"scores": 0, "p32": 1, "counts": 2, "offsets": 3, "slot_of": 4, "perm_tok": 5, "Z": 6, "H": 7,
          "Y": 8, "HS": 9, "status": 10, "cutoff": 11, "Zp": 12}

EXPORTS = ("lmoe_config_from_base", "lmoe_create", "lmoe_workspace_size", "lmoe_forward", "lmoe_host_workspace_size",
           "lmoe_forward_host", "lmoe_forward_noalloc", "lmoe_debug_inject", "lmoe_set_bias", "lmoe_qb_histogram", "lmoe_qb_bias_update", "lmoe_set_stage_events", "lmoe_launch_count", "lmoe_workspace_region", "lmoe_check_device", "lmoe_check_device_host",
           "lmoe_last_error", "lmoe_destroy")


class LmoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class lmoe_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("l", ctypes.c_int32), ("f", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f_shared", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("eps", ctypes.c_float), ("dtype", ctypes.c_int32), ("act", ctypes.c_int32),
                ("gate_cap", ctypes.c_float), ("up_cap", ctypes.c_float), ("gemm", ctypes.c_int32),
                ("standard", ctypes.c_int32)]


class lmoe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_r", "b", "W_down", "W_up", "G", "U", "D", "Gs", "Us", "Ds")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python latent_space_routed_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "lmoe_config_from_base": (I32, [I32, I32, I32, I32, I32, I32, ctypes.c_char_p, ctypes.POINTER(lmoe_config)]),
        "lmoe_create": (I32, [ctypes.POINTER(lmoe_config), ctypes.POINTER(lmoe_weights), P, ctypes.POINTER(P)]),
        "lmoe_workspace_size": (I32, [P, I64, ctypes.POINTER(SZ)]),
        "lmoe_forward": (I32, [P, P, I64, P, P, P, P, P, SZ, P]),
        "lmoe_host_workspace_size": (I32, [P, I64, ctypes.POINTER(SZ)]),
        "lmoe_forward_host": (I32, [P, P, I64, P, P, P, P, P, SZ, P]),
        "lmoe_forward_noalloc": (I32, [P, P, I64, P, P, P, P, P]),
        "lmoe_debug_inject": (I32, [I32, I32]),
        "lmoe_set_bias": (I32, [P, P, P]),
        "lmoe_qb_histogram": (I32, [P, P, I64, I32, ctypes.c_float, ctypes.c_float, P, P]),
        "lmoe_qb_bias_update": (I32, [P, P, I32, ctypes.c_float, ctypes.c_float, I64, P, P]),
        "lmoe_set_stage_events": (I32, [P, P, I32]),
        "lmoe_launch_count": (I32, [P, I64, ctypes.POINTER(I32)]),
        "lmoe_workspace_region": (I32, [P, I64, I32, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
        "lmoe_check_device": (I32, [P, I64, P, P]),
        "lmoe_check_device_host": (I32, [P, I64, P, P]),
        "lmoe_last_error": (ctypes.c_char_p, []),
        "lmoe_destroy": (None, [P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(status: int):
    if status != LMOE_OK:
        raise LmoeError(status, _lib.lmoe_last_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.data_ptr()
    return int(t)


# ------------------------------------------------------------------ C names
def lmoe_last_error() -> str:
    return _lib.lmoe_last_error().decode()


def lmoe_config_from_base(d, m, N, K, alpha, n_shared, variant) -> lmoe_config:
    cfg = lmoe_config()
    _check(_lib.lmoe_config_from_base(d, m, N, K, alpha, n_shared, variant.encode(), ctypes.byref(cfg)))
    return cfg


def make_config(d, l, f, E, k, f_shared, n_shared=2, eps=1e-6, dtype=LMOE_BF16, act=LMOE_ACT_SWIGLU,
                gate_cap=4.0, up_cap=25.0, gemm=0, standard=0) -> lmoe_config:
    return lmoe_config(d, l, f, E, k, f_shared, n_shared, eps, dtype, act, gate_cap, up_cap, gemm, standard)


def lmoe_create(cfg: lmoe_config, weights: Dict[str, torch.Tensor], stream=None) -> int:
    w = lmoe_weights(*[_ptr(weights.get(n)) for n in ("W_r", "b", "W_down", "W_up", "G", "U", "D", "Gs", "Us", "Ds")])
    h = ctypes.c_void_p()
    _check(_lib.lmoe_create(ctypes.byref(cfg), ctypes.byref(w), _stream(stream), ctypes.byref(h)))
    return h.value


def lmoe_destroy(h: int):
    _lib.lmoe_destroy(h)


def lmoe_workspace_size(h: int, T: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.lmoe_workspace_size(h, T, ctypes.byref(n)))
    return n.value


def lmoe_host_workspace_size(h: int, T: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.lmoe_host_workspace_size(h, T, ctypes.byref(n)))
    return n.value


def lmoe_forward(h, x, T, output, selected_experts, mixture_weights, latent_routed_aggregate, workspace, ws_bytes,
                 stream=None):
    _check(_lib.lmoe_forward(h, _ptr(x), T, _ptr(output), _ptr(selected_experts), _ptr(mixture_weights),
                             _ptr(latent_routed_aggregate), _ptr(workspace), ws_bytes, _stream(stream)))


def lmoe_forward_host(h, x_host, T, output_host, selected_experts_host, mixture_weights_host,
                      latent_routed_aggregate_host, workspace, ws_bytes, stream=None):
    _check(_lib.lmoe_forward_host(h, _ptr(x_host), T, _ptr(output_host), _ptr(selected_experts_host),
                                  _ptr(mixture_weights_host), _ptr(latent_routed_aggregate_host), _ptr(workspace),
                                  ws_bytes, _stream(stream)))


LMOE_NOALLOC_WORKSPACE_BYTES = 64 << 20
LMOE_INJECT_STALL_NEXT_GEMM, LMOE_INJECT_FAIL_ALLOC = 1, 2


def lmoe_debug_inject(what, arg=0):
    """Failure-detection test hooks (see include/lmoe.h)."""
    _check(_lib.lmoe_debug_inject(what, arg))



def lmoe_forward_noalloc(h, x, T, output, selected_experts, mixture_weights, latent_routed_aggregate, stream=None):
    """lmoe_forward on the library's built-in 64 MiB scratch area (no caller
    workspace, no allocation); see include/lmoe.h for its rules."""
    _check(_lib.lmoe_forward_noalloc(h, _ptr(x), T, _ptr(output), _ptr(selected_experts), _ptr(mixture_weights),
                                     _ptr(latent_routed_aggregate), _stream(stream)))


def lmoe_set_bias(h, b, stream=None):
    _check(_lib.lmoe_set_bias(h, _ptr(b), _stream(stream)))


def lmoe_qb_histogram(h, workspace, T, bins, lo, hi, hist, stream=None):
    _check(_lib.lmoe_qb_histogram(h, _ptr(workspace), T, bins, lo, hi, _ptr(hist), _stream(stream)))


def lmoe_qb_bias_update(h, hist, bins, lo, hi, target, bias_out, stream=None):
    _check(_lib.lmoe_qb_bias_update(h, _ptr(hist), bins, lo, hi, target, _ptr(bias_out), _stream(stream)))


LMOE_NUM_STAGES = 11
STAGE_NAMES = ("router", "topk", "scan", "dispatch", "down_proj", "permute", "gate_up", "down_combine",
               "combine_norm", "shared_gate_up", "final")


def lmoe_set_stage_events(h, events, n):
    """events: a ctypes array of cudaEvent_t handles (kept alive by the caller), or None."""
    _check(_lib.lmoe_set_stage_events(h, events, n))


def lmoe_launch_count(h, T) -> int:
    n = ctypes.c_int32()
    _check(_lib.lmoe_launch_count(h, T, ctypes.byref(n)))
    return n.value


def lmoe_workspace_region(h, T, region):
    off, n = ctypes.c_size_t(), ctypes.c_size_t()
    rid = REGION[region] if isinstance(region, str) else int(region)
    _check(_lib.lmoe_workspace_region(h, T, rid, ctypes.byref(off), ctypes.byref(n)))
    return off.value, n.value


def lmoe_check_device(h, T, workspace, stream=None):
    _check(_lib.lmoe_check_device(h, T, _ptr(workspace), _stream(stream)))


def lmoe_check_device_host(h, T, workspace, stream=None):
    _check(_lib.lmoe_check_device_host(h, T, _ptr(workspace), _stream(stream)))


# ------------------------------------------------------------------ convenience wrapper
_TORCH_DT = {LMOE_F32: torch.float32, LMOE_BF16: torch.bfloat16}


class LatentMoE:
    """A LatentMoE layer on the current CUDA device.

    ``weights`` holds W_r [E, d] fp32, b [E] fp32, W_down [l, d], W_up [d, l],
    G, U [E, f, l], D [E, l, f], Gs, Us [2, f_s, d], Ds [2, d, f_s] (CUDA
    tensors; copied and repacked at construction, so they may be freed after).
    ``layer(x)`` with x [..., d] returns the dict of the "Stable LatentMoE"
    contract: output [..., d], selected_experts [..., k] int32,
    mixture_weights [..., k], latent_routed_aggregate [..., l].
    """

    def __init__(self, cfg: lmoe_config, weights: Dict[str, torch.Tensor], stream=None):
        self.cfg = cfg
        self.dtype = _TORCH_DT[cfg.dtype]
        dev = torch.device("cuda", torch.cuda.current_device())
        w = {}
        for n in ("W_r", "b", "W_down", "W_up", "G", "U", "D", "Gs", "Us", "Ds"):
            if cfg.standard and n in ("W_down", "W_up"):
                continue                 # the standard-MoE form has no projections
            want = torch.float32 if n in ("W_r", "b") else self.dtype
            w[n] = weights[n].to(device=dev, dtype=want).contiguous()
        self.handle = lmoe_create(cfg, w, stream)
        self.device = dev
        self._ws = None

    def close(self):
        if getattr(self, "handle", None):
            lmoe_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, T: int, host: bool = False) -> torch.Tensor:
        n = lmoe_host_workspace_size(self.handle, T) if host else lmoe_workspace_size(self.handle, T)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def empty_outputs(self, T: int, device=None, pin: bool = False):
        c = self.cfg
        dev = self.device if device is None else device
        kw = dict(device=dev, pin_memory=pin) if str(dev) == "cpu" else dict(device=dev)
        return {"output": torch.empty(T, c.d, dtype=self.dtype, **kw),
                "selected_experts": torch.empty(T, c.k, dtype=torch.int32, **kw),
                "mixture_weights": torch.empty(T, c.k, dtype=self.dtype, **kw),
                "latent_routed_aggregate": torch.empty(T, c.l, dtype=self.dtype, **kw)}

    def forward_into(self, x: torch.Tensor, out: Dict[str, torch.Tensor], stream=None):
        T = x.shape[0]
        ws = self.workspace(T)
        lmoe_forward(self.handle, x, T, out["output"], out["selected_experts"], out["mixture_weights"],
                     out["latent_routed_aggregate"], ws, ws.numel(), stream)
        return out

    def __call__(self, x: torch.Tensor, stream=None) -> Dict[str, torch.Tensor]:
        c = self.cfg
        if x.shape[-1] != c.d:
            raise ValueError(f"last dim {x.shape[-1]} != d={c.d}")
        lead = x.shape[:-1]
        x2 = x.reshape(-1, c.d).to(device=self.device, dtype=self.dtype).contiguous()
        out = self.forward_into(x2, self.empty_outputs(x2.shape[0]), stream)
        return {"output": out["output"].reshape(*lead, c.d),
                "selected_experts": out["selected_experts"].reshape(*lead, c.k),
                "mixture_weights": out["mixture_weights"].reshape(*lead, c.k),
                "latent_routed_aggregate": out["latent_routed_aggregate"].reshape(*lead, c.l)}

    def forward_host(self, x_host: torch.Tensor, out_host: Dict[str, torch.Tensor], stream=None):
        """Host buffers in and out (pinned for async copies); copies are inside the library call."""
        T = x_host.shape[0]
        ws = self.workspace(T, host=True)
        lmoe_forward_host(self.handle, x_host, T, out_host["output"], out_host["selected_experts"],
                          out_host["mixture_weights"], out_host["latent_routed_aggregate"], ws, ws.numel(), stream)
        return out_host

    def region(self, T: int, name: str, dtype: torch.dtype, shape) -> torch.Tensor:
        """View of one intermediate in the workspace of the last forward of T tokens."""
        off, n = lmoe_workspace_region(self.handle, T, name)
        ws = self.workspace(T)
        return ws[off:off + n].view(dtype).reshape(shape)

    def check_device(self, T: int, stream=None):
        lmoe_check_device(self.handle, T, self.workspace(T), stream)

    def check_device_host(self, T: int, stream=None):
        """lmoe_check_device after forward_host of T tokens."""
        lmoe_check_device_host(self.handle, T, self.workspace(T, host=True), stream)

    def launch_count(self, T: int) -> int:
        return lmoe_launch_count(self.handle, T)

    def set_bias(self, b: torch.Tensor, stream=None):
        """Replace the selection bias with b [E] (device fp32)."""
        lmoe_set_bias(self.handle, b, stream)

    def qb_histogram(self, T: int, hist: torch.Tensor, bins: int, lo: float, hi: float, stream=None):
        """Add the last forward's (T tokens) Quantile-Balancing margin histogram to hist [E, bins] int32."""
        lmoe_qb_histogram(self.handle, self.workspace(T), T, bins, lo, hi, hist, stream)
        return hist

    def qb_bias_update(self, hist: torch.Tensor, bins: int, lo: float, hi: float, target: int, stream=None):
        """The next step's bias [E] fp32 from an accumulated histogram (apply with set_bias)."""
        out = torch.empty(self.cfg.E, dtype=torch.float32, device=self.device)
        lmoe_qb_bias_update(self.handle, hist, bins, lo, hi, target, out, stream)
        return out


def config_for(workload, gemm: int = 0, act: int = LMOE_ACT_SWIGLU) -> lmoe_config:
    """lmoe_config from an lmoe_inputs.Workload."""
    return make_config(workload.d, workload.l, workload.f, workload.E, workload.k, workload.f_s,
                       workload.n_shared, workload.eps, LMOE_F32 if workload.dtype == "f32" else LMOE_BF16, act,
                       4.0, 25.0, gemm, 1 if getattr(workload, "standard", False) else 0)
