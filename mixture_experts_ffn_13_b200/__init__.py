"""Routed Mixture-of-Experts FFN layer for NVIDIA B200 (sm_100a): Python binding.

Argument marshalling only: every step of the layer runs in the CUDA library
``libmoe_b200.so`` (built in-tree by ``build.py``) behind the C ABI declared in
``include/moe_b200.h``.  The functions here carry the C names (``moe_plan``, ``moe_route``,
``moe_forward``, ``moe_get_status``, ``moe_destroy``, ``moe_strerror``) and take torch tensors
for device buffers.  There is no fallback: if the library is missing or a CUDA device is not
available the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_W_FP8_SC512 = 1
MOE_W_INT4_G128 = 2
MOE_W_MXFP4_G32 = 3
MOE_W_NVFP4_G16 = 4
_WFMT = {"fp8": MOE_W_FP8_SC512, "int4": MOE_W_INT4_G128, "mxfp4": MOE_W_MXFP4_G32, "nvfp4": MOE_W_NVFP4_G16}
MOE_OK = 0
ERRORS = {-1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_WORKSPACE",
          -4: "MOE_ERR_CUDA", -5: "MOE_ERR_DEVICE_TIMEOUT", -6: "MOE_ERR_BOUNDS"}
EXPORTS = ("moe_plan", "moe_route", "moe_forward", "moe_get_status", "moe_last_cuda_error",
           "moe_destroy", "moe_strerror", "moe_profile_enable", "moe_profile_read",
           "moe_profile_stage_name", "moe_launch_count", "moe_route_static", "moe_router_logits",
           "moe_router_topk", "moe_forward_x", "moe_set_checked")
STAGES = ("route", "permute", "quant_x", "gemm_gateup", "quant_h", "gemm_down", "combine")


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str, cuda_error: int = 0):
        msg = f"{what}: {ERRORS.get(code, code)}"
        if cuda_error:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)
        self.code = code


class moe_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T_max", "H", "E", "I", "k", "I_shared", "wfmt")]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down",
        "ws_gate", "ws_up", "ws_down", "ss_gate", "ss_up", "ss_down",
        "t_gate", "t_up", "t_down", "ts_gate", "ts_up", "ts_down")]


_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (no compute happens here; works without a GPU)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"CUDA library not built: {path} is missing "
                                   "(run mixture_experts_ffn_13_b200/build.py)")
            L = ctypes.CDLL(path)
            P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            L.moe_plan.argtypes = [ctypes.POINTER(moe_dims), ctypes.POINTER(P), ctypes.POINTER(SZ)]
            L.moe_plan.restype = ctypes.c_int
            L.moe_route.argtypes = [P, I32, P, P, P, P, P, P, P, SZ, P]
            L.moe_route.restype = ctypes.c_int
            L.moe_forward.argtypes = [P, I32, P, P, ctypes.POINTER(moe_weights), P, P, SZ, P]
            L.moe_forward.restype = ctypes.c_int
            L.moe_get_status.argtypes = [P, P]
            L.moe_get_status.restype = ctypes.c_int
            L.moe_last_cuda_error.argtypes = [P]
            L.moe_last_cuda_error.restype = ctypes.c_int
            L.moe_destroy.argtypes = [P]
            L.moe_destroy.restype = None
            L.moe_strerror.argtypes = [ctypes.c_int]
            L.moe_strerror.restype = ctypes.c_char_p
            L.moe_profile_enable.argtypes = [P, ctypes.c_int]
            L.moe_profile_enable.restype = ctypes.c_int
            L.moe_profile_read.argtypes = [P, ctypes.POINTER(ctypes.c_float), ctypes.c_int]
            L.moe_profile_read.restype = ctypes.c_int
            L.moe_profile_stage_name.argtypes = [ctypes.c_int]
            L.moe_profile_stage_name.restype = ctypes.c_char_p
            L.moe_launch_count.argtypes = [P]
            L.moe_launch_count.restype = ctypes.c_int
            L.moe_router_logits.argtypes = [P, I32, P, P, P, P]
            L.moe_router_logits.restype = ctypes.c_int
            L.moe_router_topk.argtypes = [P, I32, P, P, P, P, P, P]
            L.moe_router_topk.restype = ctypes.c_int
            L.moe_forward_x.argtypes = [P, I32, P, P, ctypes.POINTER(moe_weights), P, P, SZ, P]
            L.moe_forward_x.restype = ctypes.c_int
            L.moe_set_checked.argtypes = [P, ctypes.c_int]
            L.moe_set_checked.restype = ctypes.c_int
            L.moe_route_static.argtypes = [I32, I32, I32, P, P, P, P, P, P, P]
            L.moe_route_static.restype = ctypes.c_int
            _lib = L
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda:
        raise ValueError("device buffers must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("buffers must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(rc: int, what: str, plan=None):
    if rc != MOE_OK:
        ce = load_library().moe_last_cuda_error(plan) if plan is not None else 0
        raise MoEError(rc, what, ce)


def moe_strerror(code: int) -> str:
    return load_library().moe_strerror(int(code)).decode()


class Plan:
    """A plan (host object owning one device status word) plus its workspace size."""

    def __init__(self, T_max, H, E, I, k, I_shared=0, wfmt="fp8"):
        L = load_library()
        if wfmt not in _WFMT and wfmt not in _WFMT.values():
            raise ValueError(f"unknown weight format {wfmt!r}")
        fmt = _WFMT.get(wfmt, wfmt)
        self.dims = moe_dims(T_max, H, E, I, k, I_shared, fmt)
        self.wfmt = next(n for n, v in _WFMT.items() if v == fmt)
        h = ctypes.c_void_p()
        ws = ctypes.c_size_t()
        _check(L.moe_plan(ctypes.byref(self.dims), ctypes.byref(h), ctypes.byref(ws)), "moe_plan")
        self.handle = h.value
        self.workspace_bytes = ws.value

    def new_workspace(self, device=None) -> torch.Tensor:
        return torch.empty(max(self.workspace_bytes, 1), dtype=torch.uint8, device=device or "cuda")

    def close(self):
        if getattr(self, "handle", None):
            load_library().moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_plan(T_max, H, E, I, k, I_shared=0, wfmt="fp8") -> Plan:
    return Plan(T_max, H, E, I, k, I_shared, wfmt)


def moe_destroy(plan: Plan):
    plan.close()


def moe_get_status(plan: Plan, stream=None) -> int:
    return load_library().moe_get_status(plan.handle, _stream(stream))


def moe_profile_enable(plan: Plan, enable: bool = True):
    _check(load_library().moe_profile_enable(plan.handle, int(bool(enable))), "moe_profile_enable", plan.handle)


def moe_profile_read(plan: Plan) -> dict:
    """Stage name -> device milliseconds of the last moe_forward (waits for its events)."""
    buf = (ctypes.c_float * len(STAGES))()
    n = load_library().moe_profile_read(plan.handle, buf, len(STAGES))
    if n < 0:
        _check(n, "moe_profile_read", plan.handle)
    return {STAGES[i]: float(buf[i]) for i in range(n)}


def moe_set_checked(plan: Plan, enable: bool = True):
    """Checked mode: device-side checks of the router logits (finite) and permuted row indices;
    a failure shows as MOE_ERR_BOUNDS from moe_get_status."""
    _check(load_library().moe_set_checked(plan.handle, 1 if enable else 0), "moe_set_checked")


def moe_launch_count(plan: Plan) -> int:
    return load_library().moe_launch_count(plan.handle)


def _weights_struct(w: dict) -> moe_weights:
    g = lambda n: _ptr(w.get(n))
    return moe_weights(g("w_gate"), g("w_up"), g("w_down"), g("s_gate"), g("s_up"), g("s_down"),
                       g("ws_gate"), g("ws_up"), g("ws_down"), g("ss_gate"), g("ss_up"), g("ss_down"),
                       g("t_gate"), g("t_up"), g("t_down"), g("ts_gate"), g("ts_up"), g("ts_down"))


def moe_route(plan: Plan, logits: torch.Tensor, workspace: torch.Tensor, out: dict | None = None,
              stream=None) -> dict:
    """Steps A1 + A3 -> dict(topk_idx, topk_w, counts, offsets, perm_tok) device tensors."""
    d = plan.dims
    T = logits.shape[0]
    if logits.dtype != torch.float32 or logits.dim() != 2 or logits.shape[1] != d.E:
        raise ValueError("logits must be fp32 [T, E]")
    dev = logits.device
    if out is None:
        out = dict(topk_idx=torch.empty((T, d.k), dtype=torch.int32, device=dev),
                   topk_w=torch.empty((T, d.k), dtype=torch.float32, device=dev),
                   counts=torch.empty((d.E,), dtype=torch.int32, device=dev),
                   offsets=torch.empty((d.E + 1,), dtype=torch.int32, device=dev),
                   perm_tok=torch.empty((max(T * d.k, 1),), dtype=torch.int32, device=dev))
    rc = load_library().moe_route(plan.handle, T, _ptr(logits), _ptr(out["topk_idx"]), _ptr(out["topk_w"]),
                                  _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["perm_tok"]),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "moe_route", plan.handle)
    return out


def moe_router_logits(plan: Plan, x: torch.Tensor, w_router: torch.Tensor, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """Router logits [T, E] fp32 = x [T, H] bf16 . w_router [E, H]^T bf16, on the tensor cores."""
    d = plan.dims
    T = x.shape[0]
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != d.H:
        raise ValueError("x must be bf16 [T, H]")
    if w_router.dtype != torch.bfloat16 or tuple(w_router.shape) != (d.E, d.H):
        raise ValueError("w_router must be bf16 [E, H]")
    if out is None:
        out = torch.empty((T, d.E), dtype=torch.float32, device=x.device)
    rc = load_library().moe_router_logits(plan.handle, T, _ptr(x), _ptr(w_router), _ptr(out), _stream(stream))
    _check(rc, "moe_router_logits", plan.handle)
    return out


def moe_router_topk(plan: Plan, x: torch.Tensor, w_router: torch.Tensor, out: dict | None = None,
                    stream=None) -> dict:
    """Router logits and their softmax top-k from hidden states: dict(logits [T, E] fp32,
    topk_idx [T, k] int32, topk_w [T, k] fp32)."""
    d = plan.dims
    T = x.shape[0]
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != d.H:
        raise ValueError("x must be bf16 [T, H]")
    if w_router.dtype != torch.bfloat16 or tuple(w_router.shape) != (d.E, d.H):
        raise ValueError("w_router must be bf16 [E, H]")
    dev = x.device
    if out is None:
        out = dict(logits=torch.empty((T, d.E), dtype=torch.float32, device=dev),
                   topk_idx=torch.empty((T, d.k), dtype=torch.int32, device=dev),
                   topk_w=torch.empty((T, d.k), dtype=torch.float32, device=dev))
    rc = load_library().moe_router_topk(plan.handle, T, _ptr(x), _ptr(w_router), _ptr(out["logits"]),
                                        _ptr(out["topk_idx"]), _ptr(out["topk_w"]), _stream(stream))
    _check(rc, "moe_router_topk", plan.handle)
    return out


def moe_route_static(logits: torch.Tensor, k: int, out: dict | None = None, stream=None) -> dict:
    """moe_route without a plan or workspace (fixed static scratch inside the library; for
    callers that cannot allocate device memory -- see include/moe_b200.h for its limits)."""
    if logits.dtype != torch.float32 or logits.dim() != 2:
        raise ValueError("logits must be fp32 [T, E]")
    T, E = logits.shape
    dev = logits.device
    if out is None:
        out = dict(topk_idx=torch.empty((T, k), dtype=torch.int32, device=dev),
                   topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
                   counts=torch.empty((E,), dtype=torch.int32, device=dev),
                   offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
                   perm_tok=torch.empty((max(T * k, 1),), dtype=torch.int32, device=dev))
    if any(t.device != dev for t in out.values()):
        raise ValueError("outputs must live on the logits' device")
    # the library launches on the current device with that device's scratch array: make the
    # logits' device current for the call (its default stream unless one is given)
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        rc = load_library().moe_route_static(T, E, k, _ptr(logits), _ptr(out["topk_idx"]), _ptr(out["topk_w"]),
                                             _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["perm_tok"]),
                                             s.cuda_stream)
    _check(rc, "moe_route_static")
    return out


def moe_forward(plan: Plan, x: torch.Tensor, logits: torch.Tensor, weights: dict, workspace: torch.Tensor,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The whole layer: out[T, H] bf16."""
    d = plan.dims
    T = x.shape[0]
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != d.H:
        raise ValueError("x must be bf16 [T, H]")
    if logits.dtype != torch.float32 or tuple(logits.shape) != (T, d.E):
        raise ValueError("logits must be fp32 [T, E]")
    if out is None:
        out = torch.empty((T, d.H), dtype=torch.bfloat16, device=x.device)
    W = _weights_struct(weights)
    rc = load_library().moe_forward(plan.handle, T, _ptr(x), _ptr(logits), ctypes.byref(W), _ptr(out),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "moe_forward", plan.handle)
    return out


def moe_forward_x(plan: Plan, x: torch.Tensor, w_router: torch.Tensor, weights: dict, workspace: torch.Tensor,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The whole layer from hidden states and router weights: out[T, H] bf16."""
    d = plan.dims
    T = x.shape[0]
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != d.H:
        raise ValueError("x must be bf16 [T, H]")
    if w_router.dtype != torch.bfloat16 or tuple(w_router.shape) != (d.E, d.H):
        raise ValueError("w_router must be bf16 [E, H]")
    if out is None:
        out = torch.empty((T, d.H), dtype=torch.bfloat16, device=x.device)
    W = _weights_struct(weights)
    rc = load_library().moe_forward_x(plan.handle, T, _ptr(x), _ptr(w_router), ctypes.byref(W), _ptr(out),
                                      _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "moe_forward_x", plan.handle)
    return out


class MoELayer:
    """Convenience wrapper: a plan, its workspace and a set of device weights."""

    def __init__(self, layer: dict, T_max: int | None = None):
        d = layer["dims"]
        self.dims = d
        self.plan = Plan(T_max or d["T"], d["H"], d["E"], d["I"], d["k"], d["Is"], d["wfmt"])
        self.weights = {k: v for k, v in layer.items() if isinstance(v, torch.Tensor)
                        and k[:2] in ("w_", "s_", "ws", "ss", "t_", "ts")}
        self.workspace = self.plan.new_workspace(layer["x"].device)

    def route(self, logits, stream=None):
        return moe_route(self.plan, logits, self.workspace, stream=stream)

    def forward(self, x, logits, out=None, stream=None):
        return moe_forward(self.plan, x, logits, self.weights, self.workspace, out=out, stream=stream)

    __call__ = forward
