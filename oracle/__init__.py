"""fp64 CPU oracle of the routed Mixture-of-Experts FFN layer -- TEST INFRASTRUCTURE ONLY.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, written from the pages' statement of
the layer; see that file's header for the passages it follows and the readings it takes where
the pages are silent).  This module compiles it with gcc and marshals numpy arrays into it.

Only ``tests/``, the package entry's ``smoke()`` check and the benchmark's CPU-baseline leg may
import this module.  The CUDA library does not import it and shares no code with it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FP8_SC512 = 1
INT4_G128 = 2
MXFP4_G32 = 3
NVFP4_G16 = 4
_WFMT = {"fp8": FP8_SC512, "int4": INT4_G128, "mxfp4": MXFP4_G32, "nvfp4": NVFP4_G16}


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("T", "H", "E", "I", "k", "Is", "wfmt")]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down",
        "ws_gate", "ws_up", "ws_down", "ss_gate", "ss_up", "ss_down",
        "t_gate", "t_up", "t_down", "ts_gate", "ts_up", "ts_down")]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so next to it (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
               "-Wall", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load(_LIB)
    return _lib


def load(path: str):
    """Open a compiled copy of moe_oracle.c and declare its entry points."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_e4m3_encode_n.argtypes = [I, P, P]
    L.orc_e2m1_decode.restype = ctypes.c_double
    L.orc_e2m1_decode.argtypes = [I]
    L.orc_e8m0_decode.restype = ctypes.c_double
    L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
    L.orc_double_to_bf16.restype = ctypes.c_uint16
    L.orc_double_to_bf16.argtypes = [ctypes.c_double]
    L.orc_route.argtypes = [I, I, I, P, P, P]
    L.orc_router_logits.argtypes = [I, I, I, P, P, P, P]
    L.orc_permute.argtypes = [I, I, I, P, P, P, P, P]
    L.orc_quant_row_fp8.argtypes = [I, P, P, P]
    L.orc_quant_rows_bf16.argtypes = [I, I, P, P, P]
    L.orc_expert_fp8_row.argtypes = [I, I] + [P] * 10
    L.orc_expert_int4_row.argtypes = [I, I] + [P] * 9
    L.orc_expert_w4_row.argtypes = [I, I, I] + [P] * 10
    L.orc_layer.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(Weights), P, P, I, P, P, P, P, I]
    return L


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(x) -> np.ndarray:
    x = _c(np.atleast_1d(x), np.float32)
    q = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_n(x.size, _p(x), _p(q))
    return q


def e2m1_decode(nib: int) -> float:
    return lib().orc_e2m1_decode(int(nib))


def e8m0_decode(code: int) -> float:
    return lib().orc_e8m0_decode(int(code))


def double_to_bf16(x: float) -> int:
    return int(lib().orc_double_to_bf16(float(x)))


# --------------------------------------------------------------------------------------
# single steps
# --------------------------------------------------------------------------------------

def route(logits: np.ndarray, k: int):
    """A1 -> (topk_idx int32 [T,k], topk_w float64 [T,k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    rc = lib().orc_route(T, E, k, _p(logits), _p(idx), _p(w))
    if rc != 0:
        raise ValueError("oracle route: bad arguments")
    return idx, w


def router_logits(x_bits: np.ndarray, w_bits: np.ndarray):
    """Router logits in fp64 from bf16 x [T,H] and W [E,H] (bit patterns) ->
    (logits float64 [T,E], bound float64 [T,E] = sum |x_i w_i|)."""
    x_bits, w_bits = _c(x_bits, np.uint16), _c(w_bits, np.uint16)
    T, H = x_bits.shape
    E = w_bits.shape[0]
    lg = np.empty((T, E), np.float64)
    bd = np.empty((T, E), np.float64)
    rc = lib().orc_router_logits(T, H, E, _p(x_bits), _p(w_bits), _p(lg), _p(bd))
    if rc != 0:
        raise ValueError("oracle router: bad arguments")
    return lg, bd


def permute(topk_idx: np.ndarray, E: int):
    """A3 -> (counts [E], offsets [E+1], perm_tok [T*k], pos [T,k]) all int32."""
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    pos = np.empty((T, k), np.int32)
    rc = lib().orc_permute(T, E, k, _p(topk_idx), _p(counts), _p(offsets), _p(perm), _p(pos))
    if rc != 0:
        raise ValueError("oracle permute: expert index out of range")
    return counts, offsets, perm, pos


def quant_rows_f32(x: np.ndarray):
    """A2 on fp32 rows -> (codes uint8 [R,K], scales float32 [R,nb])."""
    x = _c(x, np.float32)
    R, K = x.shape
    nb = (K + 511) // 512
    q = np.empty((R, K), np.uint8)
    s = np.empty((R, nb), np.float32)
    L = lib()
    for r in range(R):
        L.orc_quant_row_fp8(K, _p(x[r]), _p(q[r]), _p(s[r]))
    return q, s


def quant_rows_bf16(x_bits: np.ndarray):
    """A2 on bf16 rows (uint16 bit patterns) -> (codes uint8 [R,K], scales float32 [R,nb])."""
    x_bits = _c(x_bits, np.uint16)
    R, K = x_bits.shape
    nb = (K + 511) // 512
    q = np.empty((R, K), np.uint8)
    s = np.empty((R, nb), np.float32)
    lib().orc_quant_rows_bf16(R, K, _p(x_bits), _p(q), _p(s))
    return q, s


def expert_fp8_row(qx, sx, wg, sg, wu, su, wd, sd):
    """One FP8 expert on one quantised row -> (y float64 [H], h float32 [I])."""
    qx, sx = _c(qx, np.uint8), _c(sx, np.float32)
    wg, wu, wd = _c(wg, np.uint8), _c(wu, np.uint8), _c(wd, np.uint8)
    sg, su, sd = _c(sg, np.float32), _c(su, np.float32), _c(sd, np.float32)
    I, H = wg.shape
    y = np.empty(H, np.float64)
    h = np.empty(I, np.float32)
    lib().orc_expert_fp8_row(H, I, _p(qx), _p(sx), _p(wg), _p(sg), _p(wu), _p(su), _p(wd), _p(sd),
                             _p(y), _p(h))
    return y, h


def expert_int4_row(x_bits, wg, sg, wu, su, wd, sd):
    """One int4 expert on one bf16 row -> (y float64 [H], h float64 [I], bf16-rounded)."""
    x_bits = _c(x_bits, np.uint16)
    wg, wu, wd = _c(wg, np.uint8), _c(wu, np.uint8), _c(wd, np.uint8)
    sg, su, sd = _c(sg, np.uint16), _c(su, np.uint16), _c(sd, np.uint16)
    I = wg.shape[0]
    H = x_bits.shape[0]
    y = np.empty(H, np.float64)
    h = np.empty(I, np.float64)
    lib().orc_expert_int4_row(H, I, _p(x_bits), _p(wg), _p(sg), _p(wu), _p(su), _p(wd), _p(sd),
                              _p(y), _p(h))
    return y, h


def expert_mxfp4_row(x_bits, wg, sg, wu, su, wd, sd):
    """One MXFP4 expert on one bf16 row -> (y float64 [H], h float64 [I], bf16-rounded)."""
    x_bits = _c(x_bits, np.uint16)
    wg, wu, wd = _c(wg, np.uint8), _c(wu, np.uint8), _c(wd, np.uint8)
    sg, su, sd = _c(sg, np.uint8), _c(su, np.uint8), _c(sd, np.uint8)
    I = wg.shape[0]
    H = x_bits.shape[0]
    y = np.empty(H, np.float64)
    h = np.empty(I, np.float64)
    ones = np.ones(3)
    lib().orc_expert_w4_row(MXFP4_G32, H, I, _p(x_bits), _p(wg), _p(sg), _p(wu), _p(su), _p(wd),
                            _p(sd), _p(ones), _p(y), _p(h))
    return y, h


# --------------------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------------------

def layer(layer_np: dict, tokens=None, nthreads: int | None = None, ambiguity: bool = False):
    """Layer output for ``tokens`` (default: all) -> (out float64 [n,H], out_bf16 uint16 [n,H]),
    plus, with ``ambiguity=True``, the envelope float64 [n,H] of the equally valid outputs
    that an h code sitting on a rounding midpoint allows (see moe_oracle.c, reading R10a).

    ``layer_np`` holds numpy arrays with the keys of ``moe_synth`` (x as bf16 bit patterns).
    """
    d = layer_np["dims"]
    wfmt = _WFMT[d["wfmt"]]
    dims = Dims(d["T"], d["H"], d["E"], d["I"], d["k"], d["Is"], wfmt)
    keep = {}

    def arr(name, dtype):
        a = layer_np.get(name)
        if a is None:
            return None
        a = _c(a, dtype)
        keep[name] = a
        return _p(a)

    sdt = {FP8_SC512: np.float32, INT4_G128: np.uint16, MXFP4_G32: np.uint8, NVFP4_G16: np.uint8}[wfmt]
    W = Weights(arr("w_gate", np.uint8), arr("w_up", np.uint8), arr("w_down", np.uint8),
                arr("s_gate", sdt), arr("s_up", sdt), arr("s_down", sdt),
                arr("ws_gate", np.uint8), arr("ws_up", np.uint8), arr("ws_down", np.uint8),
                arr("ss_gate", sdt), arr("ss_up", sdt), arr("ss_down", sdt),
                arr("t_gate", np.float32), arr("t_up", np.float32), arr("t_down", np.float32),
                arr("ts_gate", np.float32), arr("ts_up", np.float32), arr("ts_down", np.float32))
    x = _c(layer_np["x"], np.uint16)
    logits = _c(layer_np["logits"], np.float32)
    if tokens is None:
        tokens = np.arange(d["T"], dtype=np.int32)
    tokens = _c(tokens, np.int32)
    n = tokens.size
    out = np.empty((n, d["H"]), np.float64)
    outb = np.empty((n, d["H"]), np.uint16)
    amb = np.empty((n, d["H"]), np.float64) if ambiguity else None
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = lib().orc_layer(ctypes.byref(dims), ctypes.byref(W), _p(x), _p(logits), n, _p(tokens),
                         _p(out), _p(outb), _p(amb), int(nthreads))
    if rc != 0:
        raise ValueError("oracle layer: bad dims or token index")
    if ambiguity:
        return out, outb, amb
    return out, outb
