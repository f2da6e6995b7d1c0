"""Python side of the fp64 CPU oracle (test infrastructure only).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark use
this module. It builds ``tfmoe_oracle.c`` with gcc into ``libtfmoe_oracle.so``
beside it (on first use, or through :func:`build`) and calls it via ctypes.
It imports nothing from the CUDA package.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tfmoe_oracle.c")
LIB = os.path.join(HERE, "libtfmoe_oracle.so")

_u16p = ctypes.POINTER(ctypes.c_uint16)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)


class _Layer(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("intermediate", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("router_w", _u16p), ("router_bias", _f32p),
                ("gate_codes", _u8p), ("up_codes", _u8p),
                ("gate_scales", _u8p), ("up_scales", _u8p),
                ("gate_global", _f32p), ("up_global", _f32p),
                ("down_codes", _u8p), ("down_scales", _u8p), ("down_global", _f32p),
                ("shared_intermediate", ctypes.c_int32),
                ("sh_gate_codes", _u8p), ("sh_up_codes", _u8p),
                ("sh_gate_scales", _u8p), ("sh_up_scales", _u8p),
                ("sh_gate_global", ctypes.c_float), ("sh_up_global", ctypes.c_float),
                ("sh_down_codes", _u8p), ("sh_down_scales", _u8p), ("sh_down_global", ctypes.c_float)]


class _Epilogue(ctypes.Structure):
    _fields_ = [("residual", _u16p), ("norm_w", _u16p), ("eps", ctypes.c_double), ("act_fp4", ctypes.c_int32)]


class _Outputs(ctypes.Structure):
    _fields_ = [("out", _u16p), ("out64", _f64p), ("S", _f64p), ("logits", _f32p),
                ("ids", _i32p), ("g", _f64p), ("G", _f32p), ("U", _f32p),
                ("a", _u16p), ("y", _f64p), ("yabs", _f64p),
                ("out_norm", _u16p), ("a_sh", _u16p), ("y_sh", _f64p)]

# Keys of the optional shared expert in a layer dict (canonical layout, see forward()).
SHARED_KEYS = ("shared_gate_codes", "shared_up_codes", "shared_gate_scales", "shared_up_scales",
               "shared_gate_global", "shared_up_global", "shared_down_codes", "shared_down_scales",
               "shared_down_global")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE semantics: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-std=c11", SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_e2m1.restype = ctypes.c_double
        _lib.oracle_e2m1.argtypes = [ctypes.c_uint]
        _lib.oracle_e4m3.restype = ctypes.c_double
        _lib.oracle_e4m3.argtypes = [ctypes.c_uint]
        _lib.oracle_round_bf16.restype = ctypes.c_uint16
        _lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        _lib.oracle_bf16_to_double.restype = ctypes.c_double
        _lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        _lib.oracle_forward.restype = ctypes.c_int
        _lib.oracle_forward.argtypes = [ctypes.POINTER(_Layer), _u16p, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.POINTER(_Epilogue), ctypes.POINTER(_Outputs)]
        _lib.oracle_rms_norm.restype = ctypes.c_int
        _lib.oracle_e2m1_rne.restype = ctypes.c_uint
        _lib.oracle_e2m1_rne.argtypes = [ctypes.c_double]
        _lib.oracle_e4m3_rne.restype = ctypes.c_uint
        _lib.oracle_e4m3_rne.argtypes = [ctypes.c_double]
        _lib.oracle_quant_act_row.restype = ctypes.c_int
        _lib.oracle_quant_act_row.argtypes = [_f64p, ctypes.c_int32, _u8p, _u8p, _f32p, _f64p]
        _lib.oracle_rms_norm.argtypes = [_u16p, _u16p, ctypes.c_int32, ctypes.c_int32, ctypes.c_double, _u16p]
        _lib.oracle_route.restype = ctypes.c_int
        _lib.oracle_route.argtypes = [ctypes.POINTER(_Layer), _u16p, ctypes.c_int32, ctypes.c_int32,
                                      _f32p, _i32p, _f64p]
        _lib.oracle_max_threads.restype = ctypes.c_int
    return _lib


def e2m1(code: int) -> float:
    return lib().oracle_e2m1(code)


def e4m3(byte: int) -> float:
    return lib().oracle_e4m3(byte)


def round_bf16(v: float) -> int:
    return int(lib().oracle_round_bf16(v))


def bf16_to_float(bits: int) -> float:
    return lib().oracle_bf16_to_double(bits)


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _ptr(a: Optional[np.ndarray], t):
    if a is None:
        return ctypes.cast(None, t)
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


def e2m1_rne(v: float) -> int:
    return int(lib().oracle_e2m1_rne(v))


def e4m3_rne(v: float) -> int:
    return int(lib().oracle_e4m3_rne(v))


def quant_act_row(v: np.ndarray):
    """The oracle's NVFP4 quantisation of one activation row (values exactly representable in
    fp32, length a multiple of 16): (codes uint8 [K], scales uint8 [K/16], g fp32, deq fp64 [K])."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    K = v.shape[0]
    codes, scales = np.zeros(K, np.uint8), np.zeros(K // 16, np.uint8)
    g = ctypes.c_float()
    deq = np.zeros(K, np.float64)
    rc = lib().oracle_quant_act_row(_ptr(v, _f64p), K, _ptr(codes, _u8p), _ptr(scales, _u8p), ctypes.byref(g),
                                    _ptr(deq, _f64p))
    if rc != 0:
        raise RuntimeError(f"oracle_quant_act_row failed with code {rc}")
    return codes, scales, float(g.value), deq


def rms_norm(v: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """The oracle's RMS norm of bf16 rows v [T][H] with bf16 gamma [H] (bf16 bits out)."""
    v = np.ascontiguousarray(v, dtype=np.uint16)
    gamma = np.ascontiguousarray(gamma, dtype=np.uint16)
    T, H = v.shape
    out = np.zeros((T, H), np.uint16)
    rc = lib().oracle_rms_norm(_ptr(v, _u16p), _ptr(gamma, _u16p), T, H, eps, _ptr(out, _u16p))
    if rc != 0:
        raise RuntimeError(f"oracle_rms_norm failed with code {rc}")
    return out


def forward(layer: Dict[str, Optional[np.ndarray]], x: np.ndarray, *, top_k: int,
            nthreads: int = 0, intermediates: bool = False, residual: Optional[np.ndarray] = None,
            norm_w: Optional[np.ndarray] = None, eps: float = 1e-6, act_fp4: bool = False) -> Dict[str, np.ndarray]:
    """Run the oracle on host arrays in the canonical layout.

    ``x`` is bf16 bits [T][H]. Returns out (bf16 bits), out64, S, and with
    ``intermediates`` also logits, ids, g, G, U, a and y.
    A layer dict holding the SHARED_KEYS (codes/scales [Is][H/2], [Is][H/16], down
    [H][Is/2], [H][Is/16], globals as one-element fp32 arrays) adds the shared expert
    (``a_sh``, ``y_sh`` with ``intermediates``). ``residual`` (bf16 bits [T][H]) is added
    to the output; ``norm_w`` (bf16 bits [H]) adds ``out_norm``, the RMS norm of ``out``.
    ``act_fp4`` selects the W4A4 variant: the routed experts read NVFP4-quantised x (gate/up)
    and a (down) rows (see quant_act_row).
    """
    E, H = layer["router_w"].shape
    I = layer["gate_codes"].shape[1]
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T = x.shape[0]
    assert x.shape == (T, H)
    keep = []

    def arr(name, dtype):
        a = np.ascontiguousarray(layer[name], dtype=dtype)
        keep.append(a)
        return a

    L = _Layer(H, I, E, top_k,
               _ptr(arr("router_w", np.uint16), _u16p),
               _ptr(None if layer.get("router_bias") is None else arr("router_bias", np.float32), _f32p),
               _ptr(arr("gate_codes", np.uint8), _u8p), _ptr(arr("up_codes", np.uint8), _u8p),
               _ptr(arr("gate_scales", np.uint8), _u8p), _ptr(arr("up_scales", np.uint8), _u8p),
               _ptr(arr("gate_global", np.float32), _f32p), _ptr(arr("up_global", np.float32), _f32p),
               _ptr(arr("down_codes", np.uint8), _u8p), _ptr(arr("down_scales", np.uint8), _u8p),
               _ptr(arr("down_global", np.float32), _f32p))
    Is = 0
    if layer.get("shared_gate_codes") is not None:
        Is = layer["shared_gate_codes"].shape[0]
        assert layer["shared_down_codes"].shape == (H, Is // 2)
        L.shared_intermediate = Is
        L.sh_gate_codes = _ptr(arr("shared_gate_codes", np.uint8), _u8p)
        L.sh_up_codes = _ptr(arr("shared_up_codes", np.uint8), _u8p)
        L.sh_gate_scales = _ptr(arr("shared_gate_scales", np.uint8), _u8p)
        L.sh_up_scales = _ptr(arr("shared_up_scales", np.uint8), _u8p)
        L.sh_gate_global = float(np.float32(layer["shared_gate_global"].reshape(-1)[0]))
        L.sh_up_global = float(np.float32(layer["shared_up_global"].reshape(-1)[0]))
        L.sh_down_codes = _ptr(arr("shared_down_codes", np.uint8), _u8p)
        L.sh_down_scales = _ptr(arr("shared_down_scales", np.uint8), _u8p)
        L.sh_down_global = float(np.float32(layer["shared_down_global"].reshape(-1)[0]))
    epi = _Epilogue(_ptr(None, _u16p), _ptr(None, _u16p), float(eps), 1 if act_fp4 else 0)
    if residual is not None:
        residual = np.ascontiguousarray(residual, dtype=np.uint16)
        assert residual.shape == (T, H)
        epi.residual = _ptr(residual, _u16p)
    if norm_w is not None:
        norm_w = np.ascontiguousarray(norm_w, dtype=np.uint16)
        assert norm_w.shape == (H,)
        epi.norm_w = _ptr(norm_w, _u16p)
    P = T * top_k
    res = {"out": np.zeros((T, H), np.uint16), "out64": np.zeros((T, H), np.float64),
           "S": np.zeros((T, H), np.float64)}
    if norm_w is not None:
        res["out_norm"] = np.zeros((T, H), np.uint16)
    if intermediates and Is:
        res.update(a_sh=np.zeros((T, Is), np.uint16), y_sh=np.zeros((T, H), np.float64))
    if intermediates:
        res.update(logits=np.zeros((T, E), np.float32), ids=np.zeros((T, top_k), np.int32),
                   g=np.zeros((T, top_k), np.float64), G=np.zeros((T, top_k, I), np.float32),
                   U=np.zeros((T, top_k, I), np.float32), a=np.zeros((T, top_k, I), np.uint16),
                   y=np.zeros((T, top_k, H), np.float64), yabs=np.zeros((T, top_k, H), np.float64))
    O = _Outputs(_ptr(res["out"], _u16p), _ptr(res["out64"], _f64p), _ptr(res["S"], _f64p),
                 _ptr(res.get("logits"), _f32p), _ptr(res.get("ids"), _i32p),
                 _ptr(res.get("g"), _f64p), _ptr(res.get("G"), _f32p), _ptr(res.get("U"), _f32p),
                 _ptr(res.get("a"), _u16p), _ptr(res.get("y"), _f64p), _ptr(res.get("yabs"), _f64p),
                 _ptr(res.get("out_norm"), _u16p), _ptr(res.get("a_sh"), _u16p), _ptr(res.get("y_sh"), _f64p))
    rc = lib().oracle_forward(ctypes.byref(L), _ptr(x, _u16p), T, nthreads, ctypes.byref(epi), ctypes.byref(O))
    if rc != 0:
        raise RuntimeError(f"oracle_forward failed with code {rc}")
    del keep, P, residual, norm_w
    return res


def route(layer: Dict[str, Optional[np.ndarray]], x: np.ndarray, *, top_k: int,
          nthreads: int = 0) -> Dict[str, np.ndarray]:
    """Routing alone (logits, ids, g) of every token of ``x`` (bf16 bits [T][H]): the
    oracle's routing step, without the expert projections."""
    E, H = layer["router_w"].shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T = x.shape[0]
    assert x.shape == (T, H)
    rw = np.ascontiguousarray(layer["router_w"], dtype=np.uint16)
    bias = None if layer.get("router_bias") is None else np.ascontiguousarray(layer["router_bias"], np.float32)
    null8 = ctypes.cast(None, _u8p)
    nullf = ctypes.cast(None, _f32p)
    L = _Layer(H, 16, E, top_k, _ptr(rw, _u16p), _ptr(bias, _f32p), null8, null8, null8, null8, nullf, nullf,
               null8, null8, nullf)
    res = {"logits": np.zeros((T, E), np.float32), "ids": np.zeros((T, top_k), np.int32),
           "g": np.zeros((T, top_k), np.float64)}
    rc = lib().oracle_route(ctypes.byref(L), _ptr(x, _u16p), T, nthreads, _ptr(res["logits"], _f32p),
                            _ptr(res["ids"], _i32p), _ptr(res["g"], _f64p))
    if rc != 0:
        raise RuntimeError(f"oracle_route failed with code {rc}")
    return res


def tolerance(S: np.ndarray) -> np.ndarray:
    """Per-element bound |gpu - oracle| <= 4e-3 * S + 1e-3, S = sum |a*w| (g-weighted)."""
    return 4e-3 * S + 1e-3
