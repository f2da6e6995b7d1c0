"""ctypes binding of libtfmoe (include/tfmoe.h): argument marshalling only.

Every step of the layer runs in the CUDA library; this module only passes
device pointers, sizes and the current torch stream. There is no fallback:
if libtfmoe.so is missing or cannot be loaded, importing the layer raises.
PyTorch is used for device memory and streams.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("TFMOE_LIB", os.path.join(PKG, "libtfmoe.so"))

OK, ERR_INVALID_ARG, ERR_OOM, ERR_CUDA, ERR_NOT_LOADED, ERR_UNSUPPORTED, ERR_TIMEOUT, ERR_DEVICE = range(8)
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "OOM", 3: "CUDA", 4: "NOT_LOADED", 5: "UNSUPPORTED",
                6: "TIMEOUT", 7: "DEVICE"}

FLAG_FORCE_GEMV = 0x1
FLAG_FORCE_MMA = 0x2
FLAG_DEBUG_CHECKS = 0x4
FLAG_TEST_TIMEOUT = 0x8

BUF_LOGITS, BUF_TOPK_IDS, BUF_TOPK_WEIGHTS, BUF_EXPERT_COUNTS, BUF_EXPERT_OFFSETS, BUF_PERM, BUF_INV, \
    BUF_ACT, BUF_EXPERT_OUT, BUF_REGIME = range(10)

EXPORTED = ["tfmoe_create", "tfmoe_load_weights", "tfmoe_forward", "tfmoe_forward_host", "tfmoe_sync_status",
            "tfmoe_destroy", "tfmoe_last_error", "tfmoe_get_buffer", "tfmoe_last_launch_count",
            "tfmoe_profile_enable", "tfmoe_profile_read", "tfmoe_route_noalloc", "tfmoe_forward_stage",
            "tfmoe_forward_add_norm"]

ROUTE_NOALLOC_MAX_LOGITS = 1 << 20

STAGES = ["router", "topk", "permute", "gemv_gate_up", "gemv_down", "mma_gate_up", "mma_down", "combine", "gather"]
STAGE_ID = {n: i for i, n in enumerate(STAGES)}


class LayerDesc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("intermediate", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("has_router_bias", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("gemv_max_tokens", ctypes.c_int32),
                ("shared_intermediate", ctypes.c_int32), ("norm_eps", ctypes.c_float)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_bias", "gate_codes", "up_codes", "gate_scales", "up_scales",
        "gate_global", "up_global", "down_codes", "down_scales", "down_global",
        "shared_gate_codes", "shared_up_codes", "shared_gate_scales", "shared_up_scales",
        "shared_gate_global", "shared_up_global", "shared_down_codes", "shared_down_scales",
        "shared_down_global")]


class TfmoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libtfmoe.so and declare its signatures. Raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libtfmoe.so not built ({path}); run python -m nvfp4_weight_only_route_b200.build")
    lib = ctypes.CDLL(path)
    vp, i32, u32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32
    lib.tfmoe_create.argtypes = [ctypes.POINTER(LayerDesc), ctypes.POINTER(vp)]
    lib.tfmoe_create.restype = ctypes.c_int
    lib.tfmoe_load_weights.argtypes = [vp, ctypes.POINTER(Weights)]
    lib.tfmoe_load_weights.restype = ctypes.c_int
    lib.tfmoe_forward.argtypes = [vp, vp, i32, vp, vp]
    lib.tfmoe_forward.restype = ctypes.c_int
    lib.tfmoe_forward_add_norm.argtypes = [vp, vp, i32, vp, vp, vp, vp, vp]
    lib.tfmoe_forward_add_norm.restype = ctypes.c_int
    lib.tfmoe_forward_host.argtypes = [vp, vp, i32, vp, vp]
    lib.tfmoe_forward_host.restype = ctypes.c_int
    lib.tfmoe_sync_status.argtypes = [vp, vp]
    lib.tfmoe_sync_status.restype = ctypes.c_int
    lib.tfmoe_destroy.argtypes = [vp]
    lib.tfmoe_destroy.restype = None
    lib.tfmoe_last_error.argtypes = []
    lib.tfmoe_last_error.restype = ctypes.c_char_p
    lib.tfmoe_get_buffer.argtypes = [vp, ctypes.c_int, ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_size_t)]
    lib.tfmoe_get_buffer.restype = ctypes.c_int
    lib.tfmoe_last_launch_count.argtypes = [vp]
    lib.tfmoe_last_launch_count.restype = i32
    lib.tfmoe_profile_enable.argtypes = [vp, i32]
    lib.tfmoe_profile_enable.restype = ctypes.c_int
    lib.tfmoe_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(i32), i32]
    lib.tfmoe_profile_read.restype = ctypes.c_int
    lib.tfmoe_forward_stage.argtypes = [vp, i32, vp, i32, vp, vp]
    lib.tfmoe_forward_stage.restype = ctypes.c_int
    lib.tfmoe_route_noalloc.argtypes = [vp, i32, i32, vp, vp, i32, i32, vp, vp, vp]
    lib.tfmoe_route_noalloc.restype = ctypes.c_int
    del u32
    _lib = lib
    return lib


def last_error() -> str:
    return load_library().tfmoe_last_error().decode()


def check(status: int):
    if status != OK:
        raise TfmoeError(status, last_error())


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class MoELayer:
    """One NVFP4 W4A16 MoE FFN layer held by libtfmoe on the current CUDA device."""

    def __init__(self, hidden: int, intermediate: int, num_experts: int, top_k: int, max_tokens: int,
                 has_router_bias: bool = False, flags: int = 0, gemv_max_tokens: int = 0,
                 shared_intermediate: int = 0, norm_eps: float = 1e-6):
        self.lib = load_library()
        self.desc = LayerDesc(hidden, intermediate, num_experts, top_k, max_tokens,
                              1 if has_router_bias else 0, flags, gemv_max_tokens, shared_intermediate, norm_eps)
        h = ctypes.c_void_p()
        check(self.lib.tfmoe_create(ctypes.byref(self.desc), ctypes.byref(h)))
        self.handle = h

    def load_weights(self, w: Dict[str, "object"]):
        """w: canonical-layout device tensors (see synth.LAYER_KEYS); router_bias may be None."""
        ws = Weights(*[_ptr(w.get(n)) for n, _ in Weights._fields_])
        check(self.lib.tfmoe_load_weights(self.handle, ctypes.byref(ws)))

    def forward(self, x, out=None, T: Optional[int] = None, stream=None):
        """x: bf16 device tensor [T, H] (or raw bits as int16/uint16); returns out [T, H] bf16."""
        import torch
        if T is None:
            T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.desc.hidden), dtype=torch.bfloat16, device=x.device)
        check(self.lib.tfmoe_forward(self.handle, _ptr(x), T, _ptr(out), _stream_handle(stream)))
        return out

    def forward_add_norm(self, x, residual=None, norm_w=None, out=None, out_norm=None, T: Optional[int] = None,
                         stream=None):
        """The layer, + residual (may be out itself), and with norm_w the RMS norm of the result
        (tfmoe_forward_add_norm). Returns (out, out_norm or None)."""
        import torch
        if T is None:
            T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.desc.hidden), dtype=torch.bfloat16, device=x.device)
        if norm_w is not None and out_norm is None:
            out_norm = torch.empty((T, self.desc.hidden), dtype=torch.bfloat16, device=x.device)
        check(self.lib.tfmoe_forward_add_norm(self.handle, _ptr(x), T, _ptr(residual), _ptr(norm_w), _ptr(out),
                                              _ptr(out_norm) if norm_w is not None else None,
                                              _stream_handle(stream)))
        return out, (out_norm if norm_w is not None else None)

    def forward_raw(self, x_ptr: int, T: int, out_ptr: int, stream_handle: int) -> int:
        return self.lib.tfmoe_forward(self.handle, x_ptr, T, out_ptr, stream_handle)

    def forward_stage_raw(self, stage: int, x_ptr: int, T: int, out_ptr: int, stream_handle: int) -> int:
        """Re-enqueue one stage of the last forward (see tfmoe_forward_stage)."""
        return self.lib.tfmoe_forward_stage(self.handle, stage, x_ptr, T, out_ptr, stream_handle)

    def forward_host(self, x_host, out_host, T: Optional[int] = None, stream=None):
        """Host (CPU) tensors in and out; copies happen inside the call, which returns when done."""
        if T is None:
            T = x_host.shape[0]
        check(self.lib.tfmoe_forward_host(self.handle, _ptr(x_host), T, _ptr(out_host), _stream_handle(stream)))
        return out_host

    def sync_status(self, stream=None) -> int:
        return self.lib.tfmoe_sync_status(self.handle, _stream_handle(stream))

    def buffer(self, which: int):
        p, n = ctypes.c_void_p(), ctypes.c_size_t()
        check(self.lib.tfmoe_get_buffer(self.handle, which, ctypes.byref(p), ctypes.byref(n)))
        return p.value, n.value

    def buffer_tensor(self, which: int, dtype, shape):
        """Copy of an internal buffer (the leading elements that `shape` covers) as a torch tensor."""
        import torch
        ptr, nbytes = self.buffer(which)
        view = _DeviceView(ptr, nbytes, dtype)
        flat = torch.as_tensor(view, device="cuda")
        if view.bf16:
            flat = flat.view(torch.bfloat16)
        count = 1
        for s in shape:
            count *= s
        torch.cuda.current_stream().synchronize()
        return flat[:count].reshape(shape).clone()

    def last_launch_count(self) -> int:
        return int(self.lib.tfmoe_last_launch_count(self.handle))

    def profile(self, enable: bool):
        check(self.lib.tfmoe_profile_enable(self.handle, 1 if enable else 0))

    def profile_read(self, reset: bool = True):
        """{stage name: (total ms, calls)} accumulated by profiled forwards."""
        n = len(STAGES)
        ms = (ctypes.c_float * n)()
        calls = (ctypes.c_int32 * n)()
        check(self.lib.tfmoe_profile_read(self.handle, ms, calls, 1 if reset else 0))
        return {STAGES[i]: (float(ms[i]), int(calls[i])) for i in range(n)}

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            self.lib.tfmoe_destroy(self.handle)
            self.handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def route_noalloc(x, router_w, router_bias, top_k: int, ids_out, weights_out, T: Optional[int] = None,
                  stream=None) -> int:
    """Routing through tfmoe_route_noalloc: no handle, no allocation inside the library.

    For callers that cannot allocate device memory; the logits go to the
    library's fixed per-device scratch. Returns the status code."""
    if T is None:
        T = x.shape[0]
    E, H = router_w.shape
    return load_library().tfmoe_route_noalloc(_ptr(x), T, H, _ptr(router_w), _ptr(router_bias), E, top_k,
                                              _ptr(ids_out), _ptr(weights_out), _stream_handle(stream))


class _DeviceView:
    """Exposes a raw device allocation through __cuda_array_interface__ (zero copy)."""

    _TYPESTR = {"float32": "<f4", "int32": "<i4", "int16": "<i2", "bfloat16": "<i2", "uint8": "|u1"}

    def __init__(self, ptr: int, nbytes: int, dtype):
        import torch
        name = str(dtype).replace("torch.", "")
        self.bf16 = name == "bfloat16"
        itemsize = torch.empty((), dtype=dtype).element_size()
        self.__cuda_array_interface__ = {"shape": (nbytes // itemsize,), "typestr": self._TYPESTR[name],
                                         "data": (ptr, False), "version": 3, "strides": None}


def layer_to_device(layer_np: Dict[str, object], device="cuda"):
    """Move a canonical-layout host layer (numpy arrays from synth) to device tensors."""
    import numpy as np
    import torch
    out = {}
    for k, v in layer_np.items():
        if v is None:
            out[k] = None
            continue
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            t = torch.from_numpy(a.view(np.int16))
        else:
            t = torch.from_numpy(a)
        out[k] = t.to(device)
    return out
