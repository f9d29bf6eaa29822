"""Ternary-weight mixture-of-experts FFN layer for NVIDIA B200 (sm_100a).

A thin ctypes binding of libmaple_moe.so, whose C ABI is declared in
include/maple_moe.h.  Functions keep the C names and only marshal arguments:
a pointer argument takes a torch tensor (its data_ptr()), an int, or None.
Every step of the layer runs in the library's CUDA kernels; there is no CPU
path.  PyTorch is used only to allocate device memory and to supply streams.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmaple_moe.so")

MAPLE_OK = 0
MAPLE_ERR_INVALID_ARG = -1
MAPLE_ERR_UNSUPPORTED_SHAPE = -2
MAPLE_ERR_OOM = -3
MAPLE_ERR_CUDA = -4
MAPLE_ERR_TIMEOUT = -5
MAPLE_ERR_DEVICE_FLAG = -6

MAPLE_FLAG_NAN_LOGIT = 0x1
MAPLE_FLAG_BAD_INDEX = 0x2
MAPLE_FLAG_BAD_VALUE = 0x4
MAPLE_FLAG_TIMEOUT = 0x8

MAPLE_CFG_FORCE_GEMV = 0x1
MAPLE_CFG_FORCE_TC = 0x2
MAPLE_CFG_DECODE_ONLY = 0x4

MAPLE_DEBUG_STALL_DOWN = 0x1
MAPLE_DEBUG_SPLIT_SMALL = 0x2

MAPLE_PATH_TC = 0
MAPLE_PATH_DECODE = 1
MAPLE_PATH_DECODE_FUSED = 2

EXPORTED = ("maple_moe_status_string", "maple_moe_pack_ternary", "maple_moe_create", "maple_moe_route",
            "maple_moe_forward", "maple_moe_stack_forward", "maple_moe_set_stage_events", "maple_moe_device_flags",
            "maple_moe_destroy", "maple_moe_route_noalloc", "maple_moe_set_debug", "maple_moe_expert_path")


class MapleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {maple_moe_status_string(code)} ({code})")
        self.code = code


class maple_moe_config(C.Structure):
    _fields_ = [("d_model", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32), ("d_ff", C.c_int32),
                ("max_tokens", C.c_int32), ("decode_max_tokens", C.c_int32), ("flags", C.c_uint32)]


class maple_moe_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_gate", "w_up", "w_down", "alpha_gate", "alpha_up", "alpha_down",
                                          "router_w", "router_bias")]


TAP_FIELDS = ("q_x", "s_x", "logits", "topk_idx", "topk_w", "acc_gate", "acc_up", "q_h", "s_h", "acc_down",
              "expert_counts", "expert_offsets", "perm")


class maple_moe_taps(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in TAP_FIELDS]


_lib = None


def lib():
    """Load libmaple_moe.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m ternary_weight_moe_forward_b200.build_lib`")
        L = C.CDLL(LIB_PATH)
        P, I32, I64 = C.c_void_p, C.c_int32, C.c_int64
        L.maple_moe_status_string.argtypes = [C.c_int]
        L.maple_moe_status_string.restype = C.c_char_p
        L.maple_moe_pack_ternary.argtypes = [P, I64, I32, P, P, P]
        L.maple_moe_create.argtypes = [C.POINTER(maple_moe_config), C.POINTER(maple_moe_weights), P, C.POINTER(P)]
        L.maple_moe_route.argtypes = [P, P, I32, P, P, P, P]
        L.maple_moe_forward.argtypes = [P, P, I32, P, C.POINTER(maple_moe_taps), P]
        L.maple_moe_stack_forward.argtypes = [C.POINTER(P), I32, P, I32, P]
        L.maple_moe_set_stage_events.argtypes = [P, C.POINTER(C.c_void_p), I32]
        L.maple_moe_device_flags.argtypes = [P, C.POINTER(C.c_uint32), I32]
        L.maple_moe_destroy.argtypes = [P]
        L.maple_moe_route_noalloc.argtypes = [P, I32, I32, I32, I32, P, P, P, P, P, P]
        L.maple_moe_set_debug.argtypes = [P, I32, C.c_uint32]
        L.maple_moe_expert_path.argtypes = [P, I32, C.POINTER(C.c_int32)]
        for name in EXPORTED:
            if name != "maple_moe_status_string":
                getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def _p(x):
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    return int(x)


def _check(rc: int, what: str):
    if rc != MAPLE_OK:
        raise MapleError(rc, what)


def maple_moe_status_string(code: int) -> str:
    return lib().maple_moe_status_string(code).decode()


def maple_moe_pack_ternary(values, rows: int, cols: int, packed, bad_count=None, stream=None) -> None:
    _check(lib().maple_moe_pack_ternary(_p(values), rows, cols, _p(packed), _p(bad_count), _p(stream)),
           "maple_moe_pack_ternary")


def maple_moe_create(config: maple_moe_config, weights: maple_moe_weights, stream=None) -> int:
    h = C.c_void_p()
    _check(lib().maple_moe_create(C.byref(config), C.byref(weights), _p(stream), C.byref(h)), "maple_moe_create")
    return h.value


def maple_moe_route(handle, x, T: int, topk_idx=None, topk_w=None, expert_counts=None, stream=None) -> None:
    _check(lib().maple_moe_route(handle, _p(x), T, _p(topk_idx), _p(topk_w), _p(expert_counts), _p(stream)),
           "maple_moe_route")


def make_taps(**tensors) -> maple_moe_taps:
    return maple_moe_taps(*[_p(tensors.get(n)) for n in TAP_FIELDS])


def maple_moe_forward(handle, x, T: int, y, taps: maple_moe_taps | None = None, stream=None) -> None:
    _check(lib().maple_moe_forward(handle, _p(x), T, _p(y), C.byref(taps) if taps is not None else None, _p(stream)),
           "maple_moe_forward")


def maple_moe_stack_forward(handles, resid, T: int, stream=None) -> None:
    arr = (C.c_void_p * len(handles))(*handles)
    _check(lib().maple_moe_stack_forward(arr, len(handles), _p(resid), T, _p(stream)), "maple_moe_stack_forward")


def maple_moe_set_stage_events(handle, events) -> None:
    """events: four torch.cuda.Event (recorded once so they exist) or None."""
    if events is None:
        _check(lib().maple_moe_set_stage_events(handle, None, 0), "maple_moe_set_stage_events")
        return
    arr = (C.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().maple_moe_set_stage_events(handle, arr, len(events)), "maple_moe_set_stage_events")


def maple_moe_device_flags(handle, clear: bool = False) -> int:
    f = C.c_uint32()
    _check(lib().maple_moe_device_flags(handle, C.byref(f), 1 if clear else 0), "maple_moe_device_flags")
    return f.value


def maple_moe_route_noalloc(x, T: int, d_model: int, n_experts: int, top_k: int, router_w, router_bias,
                            topk_idx, topk_w, expert_counts=None, stream=None) -> None:
    """Routing with no device allocation (scratch in a fixed array of the library)."""
    _check(lib().maple_moe_route_noalloc(_p(x), T, d_model, n_experts, top_k, _p(router_w), _p(router_bias),
                                         _p(topk_idx), _p(topk_w), _p(expert_counts), _p(stream)),
           "maple_moe_route_noalloc")


def maple_moe_set_debug(handle, wait_limit_us: int = 0, debug_flags: int = 0) -> None:
    """Wait limit of the handle's bounded device waits (0 = 2 s) and test hooks."""
    _check(lib().maple_moe_set_debug(handle, wait_limit_us, debug_flags), "maple_moe_set_debug")


def maple_moe_expert_path(handle, T: int) -> int:
    """MAPLE_PATH_* of a forward of T tokens on this handle."""
    p = C.c_int32(-1)
    _check(lib().maple_moe_expert_path(handle, T, C.byref(p)), "maple_moe_expert_path")
    return p.value


def maple_moe_destroy(handle) -> None:
    _check(lib().maple_moe_destroy(handle), "maple_moe_destroy")


from .layer import Layer, upload_layer  # noqa: E402  (torch-side convenience)
