"""ctypes front end of the CPU oracle (test infrastructure).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this module.  The CUDA library has no path into it.

The oracle itself is plain C (maple_oracle.c); this file only marshals numpy
arrays into it.  Weights are handed over unpacked (int8 in {-1, 0, +1}); the
oracle packs them into the 2-bit interchange format with its own packer and
computes from the packed codes.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.orc_pack_ternary.argtypes = [P, C.c_int64, C.c_int32, P]
        L.orc_unpack_ternary.argtypes = [P, C.c_int64, C.c_int32, P]
        L.orc_exp.argtypes = [C.c_float]
        L.orc_exp.restype = C.c_float
        L.orc_exp_array.argtypes = [P, C.c_int64, P]
        L.orc_quantize_row.argtypes = [P, C.c_int32, P, P]
        L.orc_router_logit.argtypes = [P, P, C.c_int32]
        L.orc_router_logit.restype = C.c_float
        L.orc_topk.argtypes = [P, C.c_int32, C.c_int32, P]
        L.orc_softmax_kept.argtypes = [P, C.c_int32, P]
        L.orc_permute.argtypes = [P, C.c_int32, C.c_int32, C.c_int32, P, P, P, P]
        L.orc_route.argtypes = [P, P, P, C.c_int32, P, P, P]
        L.orc_forward_tokens.argtypes = [P, P, P, P, C.c_int32, P, P]
        L.orc_rmsnorm_bf16.argtypes = [P, C.c_int32, P]
        L.orc_stack_forward.argtypes = [P, P, C.c_int32, P, C.c_int32]
        _lib = L
    return _lib


class _Shape(C.Structure):
    _fields_ = [("d_model", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32), ("d_ff", C.c_int32)]


class _Weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_gate", "w_up", "w_down", "alpha_gate", "alpha_up",
                                          "alpha_down", "router_w", "router_bias")]


_TAP_FIELDS = ("q_x", "s_x", "logits", "topk_idx", "topk_w", "acc_gate", "acc_up", "h", "q_h", "s_h",
               "acc_down", "y_e")


class _Taps(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _TAP_FIELDS]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


# ------------------------------------------------------------------ building blocks
def pack_ternary(t: np.ndarray) -> np.ndarray:
    """int8 [..., cols] in {-1,0,1} -> uint32 [..., cols/16] (interchange format)."""
    t = np.ascontiguousarray(t, dtype=np.int8)
    cols = t.shape[-1]
    rows = t.size // cols if cols else 0
    out = np.empty(t.shape[:-1] + (cols // 16,), dtype=np.uint32)
    _check(lib().orc_pack_ternary(_ptr(t), rows, cols, _ptr(out)), "pack")
    return out


def unpack_ternary(p: np.ndarray, cols: int) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint32)
    rows = p.size // (cols // 16)
    out = np.empty(p.shape[:-1] + (cols,), dtype=np.int8)
    _check(lib().orc_unpack_ternary(_ptr(p), rows, cols, _ptr(out)), "unpack")
    return out


def exp(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    lib().orc_exp_array(_ptr(x), x.size, _ptr(out))
    return out


def quantize_row(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float32)
    q = np.empty(v.shape, dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    lib().orc_quantize_row(_ptr(v), v.size, _ptr(q), _ptr(s))
    return q, float(s[0])


def router_logit(x: np.ndarray, w: np.ndarray) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    return float(lib().orc_router_logit(_ptr(x), _ptr(w), x.size))


def topk(logits: np.ndarray, k: int) -> np.ndarray:
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    idx = np.empty(k, dtype=np.int32)
    _check(lib().orc_topk(_ptr(logits), logits.size, k, _ptr(idx)), "topk")
    return idx


def softmax_kept(kept: np.ndarray) -> np.ndarray:
    kept = np.ascontiguousarray(kept, dtype=np.float32)
    w = np.empty_like(kept)
    lib().orc_softmax_kept(_ptr(kept), kept.size, _ptr(w))
    return w


def permute(idx: np.ndarray, n_experts: int):
    """idx [T][K] -> counts [E], offsets [E+1], perm [T*K], inv [T*K]."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    counts = np.empty(n_experts, dtype=np.int32)
    offsets = np.empty(n_experts + 1, dtype=np.int32)
    perm = np.empty(T * K, dtype=np.int32)
    inv = np.empty(T * K, dtype=np.int32)
    _check(lib().orc_permute(_ptr(idx), T, K, n_experts, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv)),
           "permute")
    return counts, offsets, perm, inv


def rmsnorm_bf16(r: np.ndarray) -> np.ndarray:
    r = np.ascontiguousarray(r, dtype=np.float32)
    out = np.empty(r.shape, dtype=np.uint16)
    D = r.shape[-1]
    for i in range(r.size // D):
        lib().orc_rmsnorm_bf16(_ptr(r.reshape(-1, D)[i]), D, _ptr(out.reshape(-1, D)[i]))
    return out


# ------------------------------------------------------------------ a whole layer
class Layer:
    """One MoE layer held by the oracle: packed codes, scales, router."""

    def __init__(self, shape, weights: dict):
        self.shape = shape
        self.packed = {k: pack_ternary(weights[k]) for k in ("gate", "up", "down")}
        self.f32 = {k: np.ascontiguousarray(weights[k], dtype=np.float32)
                    for k in ("alpha_gate", "alpha_up", "alpha_down", "router_w")}
        b = weights.get("router_bias")
        self.bias = None if b is None else np.ascontiguousarray(b, dtype=np.float32)
        self._shape_c = _Shape(shape.d_model, shape.n_experts, shape.top_k, shape.d_ff)
        self._w_c = _Weights(*[_ptr(a) for a in (self.packed["gate"], self.packed["up"], self.packed["down"],
                                                  self.f32["alpha_gate"], self.f32["alpha_up"],
                                                  self.f32["alpha_down"], self.f32["router_w"], self.bias)])

    def route(self, x_bits: np.ndarray):
        """All tokens: logits [T][E], idx [T][K], w [T][K]."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        T = x_bits.shape[0]
        s = self.shape
        logits = np.empty((T, s.n_experts), dtype=np.float32)
        idx = np.empty((T, s.top_k), dtype=np.int32)
        w = np.empty((T, s.top_k), dtype=np.float32)
        _check(lib().orc_route(C.byref(self._shape_c), C.byref(self._w_c), _ptr(x_bits), T, _ptr(logits),
                               _ptr(idx), _ptr(w)), "route")
        return logits, idx, w

    def forward_tokens(self, x_bits: np.ndarray, tokens=None, taps: bool = True) -> dict:
        """y and (optionally) every intermediate for the listed tokens."""
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
        if tokens is None:
            tokens = np.arange(x_bits.shape[0], dtype=np.int32)
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tokens.size
        s = self.shape
        D, E, K, F = s.d_model, s.n_experts, s.top_k, s.d_ff
        out = {"y": np.empty((n, D), dtype=np.float32)}
        t_c = None
        if taps:
            spec = {"q_x": ((n, D), np.int8), "s_x": ((n,), np.float32), "logits": ((n, E), np.float32),
                    "topk_idx": ((n, K), np.int32), "topk_w": ((n, K), np.float32),
                    "acc_gate": ((n, K, F), np.int32), "acc_up": ((n, K, F), np.int32),
                    "h": ((n, K, F), np.float32), "q_h": ((n, K, F), np.int8), "s_h": ((n, K), np.float32),
                    "acc_down": ((n, K, D), np.int32), "y_e": ((n, K, D), np.float32)}
            for k, (shp, dt) in spec.items():
                out[k] = np.empty(shp, dtype=dt)
            t_c = _Taps(*[_ptr(out[k]) for k in _TAP_FIELDS])
        _check(lib().orc_forward_tokens(C.byref(self._shape_c), C.byref(self._w_c), _ptr(x_bits), _ptr(tokens),
                                        n, _ptr(out["y"]), C.byref(t_c) if t_c is not None else None),
               "forward")
        return out


def stack_forward(layers, resid: np.ndarray) -> np.ndarray:
    """Residual stream after all layers: resid + MoE(RMSNorm(resid)), layer by layer."""
    resid = np.array(resid, dtype=np.float32, copy=True, order="C")
    shape = layers[0].shape
    arr = (_Weights * len(layers))(*[l._w_c for l in layers])
    _check(lib().orc_stack_forward(C.byref(layers[0]._shape_c), arr, len(layers), _ptr(resid), resid.shape[0]),
           "stack")
    return resid
