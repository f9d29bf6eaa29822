"""Torch-side convenience around the C ABI: device allocation and marshalling.

Layer uploads one layer's weights (int8 ternary values, scales, router),
packs the ternary values on the device with maple_moe_pack_ternary, creates
the library handle and offers route() / forward() that allocate outputs with
torch and call the library.  No arithmetic of the layer happens here.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (MAPLE_OK, make_taps, maple_moe_config, maple_moe_create, maple_moe_destroy, maple_moe_device_flags,
               maple_moe_forward, maple_moe_pack_ternary, maple_moe_route, maple_moe_weights)


def _dev(a, device, dtype=None):
    if isinstance(a, torch.Tensor):
        t = a.to(device)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a)).to(device)
    if dtype is not None and t.dtype != dtype:
        t = t.to(dtype)
    return t.contiguous()


def bf16_from_bits(bits, device) -> torch.Tensor:
    """uint16 bf16 bit patterns (numpy) -> torch.bfloat16 tensor on device."""
    if isinstance(bits, torch.Tensor):
        return bits.to(device)
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def pack_on_device(values: torch.Tensor, stream=None) -> torch.Tensor:
    """int8 [..., cols] on device -> uint32 codes [..., cols/16] (as int32 tensor)."""
    cols = values.shape[-1]
    rows = values.numel() // cols
    packed = torch.empty(values.shape[:-1] + (cols // 16,), dtype=torch.int32, device=values.device)
    bad = torch.zeros(1, dtype=torch.int32, device=values.device)
    maple_moe_pack_ternary(values, rows, cols, packed, bad, stream)
    return packed, bad


class Layer:
    """One ternary MoE layer living on a CUDA device."""

    def __init__(self, shape, weights: dict, max_tokens: int, device="cuda", decode_max_tokens: int = 0,
                 flags: int = 0, stream=None):
        self.shape = shape
        self.device = torch.device(device)
        self.max_tokens = max_tokens
        st = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        packed = {}
        bad_total = 0
        for k in ("gate", "up", "down"):
            vals = _dev(weights[k], self.device, torch.int8)
            packed[k], bad = pack_on_device(vals, st)
            del vals
            bad_total += bad
        f32 = {k: _dev(weights[k], self.device, torch.float32)
               for k in ("alpha_gate", "alpha_up", "alpha_down", "router_w")}
        bias = weights.get("router_bias")
        bias_t = None if bias is None else _dev(bias, self.device, torch.float32)
        cfg = maple_moe_config(shape.d_model, shape.n_experts, shape.top_k, shape.d_ff, max_tokens,
                               decode_max_tokens, flags)
        w = maple_moe_weights(packed["gate"].data_ptr(), packed["up"].data_ptr(), packed["down"].data_ptr(),
                              f32["alpha_gate"].data_ptr(), f32["alpha_up"].data_ptr(), f32["alpha_down"].data_ptr(),
                              f32["router_w"].data_ptr(), None if bias_t is None else bias_t.data_ptr())
        self.handle = maple_moe_create(cfg, w, st)
        torch.cuda.synchronize(self.device)
        if int(bad_total.item()) != 0:
            self.close()
            raise ValueError("ternary weights hold values outside {-1, 0, +1}")
        self.packed = packed  # interchange format, kept for inspection

    # -- calls ---------------------------------------------------------------
    def _stream(self, stream):
        return stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream

    def route(self, x: torch.Tensor, stream=None):
        T = x.shape[0]
        s = self.shape
        idx = torch.empty((T, s.top_k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, s.top_k), dtype=torch.float32, device=self.device)
        counts = torch.empty((s.n_experts,), dtype=torch.int32, device=self.device)
        maple_moe_route(self.handle, x, T, idx, w, counts, self._stream(stream))
        return idx, w, counts

    def alloc_taps(self, T: int) -> dict:
        s = self.shape
        D, E, K, F = s.d_model, s.n_experts, s.top_k, s.d_ff
        dev = self.device
        spec = {"q_x": ((T, D), torch.int8), "s_x": ((T,), torch.float32), "logits": ((T, E), torch.float32),
                "topk_idx": ((T, K), torch.int32), "topk_w": ((T, K), torch.float32),
                "acc_gate": ((T, K, F), torch.int32), "acc_up": ((T, K, F), torch.int32),
                "q_h": ((T, K, F), torch.int8), "s_h": ((T, K), torch.float32),
                "acc_down": ((T, K, D), torch.int32), "expert_counts": ((E,), torch.int32),
                "expert_offsets": ((E + 1,), torch.int32), "perm": ((T * K,), torch.int32)}
        return {k: torch.full(shp, -7, dtype=dt, device=dev) for k, (shp, dt) in spec.items()}

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, taps: dict | None = None, stream=None):
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.shape.d_model), dtype=torch.float32, device=self.device)
        maple_moe_forward(self.handle, x, T, y, make_taps(**taps) if taps else None, self._stream(stream))
        return y

    def device_flags(self, clear: bool = False) -> int:
        return maple_moe_device_flags(self.handle, clear)

    def close(self):
        if getattr(self, "handle", None):
            maple_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def upload_layer(shape, weights: dict, max_tokens: int, device="cuda", **kw) -> Layer:
    return Layer(shape, weights, max_tokens, device=device, **kw)
