"""Seeded synthetic inputs for the ternary-weight MoE FFN layer.

This module only draws random numbers and lays them out as arrays.  It holds
none of the layer's arithmetic (no packing, routing, quantisation, SwiGLU or
combine), so the CPU oracle and the CUDA library can both be fed from it
without sharing any step of the computation.

Workload recipe (ternary MoE layer of the Maple-Preview 20B-A1B model, whose
architecture table -- "linlog.top/article/1232", section 架构设计 -- gives 24
layers, 256 experts, top-8 routing and ternary weights with one scale per row):

* expert weights are i.i.d. in {-1, 0, +1} with probabilities 0.3 / 0.4 / 0.3;
* the per-row scale is alpha = 0.02 * exp(0.25 * N(0, 1)) (lognormal);
* the router matrix is fp32 N(0, 1/d_model);
* activations are N(0, 1) rounded to bf16 (round to nearest even);
* the skewed workload adds a per-expert router bias log(p_rank) whose
  popularity p follows Zipf(s = 1.1) over a seeded permutation of experts.

Every tensor has its own numpy PCG64 stream derived from (seed, layer,
tensor id), so any tensor can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "LayerShape", "CONFIGS", "layer_weights", "activations", "zipf_bias",
    "bf16_bits_to_f32", "f32_to_bf16_bits", "ternary_matrix",
]

# tensor ids for the per-tensor random streams
_T_GATE, _T_UP, _T_DOWN = 1, 2, 3
_T_AGATE, _T_AUP, _T_ADOWN = 4, 5, 6
_T_ROUTER, _T_X, _T_BIAS, _T_RESID = 7, 8, 9, 10


@dataclasses.dataclass(frozen=True)
class LayerShape:
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int


_BIG = LayerShape(d_model=2048, n_experts=256, top_k=8, d_ff=512)

# The five workloads: shapes, token counts and structure.
CONFIGS = {
    "tiny": dict(shape=LayerShape(256, 16, 2, 128), tokens=[8], layers=1, zipf=None),
    "decode": dict(shape=_BIG, tokens=[1, 8, 32, 64], layers=1, zipf=None),
    "prefill": dict(shape=_BIG, tokens=[4096], layers=1, zipf=None),
    "stack": dict(shape=_BIG, tokens=[1, 32], layers=24, zipf=None),
    "skewed": dict(shape=_BIG, tokens=[16384], layers=1, zipf=1.1),
}


def _rng(seed: int, layer: int, tensor: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, layer, tensor, extra]))


_TERNARY_LUT = np.array([-1, -1, -1, 0, 0, 0, 0, 1, 1, 1], dtype=np.int8)


def ternary_matrix(rng: np.random.Generator, shape) -> np.ndarray:
    """int8 array of i.i.d. values in {-1, 0, +1}, P = 0.3 / 0.4 / 0.3."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.int8)
    step = 1 << 24
    for lo in range(0, n, step):
        hi = min(n, lo + step)
        out[lo:hi] = _TERNARY_LUT[rng.integers(0, 10, size=hi - lo, dtype=np.uint8)]
    return out.reshape(shape)


def _lognormal_alpha(rng: np.random.Generator, shape) -> np.ndarray:
    return (0.02 * np.exp(0.25 * rng.standard_normal(shape))).astype(np.float32)


def zipf_bias(n_experts: int, s: float, seed: int, layer: int = 0, scale: float = 1.0) -> np.ndarray:
    """Router bias b_e = scale * log(p_rank(e)), p_r proportional to r^-s.

    Ranks are assigned through a seeded permutation of the experts.
    """
    rng = _rng(seed, layer, _T_BIAS)
    ranks = rng.permutation(n_experts) + 1          # rank of expert e, 1-based
    p = ranks.astype(np.float64) ** (-s)
    p /= p.sum()
    return (scale * np.log(p)).astype(np.float32)


def layer_weights(shape: LayerShape, seed: int, layer: int = 0, zipf: float | None = None) -> dict:
    """All weights of one layer as plain (unpacked) arrays.

    gate, up: int8 [E][F][D]; down: int8 [E][D][F] (row = output channel);
    alpha_gate, alpha_up: f32 [E][F]; alpha_down: f32 [E][D];
    router_w: f32 [E][D]; router_bias: f32 [E] or None.
    """
    E, D, F = shape.n_experts, shape.d_model, shape.d_ff
    w = {
        "gate": ternary_matrix(_rng(seed, layer, _T_GATE), (E, F, D)),
        "up": ternary_matrix(_rng(seed, layer, _T_UP), (E, F, D)),
        "down": ternary_matrix(_rng(seed, layer, _T_DOWN), (E, D, F)),
        "alpha_gate": _lognormal_alpha(_rng(seed, layer, _T_AGATE), (E, F)),
        "alpha_up": _lognormal_alpha(_rng(seed, layer, _T_AUP), (E, F)),
        "alpha_down": _lognormal_alpha(_rng(seed, layer, _T_ADOWN), (E, D)),
        "router_w": (_rng(seed, layer, _T_ROUTER).standard_normal((E, D)) / np.sqrt(D)).astype(np.float32),
        "router_bias": None if zipf is None else zipf_bias(E, zipf, seed, layer),
    }
    return w


def layer_weights_from_args(args) -> dict:
    """layer_weights(*args): a picklable entry point for process pools."""
    return layer_weights(*args)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(n_tokens: int, d_model: int, seed: int, stream: int = 0) -> np.ndarray:
    """bf16 activations N(0, 1), as uint16 bit patterns [T][D]."""
    rng = _rng(seed, stream, _T_X, n_tokens)
    return f32_to_bf16_bits(rng.standard_normal((n_tokens, d_model)).astype(np.float32))


def residual(n_tokens: int, d_model: int, seed: int) -> np.ndarray:
    """fp32 residual stream input for the layer stack: N(0, 1) values that are bf16-exact."""
    rng = _rng(seed, 0, _T_RESID, n_tokens)
    return bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((n_tokens, d_model)).astype(np.float32)))


def layer_weights_device(shape: LayerShape, seed: int, layer: int = 0, zipf: float | None = None, device="cuda"):
    """The same distributions as layer_weights, drawn on a CUDA device with
    torch's counter-based generator (one seeded stream per tensor), for
    workloads too large to draw on the host in time (the 24-layer stack).
    These are different numbers from layer_weights' numpy streams.  Returns
    torch tensors on `device`: gate/up/down int8, the rest fp32."""
    import torch

    E, D, F = shape.n_experts, shape.d_model, shape.d_ff
    lut = torch.tensor(_TERNARY_LUT, dtype=torch.int8, device=device)

    def gen(tensor):
        g = torch.Generator(device=device)
        g.manual_seed(int(np.random.SeedSequence([seed, layer, tensor]).generate_state(1, np.uint64)[0] >> 1))
        return g

    def ternary(tensor, shp):
        return lut[torch.randint(0, 10, shp, generator=gen(tensor), device=device, dtype=torch.int64)]

    def alpha(tensor, shp):
        return 0.02 * torch.exp(0.25 * torch.randn(shp, generator=gen(tensor), device=device, dtype=torch.float32))

    w = {
        "gate": ternary(_T_GATE, (E, F, D)),
        "up": ternary(_T_UP, (E, F, D)),
        "down": ternary(_T_DOWN, (E, D, F)),
        "alpha_gate": alpha(_T_AGATE, (E, F)),
        "alpha_up": alpha(_T_AUP, (E, F)),
        "alpha_down": alpha(_T_ADOWN, (E, D)),
        "router_w": torch.randn((E, D), generator=gen(_T_ROUTER), device=device, dtype=torch.float32) / float(np.sqrt(D)),
        "router_bias": None if zipf is None else torch.from_numpy(zipf_bias(E, zipf, seed, layer)).to(device),
    }
    return w
