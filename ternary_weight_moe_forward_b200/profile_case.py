"""A small, fixed invocation of the layer for profilers (ncu and the like).

    python -m ternary_weight_moe_forward_b200.profile_case --T 64 [--iters 3] [--tc]

Builds the decode-shape layer (d_model 2048, 256 experts, top-8, d_ff 512,
seed 0), then runs `iters` forward passes at T tokens, each after a 256 MB
write that flushes L2, and exits 0.  Launch order per forward: the routing
kernel(s), then the expert kernels.  --tc forces the tensor-core expert path
(T up to 4096 uses it by default above the decode limit).
"""
from __future__ import annotations

import argparse

import torch

from . import MAPLE_CFG_FORCE_TC, synth
from .layer import Layer, bf16_from_bits


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=64)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--tc", action="store_true")
    args = ap.parse_args()
    shape = synth.CONFIGS["decode"]["shape"]
    w = synth.layer_weights(shape, seed=0)
    layer = Layer(shape, w, max_tokens=max(args.T, 64), flags=MAPLE_CFG_FORCE_TC if args.tc else 0)
    del w
    x = bf16_from_bits(synth.activations(args.T, shape.d_model, seed=0), "cuda")
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    for _ in range(args.iters):
        flush.fill_(1.0)
        layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_flags() == 0
    layer.close()


if __name__ == "__main__":
    main()
