"""The allocation-free routing entry point against the handle-based one.

maple_moe_route_noalloc exists for callers that cannot let a library call
cudaMalloc (device memory owned by their own pool allocator, or serving loops
that forbid allocation once running); its scratch is a fixed array inside the
library.  This file is collected last so that a failure here leaves every other
test already run; it passes alone in a fresh process as well as after them.
"""
import numpy as np
import pytest
import torch

import ternary_weight_moe_forward_b200 as tw
from ternary_weight_moe_forward_b200 import synth
from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits


pytestmark = pytest.mark.gpu


def _route_weights(shape, seed, zipf=None):
    """Router weights from the seeded generator; the ternary experts are zero
    (routing does not read them), which keeps the handle cheap to build."""
    E, D, F = shape.n_experts, shape.d_model, shape.d_ff
    w = synth.layer_weights(synth.LayerShape(D, E, shape.top_k, 128), seed=seed, zipf=zipf)
    w["gate"] = np.zeros((E, F, D), np.int8)
    w["up"] = np.zeros((E, F, D), np.int8)
    w["down"] = np.zeros((E, D, F), np.int8)
    w["alpha_gate"] = np.ones((E, F), np.float32)
    w["alpha_up"] = np.ones((E, F), np.float32)
    return w


# d_model 4096 needs the raised shared-memory limit of the routing kernel; 1024
# experts take its wide top-k variant, and T * E = 16384 fills the array's limit
_SHAPES = {"tiny": synth.CONFIGS["tiny"]["shape"], "decode": synth.CONFIGS["decode"]["shape"],
           "d4096": synth.LayerShape(4096, 256, 8, 128), "e1024": synth.LayerShape(256, 1024, 8, 128)}


@pytest.mark.parametrize("name,T,zipf", [("tiny", 8, None), ("decode", 1, None), ("decode", 64, None),
                                         ("decode", 37, 1.1), ("d4096", 8, None), ("e1024", 16, None)])
def test_route_noalloc_matches_route(name, T, zipf):
    shape = _SHAPES[name]
    w = _route_weights(shape, seed=3, zipf=zipf)
    ref_layer = Layer(shape, w, max_tokens=64)
    x = bf16_from_bits(synth.activations(T, shape.d_model, seed=11), "cuda")
    idx_ref, w_ref, cnt_ref = ref_layer.route(x)
    torch.cuda.synchronize()
    rw = torch.from_numpy(w["router_w"]).cuda()
    bias = None if w["router_bias"] is None else torch.from_numpy(w["router_bias"]).cuda()
    K, E = shape.top_k, shape.n_experts
    for _ in range(2):   # two calls in a row share the scratch array
        idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
        cnt = torch.full((E,), -1, dtype=torch.int32, device="cuda")
        tw.maple_moe_route_noalloc(x, T, shape.d_model, E, K, rw, bias, idx, wt, cnt,
                                   torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        assert torch.equal(cnt, cnt_ref)
        # the same routing kernel computes both: the weights agree bit for bit
        assert torch.equal(wt.view(torch.int32), w_ref.view(torch.int32))
    ref_layer.close()


def test_route_noalloc_rejects_sizes_beyond_its_array():
    shape = synth.CONFIGS["decode"]["shape"]
    x = torch.zeros((65, shape.d_model), dtype=torch.bfloat16, device="cuda")
    rw = torch.zeros((shape.n_experts, shape.d_model), device="cuda")
    idx = torch.empty((65, 8), dtype=torch.int32, device="cuda")
    wt = torch.empty((65, 8), device="cuda")
    with pytest.raises(tw.MapleError) as e:
        tw.maple_moe_route_noalloc(x, 65, shape.d_model, shape.n_experts, 8, rw, None, idx, wt)
    assert e.value.code == tw.MAPLE_ERR_INVALID_ARG
