"""Failure handling on the GPU, without a fault: a bounded wait made to run out.

maple_moe_set_debug shortens every bounded wait of a handle to 1 ms and makes
the decode path's down kernel wait for a device word that nothing sets.  The forward pass must come back in bounded
time with MAPLE_FLAG_TIMEOUT raised, the next call must report
MAPLE_ERR_TIMEOUT (after resetting the handle's counters), and the call after
that, with the hook off, must match the oracle bit for bit.  Nothing faults,
traps or hangs: the waits give up and the kernel returns.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import ternary_weight_moe_forward_b200 as tw
from ternary_weight_moe_forward_b200 import synth
from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits

from parity import compare_permutation, compare_tokens, gpu_forward_with_taps

pytestmark = pytest.mark.gpu

TINY = synth.CONFIGS["tiny"]["shape"]
BIG = synth.CONFIGS["decode"]["shape"]


@pytest.mark.parametrize("shape,T", [(TINY, 8), (BIG, 32)])
def test_expired_wait_reports_timeout_and_recovers(shape, T):
    w = synth.layer_weights(shape, seed=4)
    L_orc, L_gpu = oracle.Layer(shape, w), Layer(shape, w, max_tokens=64)
    x_bits = synth.activations(T, shape.d_model, seed=9)
    x = bf16_from_bits(x_bits, "cuda")
    tw.maple_moe_set_debug(L_gpu.handle, 1000, tw.MAPLE_DEBUG_STALL_DOWN)
    t0 = time.perf_counter()
    L_gpu.forward(x)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0, "the stalled forward did not give up in bounded time"
    assert L_gpu.device_flags() & tw.MAPLE_FLAG_TIMEOUT
    tw.maple_moe_set_debug(L_gpu.handle, 0, 0)
    with pytest.raises(tw.MapleError) as e:
        L_gpu.forward(x)
    assert e.value.code == tw.MAPLE_ERR_TIMEOUT
    torch.cuda.synchronize()
    assert L_gpu.device_flags() == 0
    # the counters were reset: the next forward is exact again, twice in a row
    for _ in range(2):
        g = gpu_forward_with_taps(L_gpu, x_bits)
        tokens = np.arange(T, dtype=np.int32)
        ref = L_orc.forward_tokens(x_bits, tokens)
        res = compare_tokens(shape, g, ref, tokens)
        compare_permutation(shape, g, ref["topk_idx"])
        assert res["y_bit_exact"]
    L_gpu.close()


def test_set_debug_rejects_bad_arguments():
    w = synth.layer_weights(TINY, seed=4)
    L_gpu = Layer(TINY, w, max_tokens=8)
    for limit, flags in ((-1, 0), (60000001, 0), (0, 0x80)):
        with pytest.raises(tw.MapleError) as e:
            tw.maple_moe_set_debug(L_gpu.handle, limit, flags)
        assert e.value.code == tw.MAPLE_ERR_INVALID_ARG
    L_gpu.close()
