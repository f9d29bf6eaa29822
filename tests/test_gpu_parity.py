"""GPU parity: the CUDA layer against the CPU oracle on the same seeded inputs.

Bit-exact: int8 codes and scales, router logits, expert indices and weights,
per-expert counts/offsets/permutation, the int32 accumulators of all three
contractions.  fp32 layer output: max relative error <= 1e-3 (it is expected
to be bit-exact too; the tests report it).
"""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_moe_forward_b200 import synth
from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits

from parity import (Y_TOL, compare_all_tokens, compare_permutation, compare_tokens, gpu_forward_with_taps,
                    max_rel)

pytestmark = pytest.mark.gpu

TINY = synth.CONFIGS["tiny"]["shape"]
BIG = synth.CONFIGS["decode"]["shape"]


@pytest.fixture(scope="module")
def tiny():
    w = synth.layer_weights(TINY, seed=0)
    return w, oracle.Layer(TINY, w), Layer(TINY, w, max_tokens=512)


@pytest.fixture(scope="module")
def big_weights():
    return synth.layer_weights(BIG, seed=0)


@pytest.fixture(scope="module")
def big(big_weights):
    return oracle.Layer(BIG, big_weights), Layer(BIG, big_weights, max_tokens=4096)


def _full_check(shape, L_orc, L_gpu, x_bits):
    g = gpu_forward_with_taps(L_gpu, x_bits)
    tokens = np.arange(x_bits.shape[0], dtype=np.int32)
    ref = L_orc.forward_tokens(x_bits, tokens)
    res = compare_tokens(shape, g, ref, tokens)
    compare_permutation(shape, g, ref["topk_idx"])
    return g, ref, res


def test_pack_kernel_matches_oracle_packer(tiny, big_weights):
    w, L_orc, L_gpu = tiny
    for k in ("gate", "up", "down"):
        assert np.array_equal(L_gpu.packed[k].cpu().numpy().view(np.uint32), L_orc.packed[k])
    from ternary_weight_moe_forward_b200.layer import pack_on_device
    vals = torch.from_numpy(big_weights["gate"][:4]).cuda()
    packed, bad = pack_on_device(vals)
    assert int(bad.item()) == 0
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack_ternary(big_weights["gate"][:4]))


def test_pack_kernel_counts_invalid_values():
    vals = torch.zeros((2, 32), dtype=torch.int8, device="cuda")
    vals[0, 3] = 2
    vals[1, 31] = -5
    from ternary_weight_moe_forward_b200.layer import pack_on_device
    packed, bad = pack_on_device(vals)
    assert int(bad.item()) == 2
    assert not packed.any()


def test_tiny_config_full_parity(tiny):
    w, L_orc, L_gpu = tiny
    x = synth.activations(8, TINY.d_model, seed=0)
    _, _, res = _full_check(TINY, L_orc, L_gpu, x)
    assert res["y_rel"] <= Y_TOL


@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_decode_config_full_parity(big, T):
    L_orc, L_gpu = big
    x = synth.activations(T, BIG.d_model, seed=0)
    _full_check(BIG, L_orc, L_gpu, x)


@pytest.mark.parametrize("T", [3, 65, 200])
def test_ragged_token_counts(tiny, T):
    w, L_orc, L_gpu = tiny
    x = synth.activations(T, TINY.d_model, seed=T)
    _full_check(TINY, L_orc, L_gpu, x)


def test_zero_tokens_is_a_noop(tiny):
    w, L_orc, L_gpu = tiny
    x = torch.empty((0, TINY.d_model), dtype=torch.bfloat16, device="cuda")
    y = torch.full((1, TINY.d_model), 7.0, device="cuda")
    L_gpu.forward(x, y=y)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)


def test_zero_rows_and_ties(tiny):
    w, L_orc, L_gpu = tiny
    # identical router rows for experts 3 and 9 and 4 and 5 -> equal logits, lower index first
    w2 = dict(w)
    rw = w["router_w"].copy()
    rw[9] = rw[3]
    rw[5] = rw[4]
    w2["router_w"] = rw
    Lo, Lg = oracle.Layer(TINY, w2), Layer(TINY, w2, max_tokens=64)
    x = synth.activations(16, TINY.d_model, seed=3)
    x[5] = 0        # an all-zero token
    g, ref, _ = _full_check(TINY, Lo, Lg, x)
    assert not g["y"][5].any()
    Lg.close()


def test_all_tokens_to_the_same_experts(tiny):
    w, L_orc, L_gpu = tiny
    w2 = dict(w)
    b = np.zeros(TINY.n_experts, np.float32)
    b[[2, 11]] = 1000.0
    w2["router_bias"] = b
    Lo, Lg = oracle.Layer(TINY, w2), Layer(TINY, w2, max_tokens=512)
    for T in (8, 64, 300):
        x = synth.activations(T, TINY.d_model, seed=T + 1)
        g, ref, _ = _full_check(TINY, Lo, Lg, x)
        assert g["expert_counts"][2] == T and g["expert_counts"][11] == T
    Lg.close()


def test_deterministic_bits(big):
    L_orc, L_gpu = big
    x = bf16_from_bits(synth.activations(64, BIG.d_model, seed=5), "cuda")
    y1 = L_gpu.forward(x).clone()
    y2 = L_gpu.forward(x).clone()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))


def test_route_entry_point(big):
    L_orc, L_gpu = big
    x_bits = synth.activations(64, BIG.d_model, seed=6)
    idx, w, counts = L_gpu.route(bf16_from_bits(x_bits, "cuda"))
    torch.cuda.synchronize()
    _, idx_ref, w_ref = L_orc.route(x_bits)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), w_ref.view(np.uint32))
    assert np.array_equal(counts.cpu().numpy(), np.bincount(idx_ref.ravel(), minlength=BIG.n_experts))


def test_nan_input_sets_the_device_flag(tiny):
    w, L_orc, L_gpu = tiny
    x = bf16_from_bits(synth.activations(8, TINY.d_model, seed=1), "cuda")
    x[2, 7] = float("nan")
    L_gpu.device_flags(clear=True)
    L_gpu.forward(x)
    torch.cuda.synchronize()
    assert L_gpu.device_flags(clear=True) & 0x1
    # a clean call afterwards succeeds
    x[2, 7] = 0.0
    L_gpu.forward(x)
    torch.cuda.synchronize()
    assert L_gpu.device_flags() == 0


def test_prefill_config_full_parity(big):
    """T=4096 (the tensor-core path): every tap of every token against the
    oracle, which runs on token shards in parallel processes."""
    L_orc, L_gpu = big
    T = 4096
    x = synth.activations(T, BIG.d_model, seed=0)
    g = gpu_forward_with_taps(L_gpu, x)
    logits, idx, w = L_orc.route(x)
    compare_permutation(BIG, g, idx)
    res = compare_all_tokens(BIG, g, 0, None, x)
    assert res["y_rel"] <= Y_TOL


# ---------------------------------------------------------------------------- both expert paths
import ternary_weight_moe_forward_b200 as tw  # noqa: E402


@pytest.mark.parametrize("T", [1, 8, 37, 300])
def test_tensor_core_path_forced_tiny(tiny, T):
    """The tcgen05 grouped GEMM at any T (pieces of 1..256 slots, ragged N)."""
    w, L_orc, _ = tiny
    Lg = Layer(TINY, w, max_tokens=512, flags=tw.MAPLE_CFG_FORCE_TC)
    x = synth.activations(T, TINY.d_model, seed=100 + T)
    _full_check(TINY, L_orc, Lg, x)
    Lg.close()


@pytest.mark.parametrize("T", [9, 33, 64])
def test_decode_kernel_forced_beyond_its_default_limit(tiny, T):
    """MAPLE_CFG_FORCE_GEMV runs the decode kernel for every T <= 64, here
    above a handle's decode_max_tokens of 8 (units of 16 slots, 2 n-tiles)."""
    w, L_orc, _ = tiny
    Lg = Layer(TINY, w, max_tokens=512, decode_max_tokens=8, flags=tw.MAPLE_CFG_FORCE_GEMV)
    x = synth.activations(T, TINY.d_model, seed=200 + T)
    _full_check(TINY, L_orc, Lg, x)
    with pytest.raises(tw.MapleError) as e:   # beyond 64 tokens there is no decode kernel
        Lg.forward(bf16_from_bits(synth.activations(65, TINY.d_model, seed=1), "cuda"))
    assert e.value.code == tw.MAPLE_ERR_UNSUPPORTED_SHAPE
    Lg.close()


def test_decode_only_handle(big_weights, big):
    """A handle with only the decode layout serves T <= 64 and rejects more."""
    L_orc, _ = big
    Lg = Layer(BIG, big_weights, max_tokens=128, flags=tw.MAPLE_CFG_DECODE_ONLY)
    x = synth.activations(16, BIG.d_model, seed=400)
    _full_check(BIG, L_orc, Lg, x)
    with pytest.raises(tw.MapleError) as e:
        Lg.forward(bf16_from_bits(synth.activations(65, BIG.d_model, seed=1), "cuda"))
    assert e.value.code == tw.MAPLE_ERR_UNSUPPORTED_SHAPE
    Lg.close()


def test_tensor_core_path_forced_decode_shape(big_weights, big):
    L_orc, _ = big
    Lg = Layer(BIG, big_weights, max_tokens=64, flags=tw.MAPLE_CFG_FORCE_TC)
    for T in (1, 64):
        x = synth.activations(T, BIG.d_model, seed=300 + T)
        _full_check(BIG, L_orc, Lg, x)
    Lg.close()


def test_paths_agree_bitwise(big_weights, big):
    """The decode kernel and the tensor-core path give identical bits on the same input."""
    Lt = Layer(BIG, big_weights, max_tokens=64, flags=tw.MAPLE_CFG_FORCE_TC)
    Lv = Layer(BIG, big_weights, max_tokens=64, flags=tw.MAPLE_CFG_FORCE_GEMV)
    x = bf16_from_bits(synth.activations(64, BIG.d_model, seed=7), "cuda")
    yt, yv = Lt.forward(x), Lv.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(yt.view(torch.int32), yv.view(torch.int32))
    Lt.close()
    Lv.close()


@pytest.mark.parametrize("T", [1, 2, 8])
def test_small_batches_two_kernel_path(big_weights, big, T):
    """Batches of at most 8 tokens normally take the fused one-kernel expert path;
    the two-kernel path (gate/up kernel, down kernel, combine) stays exact too."""
    L_orc, _ = big
    Lg = Layer(BIG, big_weights, max_tokens=64)
    tw.maple_moe_set_debug(Lg.handle, 0, tw.MAPLE_DEBUG_SPLIT_SMALL)
    x = synth.activations(T, BIG.d_model, seed=500 + T)
    _full_check(BIG, L_orc, Lg, x)
    Lg.close()


def test_small_batch_paths_agree_bitwise(big_weights):
    """The fused small-batch expert kernel and the two-kernel path give identical bits."""
    Lf = Layer(BIG, big_weights, max_tokens=64)
    Ls = Layer(BIG, big_weights, max_tokens=64)
    tw.maple_moe_set_debug(Ls.handle, 0, tw.MAPLE_DEBUG_SPLIT_SMALL)
    for T in range(1, 9):
        x = bf16_from_bits(synth.activations(T, BIG.d_model, seed=600 + T), "cuda")
        yf, ys = Lf.forward(x), Ls.forward(x)
        torch.cuda.synchronize()
        assert torch.equal(yf.view(torch.int32), ys.view(torch.int32)), T
    assert Lf.device_flags() == 0 and Ls.device_flags() == 0
    Lf.close()
    Ls.close()


def test_expert_path_query(big_weights, big):
    _, Lg = big
    assert tw.maple_moe_expert_path(Lg.handle, 1) == tw.MAPLE_PATH_DECODE_FUSED
    assert tw.maple_moe_expert_path(Lg.handle, 64) == tw.MAPLE_PATH_DECODE
    assert tw.maple_moe_expert_path(Lg.handle, 4096) == tw.MAPLE_PATH_TC
    Ls = Layer(BIG, big_weights, max_tokens=64)
    tw.maple_moe_set_debug(Ls.handle, 0, tw.MAPLE_DEBUG_SPLIT_SMALL)
    assert tw.maple_moe_expert_path(Ls.handle, 1) == tw.MAPLE_PATH_DECODE
    with pytest.raises(tw.MapleError):
        tw.maple_moe_expert_path(Ls.handle, 65)
    Ls.close()
