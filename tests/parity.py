"""Helpers shared by the GPU parity tests: run the CUDA layer and the oracle on
the same seeded inputs and compare them element by element."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from ternary_weight_moe_forward_b200 import synth
from ternary_weight_moe_forward_b200.layer import Layer, bf16_from_bits

# fp32 layer output: max |y_gpu - y_ref| / max |y_ref| per output tensor
Y_TOL = 1e-3


def max_rel(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.max(np.abs(ref)))
    if den == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got.astype(np.float64) - ref.astype(np.float64)))) / den


def gpu_forward_with_taps(layer: Layer, x_bits: np.ndarray):
    x = bf16_from_bits(x_bits, layer.device)
    taps = layer.alloc_taps(x.shape[0])
    y = layer.forward(x, taps=taps)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in taps.items()}
    out["y"] = y.cpu().numpy()
    return out


def compare_tokens(shape, g: dict, ref: dict, tokens: np.ndarray, route_only: bool = False) -> dict:
    """Compare GPU taps (all tokens) with oracle taps for `tokens`; asserts."""
    K = shape.top_k
    T = g["q_x"].shape[0]
    assert np.array_equal(g["q_x"][tokens], ref["q_x"]), "q_x"
    assert np.array_equal(g["s_x"][tokens].view(np.uint32), ref["s_x"].view(np.uint32)), "s_x"
    assert np.array_equal(g["logits"][tokens].view(np.uint32), ref["logits"].view(np.uint32)), "logits"
    assert np.array_equal(g["topk_idx"][tokens], ref["topk_idx"]), "topk_idx"
    assert np.array_equal(g["topk_w"][tokens].view(np.uint32), ref["topk_w"].view(np.uint32)), "topk_w"
    if route_only:
        return {}
    F, D = shape.d_ff, shape.d_model
    acc_g = g["acc_gate"].reshape(T, K, F)[tokens]
    acc_u = g["acc_up"].reshape(T, K, F)[tokens]
    acc_d = g["acc_down"].reshape(T, K, D)[tokens]
    assert np.array_equal(acc_g, ref["acc_gate"]), "acc_gate"
    assert np.array_equal(acc_u, ref["acc_up"]), "acc_up"
    assert np.array_equal(g["q_h"].reshape(T, K, F)[tokens], ref["q_h"]), "q_h"
    assert np.array_equal(g["s_h"].reshape(T, K)[tokens].view(np.uint32), ref["s_h"].view(np.uint32)), "s_h"
    assert np.array_equal(acc_d, ref["acc_down"]), "acc_down"
    rel = max_rel(g["y"][tokens], ref["y"])
    assert rel <= Y_TOL, f"y max rel err {rel}"
    return {"y_rel": rel, "y_bit_exact": bool(np.array_equal(g["y"][tokens].view(np.uint32), ref["y"].view(np.uint32)))}


def compare_permutation(shape, g: dict, idx_ref: np.ndarray):
    counts, offsets, perm, inv = oracle.permute(idx_ref, shape.n_experts)
    assert np.array_equal(g["expert_counts"], counts), "expert_counts"
    assert np.array_equal(g["expert_offsets"], offsets), "expert_offsets"
    assert np.array_equal(g["perm"], perm), "perm"


# ---------------------------------------------------------------------------- the oracle over many tokens
# Tokens are independent in the layer, so the single-threaded oracle can run on
# shards of tokens in parallel processes; each worker builds the layer once from
# the seeded generator (nothing of the GPU path crosses into the workers).
_WORKER_LAYER = None


def _oracle_worker_init(shape, seed: int, zipf):
    global _WORKER_LAYER
    _WORKER_LAYER = oracle.Layer(shape, synth.layer_weights(shape, seed=seed, zipf=zipf))


def _oracle_worker_run(job):
    t0, x_rows = job
    return t0, _WORKER_LAYER.forward_tokens(x_rows, np.arange(x_rows.shape[0], dtype=np.int32))


def oracle_shards(shape, seed: int, zipf, x_bits: np.ndarray, shard: int = 32, workers: int | None = None):
    """Yield (tokens, oracle taps for those tokens) over every token of x_bits,
    computed by a pool of spawned processes (started fresh, so it is safe after
    CUDA is initialised in this process)."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    T = x_bits.shape[0]
    workers = workers or max(1, min(os.cpu_count() or 1, 64))
    jobs = [(t0, np.ascontiguousarray(x_bits[t0:t0 + shard])) for t0 in range(0, T, shard)]
    ctx = mp.get_context("spawn")
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=ctx, initializer=_oracle_worker_init,
                                initargs=(shape, seed, zipf)) as pool:
        for t0, ref in pool.map(_oracle_worker_run, jobs, chunksize=1):
            yield np.arange(t0, t0 + ref["y"].shape[0], dtype=np.int32), ref


def compare_all_tokens(shape, g: dict, seed: int, zipf, x_bits: np.ndarray) -> dict:
    """Every token of a GPU forward (taps in g) against the oracle; asserts.
    Returns the worst y error and whether y agreed bit for bit everywhere."""
    worst, exact, n = 0.0, True, 0
    for tokens, ref in oracle_shards(shape, seed, zipf, x_bits):
        res = compare_tokens(shape, g, ref, tokens)
        worst = max(worst, res["y_rel"])
        exact = exact and res["y_bit_exact"]
        n += tokens.size
    assert n == x_bits.shape[0]
    return {"y_rel": worst, "y_bit_exact": exact}
