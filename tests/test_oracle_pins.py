"""Pins of the CPU oracle against things other than itself (no GPU).

Each test checks one oracle function against an independent source: a
hand-worked fixture under tests/golden/, a closed form, numpy float64 or int64
arithmetic, a brute-force full sort, or an invariant of the mathematics.  They
are chosen so that a plausible slip anywhere in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong rounding or order) fails at
least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle
from ternary_weight_moe_forward_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = synth.CONFIGS["tiny"]["shape"]


# ------------------------------------------------------------------ packing
def _golden_pack_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "pack_layout.txt")):
        if line.startswith("#") or not line.strip():
            continue
        vals, word = line.split("|")
        rows.append(([int(v) for v in vals.split()], int(word, 16)))
    return rows


def test_pack_matches_hand_worked_words():
    for vals, word in _golden_pack_rows():
        got = oracle.pack_ternary(np.array([vals], dtype=np.int8))
        assert got.shape == (1, 1)
        assert int(got[0, 0]) == word, (vals, hex(int(got[0, 0])), hex(word))


def test_pack_unpack_round_trip_and_invalid_code():
    rng = np.random.default_rng(1)
    t = rng.integers(-1, 2, size=(7, 64)).astype(np.int8)
    p = oracle.pack_ternary(t)
    assert np.array_equal(oracle.unpack_ternary(p, 64), t)
    # code 3 is never written; a reader treats it as 0
    p3 = np.array([[0xFFFFFFFF]], dtype=np.uint32)
    assert np.array_equal(oracle.unpack_ternary(p3, 16), np.zeros((1, 16), np.int8))
    with pytest.raises(RuntimeError):
        oracle.pack_ternary(np.full((1, 16), 2, dtype=np.int8))


# ------------------------------------------------------------------ exp
def test_exp_within_one_ulp_of_float64():
    x = np.linspace(-87.0, 88.0, 1_000_003).astype(np.float32)
    x = np.concatenate([x, np.array([0.0, -0.0, 1.0, -1.0, 1e-8, -1e-8, 0.5, 87.9, -86.9], np.float32)])
    got = oracle.exp(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(got - ref) / ulp) <= 1.0
    assert oracle.exp(np.array([0.0], np.float32))[0] == 1.0


def test_exp_clamps_outside_range():
    lo, hi = oracle.exp(np.array([-87.0, 88.0], np.float32))
    below, above = oracle.exp(np.array([-1000.0, 1000.0], np.float32))
    assert below == lo and above == hi and np.isfinite(above)


# ------------------------------------------------------------------ quantiser
def test_quantize_closed_forms():
    v = np.zeros(64, np.float32)
    v[5] = -3.25
    q, s = oracle.quantize_row(v)
    assert q[5] == -127 and np.count_nonzero(q) == 1
    assert s == np.float32(3.25) / np.float32(127.0)
    q, s = oracle.quantize_row(np.zeros(64, np.float32))
    assert s == 0.0 and not q.any()
    # amax element maps to exactly +-127 and half of amax to 64 (63.5 -> 64, ties to even)
    v = np.array([2.0, 1.0, -2.0, 0.0] + [0.0] * 12, np.float32)
    q, s = oracle.quantize_row(v)
    assert list(q[:4]) == [127, 64, -127, 0]


def test_quantize_is_nearest_code_and_scale_invariant():
    rng = np.random.default_rng(2)
    for _ in range(20):
        v = rng.standard_normal(512).astype(np.float32) * np.float32(rng.uniform(0.01, 100))
        q, s = oracle.quantize_row(v)
        amax = np.max(np.abs(v.astype(np.float64)))
        exact = v.astype(np.float64) * 127.0 / amax
        assert np.all(np.abs(q - exact) <= 0.5 + 1e-4)
        assert np.all(np.abs(q) <= 127) and np.max(np.abs(q)) == 127
        assert abs(s - amax / 127.0) <= 1e-7 * amax
        # multiplying by a power of two leaves the codes alone and scales s exactly
        q2, s2 = oracle.quantize_row(v * np.float32(8.0))
        assert np.array_equal(q, q2) and s2 == s * 8.0


# ------------------------------------------------------------------ router
def _golden_router_cases():
    """(D, [(j, w_j)], expected logit, exact sum) per line; a leading D=... token
    gives the row length (256 otherwise)."""
    cases = []
    for line in open(os.path.join(GOLDEN, "router_order.txt")):
        if line.startswith("#") or not line.strip():
            continue
        terms, expect, exact = line.split("|")
        D, pairs = 256, []
        for t in terms.split():
            k, v = t.split("=")
            if k == "D":
                D = int(v)
            else:
                pairs.append((int(k), int(v)))
        cases.append((D, pairs, float(expect), float(exact)))
    return cases


def test_router_order_hand_worked_cases():
    cases = _golden_router_cases()
    assert {c[0] for c in cases} >= {256, 512, 2048}
    for D, terms, expect, exact in cases:
        x = np.zeros(D, np.float32)
        w = np.zeros(D, np.float32)
        for j, wj in terms:
            x[j] = 1.0
            w[j] = wj
        assert oracle.router_logit(x, w) == expect
        assert float(np.dot(x.astype(np.float64), w.astype(np.float64))) == exact


def test_router_logit_within_rounding_bound_of_exact():
    rng = np.random.default_rng(3)
    D = 2048
    gamma = (D // 32 + 5 + 2) * 2.0 ** -24      # fmaf chain of D/32 terms, then 5 tree levels
    for _ in range(200):
        x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rng.standard_normal(D).astype(np.float32)))
        w = (rng.standard_normal(D) / math.sqrt(D)).astype(np.float32)
        exact = float(np.dot(x.astype(np.float64), w.astype(np.float64)))
        bound = gamma * float(np.sum(np.abs(x.astype(np.float64) * w.astype(np.float64))))
        assert abs(oracle.router_logit(x, w) - exact) <= bound


def test_router_logit_uses_every_term():
    # a single nonzero product anywhere in the row comes through exactly
    for D in (256, 2048):
        for j in (0, 1, 7, 8, 255, D - 1, D // 2 + 3):
            x = np.zeros(D, np.float32)
            w = np.zeros(D, np.float32)
            x[j], w[j] = 1.5, -0.75
            assert oracle.router_logit(x, w) == np.float32(-1.125)


# ------------------------------------------------------------------ top-k and softmax
def test_topk_matches_full_stable_sort():
    rng = np.random.default_rng(4)
    for E, K in ((16, 2), (256, 8), (64, 64), (5, 1)):
        for _ in range(50):
            logits = rng.standard_normal(E).astype(np.float32)
            if rng.random() < 0.5:   # force ties
                logits = np.round(logits * 2) / 2
            order = np.lexsort((np.arange(E), -logits.astype(np.float64)))
            assert np.array_equal(oracle.topk(logits, K), order[:K])


def test_topk_ties_go_to_lower_index_and_nan_is_an_error():
    logits = np.zeros(16, np.float32)
    assert list(oracle.topk(logits, 4)) == [0, 1, 2, 3]
    logits[9] = logits[3] = 1.0
    assert list(oracle.topk(logits, 3)) == [3, 9, 0]
    logits[2] = np.nan
    with pytest.raises(RuntimeError):
        oracle.topk(logits, 3)


def test_softmax_over_kept_logits():
    rng = np.random.default_rng(5)
    for K in (1, 2, 8, 64):
        for _ in range(50):
            kept = np.sort(rng.standard_normal(K).astype(np.float32) * 3)[::-1].copy()
            w = oracle.softmax_kept(kept).astype(np.float64)
            k64 = kept.astype(np.float64)
            ref = np.exp(k64 - k64[0])
            ref /= ref.sum()
            # exp is within 1 ulp, S is a running sum of K terms, one rounded division
            assert np.all(np.abs(w - ref) <= (K + 4) * 2.0 ** -24 * ref)
            assert abs(w.sum() - 1.0) <= (K + 4) * 2.0 ** -24
            assert np.all(np.diff(w) <= 0)
    assert oracle.softmax_kept(np.array([0.3], np.float32))[0] == 1.0


# ------------------------------------------------------------------ permute
def test_permute_is_stable_counting_sort():
    rng = np.random.default_rng(6)
    for T, K, E in ((8, 2, 16), (64, 8, 256), (1, 8, 256), (300, 4, 9)):
        idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = oracle.permute(idx, E)
        flat = idx.ravel()
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        assert np.array_equal(perm, np.argsort(flat, kind="stable"))
        assert np.array_equal(inv[perm], np.arange(T * K))


# ------------------------------------------------------------------ the layer, stage by stage
@pytest.fixture(scope="module")
def tiny_layer():
    w = synth.layer_weights(TINY, seed=0)
    x = synth.activations(8, TINY.d_model, seed=0)
    L = oracle.Layer(TINY, w)
    return w, x, L, L.forward_tokens(x)


def test_layer_routing_matches_dense_float64(tiny_layer):
    w, x, L, out = tiny_layer
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = xf @ w["router_w"].astype(np.float64).T
    bound = (TINY.d_model // 32 + 8) * 2.0 ** -24 * (np.abs(xf) @ np.abs(w["router_w"].astype(np.float64)).T)
    assert np.all(np.abs(out["logits"] - ref) <= bound)
    for t in range(8):
        order = np.lexsort((np.arange(TINY.n_experts), -out["logits"][t].astype(np.float64)))
        assert np.array_equal(out["topk_idx"][t], order[:TINY.top_k])


def test_layer_accumulators_equal_int64_matmul(tiny_layer):
    w, x, L, out = tiny_layer
    for t in range(8):
        qx = out["q_x"][t].astype(np.int64)
        for k in range(TINY.top_k):
            e = out["topk_idx"][t, k]
            assert np.array_equal(out["acc_gate"][t, k], w["gate"][e].astype(np.int64) @ qx)
            assert np.array_equal(out["acc_up"][t, k], w["up"][e].astype(np.int64) @ qx)
            assert np.array_equal(out["acc_down"][t, k], w["down"][e].astype(np.int64) @ out["q_h"][t, k].astype(np.int64))


def test_layer_swiglu_and_output_match_float64(tiny_layer):
    w, x, L, out = tiny_layer
    for t in range(8):
        s_x = float(out["s_x"][t])
        y64 = np.zeros(TINY.d_model)
        for k in range(TINY.top_k):
            e = out["topk_idx"][t, k]
            g = out["acc_gate"][t, k] * (w["alpha_gate"][e].astype(np.float64) * s_x)
            u = out["acc_up"][t, k] * (w["alpha_up"][e].astype(np.float64) * s_x)
            h64 = g / (1.0 + np.exp(-g)) * u
            h = out["h"][t, k].astype(np.float64)
            assert np.all(np.abs(h - h64) <= 8 * 2.0 ** -24 * np.abs(h64) + 1e-30)
            qh, sh = out["q_h"][t, k], float(out["s_h"][t, k])
            amax = np.max(np.abs(h))
            assert abs(sh - amax / 127) <= 1e-7 * amax
            assert np.all(np.abs(qh - h * 127 / amax) <= 0.5 + 1e-4)
            ye = out["acc_down"][t, k] * (w["alpha_down"][e].astype(np.float64) * sh)
            assert np.all(np.abs(out["y_e"][t, k] - ye) <= 3 * 2.0 ** -24 * np.abs(ye))
            y64 += float(out["topk_w"][t, k]) * ye
        assert np.max(np.abs(out["y"][t] - y64)) <= 1e-6 * np.max(np.abs(y64))


def test_layer_dequantised_output_tracks_float64_layer(tiny_layer):
    """Without any int8 step the layer is y = sum_k w_k * Wd (silu(Wg x) * Wu x);
    the int8 path must stay within its quantisation error of it."""
    w, x, L, out = tiny_layer
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    for t in range(8):
        y = np.zeros(TINY.d_model)
        for k in range(TINY.top_k):
            e = out["topk_idx"][t, k]
            g = (w["alpha_gate"][e][:, None] * w["gate"][e]) @ xf[t]
            u = (w["alpha_up"][e][:, None] * w["up"][e]) @ xf[t]
            h = g / (1 + np.exp(-g)) * u
            y += out["topk_w"][t, k] * ((w["alpha_down"][e][:, None] * w["down"][e]) @ h)
        rel = np.max(np.abs(out["y"][t] - y)) / np.max(np.abs(y))
        assert rel < 0.05


def test_layer_invariants():
    w = synth.layer_weights(TINY, seed=7)
    x = synth.activations(8, TINY.d_model, seed=7)
    base = oracle.Layer(TINY, w).forward_tokens(x)
    # zero x row -> zero output
    x0 = x.copy()
    x0[3] = 0
    y0 = oracle.Layer(TINY, w).forward_tokens(x0, taps=False)["y"]
    assert not y0[3].any() and np.array_equal(y0[[0, 1, 2, 4, 5, 6, 7]], base["y"][[0, 1, 2, 4, 5, 6, 7]])
    # all-zero up (or down) rows -> zero output
    for key in ("up", "down"):
        wz = dict(w)
        wz[key] = np.zeros_like(w[key])
        assert not oracle.Layer(TINY, wz).forward_tokens(x, taps=False)["y"].any()
    # scaling alpha_down by 2^k scales y by 2^k exactly
    w2 = dict(w)
    w2["alpha_down"] = w["alpha_down"] * np.float32(4.0)
    assert np.array_equal(oracle.Layer(TINY, w2).forward_tokens(x, taps=False)["y"], base["y"] * 4)
    # a non-power-of-two alpha_down scale agrees to rounding
    w3 = dict(w)
    w3["alpha_down"] = (w["alpha_down"] * np.float32(3.0)).astype(np.float32)
    y3 = oracle.Layer(TINY, w3).forward_tokens(x, taps=False)["y"]
    assert np.max(np.abs(y3 - 3 * base["y"])) <= 1e-6 * np.max(np.abs(base["y"])) * 3
    # permuting tokens permutes outputs
    p = np.array([5, 2, 7, 0, 1, 6, 3, 4])
    assert np.array_equal(oracle.Layer(TINY, w).forward_tokens(x[p], taps=False)["y"], base["y"][p])
    # relabelling experts together with their router rows relabels the choices, y unchanged
    rl = np.random.default_rng(8).permutation(TINY.n_experts)      # new expert n = old expert rl[n]
    wr = {k: (v[rl] if v is not None else None) for k, v in w.items()}
    out_r = oracle.Layer(TINY, wr).forward_tokens(x)
    assert np.array_equal(rl[out_r["topk_idx"]], base["topk_idx"])
    assert np.array_equal(out_r["y"], base["y"])


def test_layer_top1_is_a_single_dense_swiglu_ffn():
    shape = synth.LayerShape(256, 4, 1, 32)
    w = synth.layer_weights(shape, seed=9)
    x = synth.activations(4, 256, seed=9)
    out = oracle.Layer(shape, w).forward_tokens(x)
    assert np.all(out["topk_w"] == 1.0)
    assert np.array_equal(out["y"], out["y_e"][:, 0])


def test_closed_form_layer():
    """A layer whose every value is worked out by hand.

    D=256, 2 experts, top-1, F=16.  x = 1.0 everywhere -> q_x = 127, s_x = 1/127.
    Router row 0 is +1/256, row 1 is -1/256 -> logits +1, -1; expert 0 wins, w = 1.
    Gate row r of expert 0 has +1 in its first 16*(r+1) positions, up rows are all
    +1, alpha = 2^-10: g_r = 127*16(r+1) * (2^-10 / 127) = (r+1)/64 (to rounding),
    u = 127*256 * 2^-10/127 = 1/4.  h_r = silu(g_r) * u.  Down row c has +1 at
    position c % 16 only, alpha_down = 1 -> y_c = q_h[c%16] * s_h ~ h_{c%16}.
    """
    D, E, K, F = 256, 2, 1, 16
    shape = synth.LayerShape(D, E, K, F)
    gate = np.zeros((E, F, D), np.int8)
    for r in range(F):
        gate[0, r, :16 * (r + 1)] = 1
    up = np.ones((E, F, D), np.int8)
    down = np.zeros((E, D, F), np.int8)
    for c in range(D):
        down[0, c, c % 16] = 1
    w = dict(gate=gate, up=up, down=down,
             alpha_gate=np.full((E, F), 2.0 ** -10, np.float32), alpha_up=np.full((E, F), 2.0 ** -10, np.float32),
             alpha_down=np.ones((E, D), np.float32),
             router_w=np.stack([np.full(D, 1 / 256), np.full(D, -1 / 256)]).astype(np.float32), router_bias=None)
    x = synth.f32_to_bf16_bits(np.ones((1, D), np.float32))
    out = oracle.Layer(shape, w).forward_tokens(x)
    assert out["logits"][0, 0] == 1.0 and out["logits"][0, 1] == -1.0
    assert out["topk_idx"][0, 0] == 0 and out["topk_w"][0, 0] == 1.0
    assert np.all(out["q_x"] == 127)
    assert np.array_equal(out["acc_gate"][0, 0], 127 * 16 * np.arange(1, F + 1))
    assert np.all(out["acc_up"][0, 0] == 127 * 256)
    g = np.arange(1, F + 1) / 64.0
    h = g / (1 + np.exp(-g)) * 0.25
    assert np.allclose(out["h"][0, 0], h, rtol=1e-6, atol=0)
    # int8 requantisation of h: each value moves by at most half a step amax/127
    assert np.all(np.abs(out["y"][0] - h[np.arange(D) % 16]) <= 0.5 * h.max() / 127 * (1 + 1e-5))
    assert np.array_equal(out["q_h"][0, 0], np.rint(h / h.max() * 127).astype(np.int8))


# ------------------------------------------------------------------ stack glue
def test_rmsnorm_matches_float64():
    rng = np.random.default_rng(10)
    r = rng.standard_normal((16, 2048)).astype(np.float32) * 3
    got = synth.bf16_bits_to_f32(oracle.rmsnorm_bf16(r)).astype(np.float64)
    r64 = r.astype(np.float64)
    ref = r64 / np.sqrt(np.mean(r64 * r64, axis=1, keepdims=True) + 1e-6)
    # bf16 keeps 8 significant bits: rounding moves a value by at most 2^-8 relative, plus the float rms
    assert np.all(np.abs(got - ref) <= (2.0 ** -8 + 2.0 ** -20) * np.abs(ref))


def test_stack_of_zero_layers_is_identity_and_composes():
    w = synth.layer_weights(TINY, seed=11)
    wz = dict(w)
    wz["down"] = np.zeros_like(w["down"])
    r = synth.residual(4, TINY.d_model, seed=11)
    Lz = oracle.Layer(TINY, wz)
    assert np.array_equal(oracle.stack_forward([Lz, Lz], r), r)
    # two real layers equal norm -> layer -> add, twice
    L1, L2 = oracle.Layer(TINY, w), oracle.Layer(TINY, synth.layer_weights(TINY, seed=12))
    got = oracle.stack_forward([L1, L2], r)
    ref = r.copy()
    for L in (L1, L2):
        ref = (ref + L.forward_tokens(oracle.rmsnorm_bf16(ref), taps=False)["y"]).astype(np.float32)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ shapes against the model table
def test_shapes_consistent_with_model_table():
    table = {}
    for line in open(os.path.join(GOLDEN, "model_table.txt")):
        if line.startswith("#") or "=" not in line:
            continue
        k, v = line.split("=")
        table[k.strip()] = float(v)
    big = synth.CONFIGS["decode"]["shape"]
    assert big.n_experts == table["experts"] and big.top_k == table["top_k"]
    assert synth.CONFIGS["stack"]["layers"] == table["layers"]
    expert_params = 3 * big.d_model * big.d_ff
    total = table["layers"] * big.n_experts * expert_params
    assert total <= table["total_params_billion"] * 1e9                       # FFN experts are most of the model
    assert total * table["bits_per_weight"] / 8 <= table["checkpoint_gb"] * 1e9
    assert table["layers"] * big.top_k * expert_params <= table["active_params_billion"] * 1e9
