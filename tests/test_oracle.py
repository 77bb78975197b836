"""Pins for the CPU oracle (CPU only).

The oracle is checked against things other than itself: a scalar brute force that
decides selection by rank counting, a worked two-token example evaluated from its
closed form, textbook special cases (E=1 dense SwiGLU; C=T mixture of experts),
and invariants of expert-choice routing (exactly C tokens per expert, permutation
equivariance, unselected tokens give zero, linearity in the down projection).
"""

import math

import numpy as np
import pytest

from oracle import nmoe_oracle as O
from diffusion_transformer_moe_b200 import inputs as I
from tests._brute import brute_layer


def _small(T, d, E, F, seed=0, x_std=1.0):
    t = I.make_small(T, d, E, F, "f32", seed=seed, x_std=x_std)
    return {k: I.to_numpy_f64(v) for k, v in t.items()}


def _dense_ffn(x, W1, W3, W2):
    g = x @ W1
    return (g * (1.0 / (1.0 + np.exp(-g))) * (x @ W3)) @ W2


# -- brute force ------------------------------------------------------------------------

@pytest.mark.parametrize("case", [
    dict(T=24, d=8, E=4, F=6, C=5),
    dict(T=32, d=6, E=8, F=4, C=4, score_fn="sigmoid"),
    dict(T=30, d=5, E=3, F=7, C=9, combine="normalized", route_scale=2.5),
    dict(T=32, d=4, E=4, F=3, C=3, n_segments=2, bias=True),
    dict(T=16, d=4, E=2, F=3, C=16),
])
def test_oracle_matches_brute_force(case):
    c = dict(case)
    T, d, E, F, C = (c.pop(k) for k in ("T", "d", "E", "F", "C"))
    nseg = c.pop("n_segments", 1)
    bias = None
    if c.pop("bias", False):
        bias = np.random.default_rng(3).normal(size=(nseg, E))
    a = _small(T, d, E, F, seed=11, x_std=2.0)
    ref = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C, n_segments=nseg,
                  router_bias=bias, **c)
    out, s32, chosen = brute_layer(a["x"].tolist(), a["W_r"].tolist(), a["W1"].tolist(),
                                   a["W3"].tolist(), a["W2"].tolist(), C,
                                   n_segments=nseg, router_bias=None if bias is None
                                   else bias.tolist(), **c)
    assert np.array_equal(np.asarray(s32, dtype=np.float32), ref["scores32"])
    for e in range(E):
        assert set(ref["idx"][e].tolist()) == chosen[e]
    np.testing.assert_allclose(ref["out"], np.asarray(out), rtol=1e-11, atol=1e-12)


# -- a worked example from its closed form -----------------------------------------------

def test_worked_two_token_example():
    """x0 = (1, 0), x1 = (0, 1); W_r = [[0, 0], [0, L]].

    Token 0 has logits (0, 0) -> p = (1/2, 1/2); token 1 has logits (0, L) ->
    p = (1/(1+e^L), e^L/(1+e^L)). With L > 0 and C = 1, expert 0 prefers token 0
    (1/2 > 1/(1+e^L)) and expert 1 prefers token 1. With F = 1 and expert weights
    W1_e = (a_e, b_e)^T, W3_e = (c_e, f_e)^T, W2_e = (u_e, v_e):
      out0 = 1/2 * silu(a_0) * c_0 * (u_0, v_0)
      out1 = e^L/(1+e^L) * silu(b_1) * f_1 * (u_1, v_1)
    """
    L = 0.7
    x = np.array([[1.0, 0.0], [0.0, 1.0]])
    W_r = np.array([[0.0, 0.0], [0.0, L]])
    W1 = np.array([[[0.3], [-1.2]], [[0.9], [1.5]]])     # (a_e, b_e)
    W3 = np.array([[[2.0], [0.4]], [[-0.6], [1.1]]])     # (c_e, f_e)
    W2 = np.array([[[1.0, -2.0]], [[0.5, 3.0]]])         # (u_e, v_e)
    r = O.layer(x, W_r, W1, W3, W2, C=1)
    silu = lambda g: g / (1.0 + math.exp(-g))
    p11 = math.exp(L) / (1.0 + math.exp(L))
    exp0 = 0.5 * silu(0.3) * 2.0 * np.array([1.0, -2.0])
    exp1 = p11 * silu(1.5) * 1.1 * np.array([0.5, 3.0])
    assert r["idx"].tolist() == [[0], [1]]
    np.testing.assert_allclose(r["out"][0], exp0, rtol=1e-14)
    np.testing.assert_allclose(r["out"][1], exp1, rtol=1e-14)
    # normalised combine: each token is chosen by one expert -> weight = route_scale
    rn = O.layer(x, W_r, W1, W3, W2, C=1, combine="normalized", route_scale=2.5)
    np.testing.assert_allclose(rn["out"][0], 2.5 * silu(0.3) * 2.0 * np.array([1.0, -2.0]),
                               rtol=1e-14)


def test_tie_break_prefers_lower_token():
    """L = 0: every score is exactly 1/2. Both experts take token 0 (lower index);
    token 1 is chosen by nobody and outputs exactly zero; with C = 2 both are taken."""
    x = np.array([[1.0, 0.0], [0.0, 1.0]])
    W_r = np.zeros((2, 2))
    W1 = np.ones((2, 2, 1)); W3 = np.ones((2, 2, 1)); W2 = np.ones((2, 1, 2))
    r = O.layer(x, W_r, W1, W3, W2, C=1)
    assert r["idx"].tolist() == [[0], [0]]
    assert np.all(r["out"][1] == 0.0)
    # token 0 gets both experts with weight 1/2 each: out0 = silu(1) * 1 * (1, 1)
    s = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(r["out"][0], [s, s], rtol=1e-14)
    assert O.layer(x, W_r, W1, W3, W2, C=2)["idx"].tolist() == [[0, 1], [0, 1]]


def test_select_orders_by_score_then_index():
    s = np.array([[0.5, 0.1], [0.7, 0.1], [0.5, 0.3], [0.2, 0.3]], dtype=np.float32)
    # expert 0: 0.7(t1) > 0.5(t0) = 0.5(t2) > 0.2 -> top-2 = {1, 0}; expert 1: t2, t3
    assert O.select(s, 2).tolist() == [[0, 1], [2, 3]]
    assert O.select(s, 3).tolist() == [[0, 1, 2], [0, 2, 3]]
    # per segment: two groups of two tokens, C = 1
    assert O.select(s, 1, n_segments=2).tolist() == [[1, 2], [0, 2]]


# -- special cases with textbook answers ------------------------------------------------

def test_single_expert_full_capacity_is_dense_swiglu():
    a = _small(40, 12, 1, 9, seed=5)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=40)
    assert np.all(r["p"] == 1.0)
    np.testing.assert_allclose(r["out"], _dense_ffn(a["x"], a["W1"][0], a["W3"][0], a["W2"][0]),
                               rtol=1e-12, atol=1e-13)


def test_full_capacity_is_score_weighted_mixture():
    a = _small(24, 10, 5, 7, seed=6, x_std=1.5)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=24)
    l = a["x"] @ a["W_r"]
    p = np.exp(l - l.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    want = sum(p[:, e:e + 1] * _dense_ffn(a["x"], a["W1"][e], a["W3"][e], a["W2"][e])
               for e in range(5))
    np.testing.assert_allclose(r["out"], want, rtol=1e-11, atol=1e-12)


def test_identical_experts_full_capacity_is_one_ffn():
    a = _small(20, 8, 4, 6, seed=7)
    W1 = np.repeat(a["W1"][:1], 4, 0); W3 = np.repeat(a["W3"][:1], 4, 0)
    W2 = np.repeat(a["W2"][:1], 4, 0)
    r = O.layer(a["x"], a["W_r"], W1, W3, W2, C=20)
    np.testing.assert_allclose(r["out"], _dense_ffn(a["x"], W1[0], W3[0], W2[0]),
                               rtol=1e-11, atol=1e-12)


# -- invariants --------------------------------------------------------------------------

def test_exactly_C_distinct_ascending_and_softmax_normalised():
    a = _small(64, 16, 8, 8, seed=8)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=10)
    assert r["idx"].shape == (8, 10)
    for e in range(8):
        row = r["idx"][e]
        assert len(set(row.tolist())) == 10 and np.all(np.diff(row) > 0)
        # nothing outside the chosen set beats the weakest chosen token
        s = r["scores32"][:, e]
        worst = min(row, key=lambda t: (s[t], -t))
        for t in set(range(64)) - set(row.tolist()):
            assert (s[t], -t) < (s[worst], -worst)
    np.testing.assert_allclose(r["p"].sum(1), 1.0, rtol=0, atol=1e-14)


def test_unselected_tokens_output_zero_and_selected_do_not():
    a = _small(64, 16, 4, 8, seed=9)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=4)
    chosen = set(r["idx"].ravel().tolist())
    for t in range(64):
        if t in chosen:
            assert np.any(r["out"][t] != 0.0)
        else:
            assert np.all(r["out"][t] == 0.0)


def test_permutation_equivariance():
    a = _small(48, 8, 6, 5, seed=10)
    perm = np.random.default_rng(0).permutation(48)
    r0 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=7)
    r1 = O.layer(a["x"][perm], a["W_r"], a["W1"], a["W3"], a["W2"], C=7)
    np.testing.assert_allclose(r1["out"], r0["out"][perm], rtol=1e-12, atol=1e-14)


def test_linear_in_down_projection():
    a = _small(32, 8, 4, 6, seed=12)
    r0 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=6)
    r1 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], -3.0 * a["W2"], C=6)
    np.testing.assert_allclose(r1["out"], -3.0 * r0["out"], rtol=1e-13, atol=1e-14)


def test_token_lists_invert_the_selection():
    a = _small(50, 8, 6, 4, seed=13)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=9)
    ptr, ent = O.token_lists(r["idx"], 50)
    assert ptr[-1] == 6 * 9 == len(ent)
    for t in range(50):
        es = ent[ptr[t]:ptr[t + 1]]
        assert np.all(np.diff(es // 9) > 0)  # strictly ascending experts
        for v in es:
            assert r["idx"][v // 9, v % 9] == t


def test_normalized_weights_sum_to_route_scale():
    a = _small(40, 8, 5, 4, seed=14)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=12, combine="normalized",
                route_scale=2.5)
    tot = np.zeros(40)
    for e in range(5):
        np.add.at(tot, r["idx"][e], r["w"][e])
    chosen = sorted(set(r["idx"].ravel().tolist()))
    np.testing.assert_allclose(tot[chosen], 2.5, rtol=1e-14)


def test_timestep_concat_router_is_a_segment_bias():
    rng = np.random.default_rng(1)
    T, d, dt, E, nseg = 12, 5, 3, 4, 3
    x = rng.normal(size=(T, d)); temb = rng.normal(size=(nseg, dt))
    Wg = rng.normal(size=(dt + d, E))
    lit = O.router_logits_concat(temb, x, Wg, nseg)
    bias = temb @ Wg[:dt]
    np.testing.assert_allclose(O.router_logits(x, Wg[dt:], bias, nseg), lit, rtol=1e-13,
                               atol=1e-14)


def test_separate_router_input_reproduces_the_pages_concat_gate():
    # Section 6.2: the gate reads cat([timestep, unmodulated hidden]) while the experts
    # transform the block's input. Built here from the page's literal gate, softmax,
    # each expert's top-C by (score, -token) found by sorting, and a per-token sum
    # of score-weighted dense SwiGLU outputs of the EXPERT input.
    rng = np.random.default_rng(21)
    T, d, dt, E, F, C, nseg = 16, 6, 3, 4, 5, 3, 2
    h = rng.normal(size=(T, d))              # unmodulated hidden states (router input)
    x = rng.normal(size=(T, d))              # the experts' input
    temb = rng.normal(size=(nseg, dt))
    Wg = rng.normal(size=(dt + d, E)) / np.sqrt(dt + d)
    W1 = rng.normal(size=(E, d, F)); W3 = rng.normal(size=(E, d, F))
    W2 = rng.normal(size=(E, F, d))
    lit = np.concatenate([np.repeat(temb, T // nseg, axis=0), h], axis=1) @ Wg
    z = np.exp(lit - lit.max(axis=1, keepdims=True))
    p = z / z.sum(axis=1, keepdims=True)
    p32 = p.astype(np.float32)
    want = np.zeros((T, d))
    chosen = np.zeros((E, T), dtype=bool)
    S = T // nseg
    for e in range(E):
        for g in range(nseg):
            seg = list(range(g * S, (g + 1) * S))
            for t in sorted(seg, key=lambda t: (-float(p32[t, e]), t))[:C]:
                chosen[e, t] = True
                want[t] += p[t, e] * _dense_ffn(x[t:t + 1], W1[e], W3[e], W2[e])[0]
    r = O.layer(x, Wg[dt:], W1, W3, W2, C, n_segments=nseg, router_bias=temb @ Wg[:dt],
                router_x=h)
    for e in range(E):
        assert sorted(r["idx"][e].tolist()) == np.flatnonzero(chosen[e]).tolist()
    np.testing.assert_allclose(r["out"], want, rtol=1e-11, atol=1e-12)
    # the router input decides the selection: scoring x instead changes it here
    r_x = O.layer(x, Wg[dt:], W1, W3, W2, C, n_segments=nseg, router_bias=temb @ Wg[:dt])
    assert not np.array_equal(np.sort(r_x["idx"], axis=1), np.sort(r["idx"], axis=1))
    # and router_x = x is the default layer, value for value
    r_same = O.layer(x, Wg[dt:], W1, W3, W2, C, n_segments=nseg, router_x=x)
    r_def = O.layer(x, Wg[dt:], W1, W3, W2, C, n_segments=nseg)
    assert np.array_equal(r_same["out"], r_def["out"])
    rows = O.layer_rows(x, Wg[dt:], W1, W3, W2, C, [0, 5, 11], n_segments=nseg,
                        router_bias=temb @ Wg[:dt], router_x=h)
    np.testing.assert_allclose(rows["out"], r["out"][[0, 5, 11]], rtol=1e-13, atol=1e-15)


def test_segments_are_independent_layers():
    # section 6.2 selects per sample: a layer over n_segments samples is n_segments
    # independent layers, one per sample, each with that sample's bias row
    a = _small(36, 6, 5, 4, seed=23)
    bias = np.random.default_rng(4).normal(size=(3, 5))
    whole = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=4, n_segments=3,
                    router_bias=bias, combine="normalized", route_scale=2.5)
    for g in range(3):
        part = O.layer(a["x"][12 * g:12 * (g + 1)], a["W_r"], a["W1"], a["W3"], a["W2"], C=4,
                       router_bias=bias[g:g + 1], combine="normalized", route_scale=2.5)
        np.testing.assert_array_equal(whole["out"][12 * g:12 * (g + 1)], part["out"])
        assert np.array_equal(whole["idx"][:, 4 * g:4 * (g + 1)], part["idx"] + 12 * g)


def test_sampled_rows_match_full_layer():
    a = _small(40, 8, 5, 6, seed=15)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=8, combine="normalized",
                route_scale=2.5)
    toks = [0, 3, 17, 39, 22]
    rr = O.layer_rows(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], 8, toks,
                      combine="normalized", route_scale=2.5)
    np.testing.assert_allclose(rr["out"], r["out"][toks], rtol=1e-13, atol=1e-15)


def test_shared_expert_adds_dense_ffn():
    a = _small(20, 6, 3, 4, seed=16)
    sh = (a["W1"][0], a["W3"][0], a["W2"][0])
    r0 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=5)
    r1 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=5, shared=sh)
    np.testing.assert_allclose(r1["out"] - r0["out"], _dense_ffn(a["x"], *sh), rtol=1e-12,
                               atol=1e-13)


# -- the block's gated residual (section 6.3) ----------------------------------------------

def _tanh(a):
    """tanh from its exponential definition (not numpy's tanh)."""
    import math
    return (math.exp(2 * a) - 1.0) / (math.exp(2 * a) + 1.0)


def test_gated_residual_with_a_zero_gate_is_the_residual():
    a = _small(16, 6, 3, 4, seed=30)
    res = np.random.default_rng(1).standard_normal((16, 6))
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=5, residual=res,
                gate2=np.zeros((1, 6)))
    assert np.array_equal(r["out"], res)


def test_gated_residual_clamps_to_two_then_takes_tanh():
    a = _small(16, 6, 3, 4, seed=31)
    res = np.random.default_rng(2).standard_normal((16, 6))
    gate = np.array([[-5.0, -2.0, -0.5, 0.5, 2.0, 7.0]])
    r0 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=5)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=5, residual=res, gate2=gate)
    factor = np.array([_tanh(-2.0), _tanh(-2.0), _tanh(-0.5), _tanh(0.5), _tanh(2.0),
                       _tanh(2.0)])
    np.testing.assert_allclose(r["out"], res + factor * r0["out"], rtol=1e-14, atol=1e-15)
    assert abs(factor[-1] - 0.9640275800758169) < 1e-15  # tanh(2), not tanh(7)


def test_gated_residual_takes_each_segments_gate_row():
    a = _small(24, 4, 3, 4, seed=32)
    res = np.zeros((24, 4))
    gate = np.array([[0.3, 0.3, 0.3, 0.3], [-1.0, -1.0, -1.0, -1.0], [1.5, 1.5, 1.5, 1.5]])
    r0 = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=3, n_segments=3)
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=3, n_segments=3,
                residual=res, gate2=gate)
    for seg, gval in enumerate((0.3, -1.0, 1.5)):
        rows = slice(8 * seg, 8 * seg + 8)
        np.testing.assert_allclose(r["out"][rows], _tanh(gval) * r0["out"][rows],
                                   rtol=1e-14, atol=1e-15)


def test_gated_residual_wraps_shared_plus_routed_and_rows_agree():
    a = _small(20, 6, 3, 4, seed=33)
    sh = (a["W1"][1], a["W3"][1], a["W2"][1])
    res = np.random.default_rng(3).standard_normal((20, 6))
    gate = np.random.default_rng(4).standard_normal((2, 6))
    routed = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=4, n_segments=2)["out"]
    r = O.layer(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], C=4, n_segments=2, shared=sh,
                residual=res, gate2=gate)
    g = np.array([[_tanh(min(2.0, max(-2.0, v))) for v in row] for row in gate])
    want = res + g[np.arange(20) // 10] * (_dense_ffn(a["x"], *sh) + routed)
    np.testing.assert_allclose(r["out"], want, rtol=1e-12, atol=1e-13)
    toks = [0, 7, 10, 19]
    rr = O.layer_rows(a["x"], a["W_r"], a["W1"], a["W3"], a["W2"], 4, toks, n_segments=2,
                      shared=sh, residual=res, gate2=gate)
    np.testing.assert_allclose(rr["out"], r["out"][toks], rtol=1e-13, atol=1e-14)


# -- the skewed workload has what it promises ---------------------------------------------

@pytest.mark.slow
def test_skewed_workload_has_unselected_tokens_and_threshold_ties():
    w = I.WORKLOADS["skewed_2048px"]
    a = I.make_inputs(w, parts=("x", "W_r"))
    x = I.to_numpy_f64(a["x"]); W_r = I.to_numpy_f64(a["W_r"])
    s32 = O.round_f32(O.scores_from_logits(O.router_logits(x, W_r)))
    idx = O.select(s32, w.C)
    assert len(set(idx.ravel().tolist())) < w.T  # some tokens are chosen by nobody
    tie_at_threshold = 0
    for e in range(w.E):
        col = s32[:, e]
        thr = col[idx[e]].min()
        n_eq = int(np.sum(col == thr))
        n_eq_in = int(np.sum(col[idx[e]] == thr))
        if n_eq > n_eq_in:  # equal scores on both sides of the cut
            tie_at_threshold += 1
    assert tie_at_threshold >= 1
