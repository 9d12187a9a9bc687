"""Pins of the CPU oracle to what the pages and mathematics fix (no GPU).

Each test checks the oracle against something other than itself: values the
pages print for the worked example, closed forms, brute force on tiny inputs,
invariants the pages state, or a library routine for a textbook function.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _z(T, E, seed=7, stream=mi.STREAM_TEST_ROWS, std=1.0):
    return mi.normal_f64(T * E, seed, stream).reshape(T, E) * std


# ---------------------------------------------------------------------------
# §02c worked example (printed values)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("case", ["no_bias", "with_bias"])
def test_worked_example(case):
    g = _golden("worked_example_routing.json")
    z = np.array([g["z"]])
    c = g[case]
    r = oracle.route(z, np.array(c["bias"], np.float32), g["k"], g["n_routed"], g["n_shared"])
    np.testing.assert_allclose(r["s"][0], g["s_3dp"], atol=5e-4 + 1e-12)
    assert list(r["topk_idx"][0] + 1) == c["selected_1based"]
    np.testing.assert_allclose(r["gates"][0], c["gates_3dp"], atol=1e-3)
    if "selection_scores_3dp" in c:
        for v, want in zip(r["sel"][0], c["selection_scores_3dp"]):
            if want is not None:
                assert v == pytest.approx(want, abs=5e-4 + 1e-7)


def test_worked_example_exact_gates():
    """The exact gates behind the page's rounded 0.504 and 0.501."""
    g = _golden("worked_example_routing.json")
    s = [1 / (1 + math.exp(-v)) for v in g["z"]]
    r = oracle.route(np.array([g["z"]]), np.zeros(4, np.float32), 2, 4, 0)
    assert r["gates"][0][0] == pytest.approx(s[0] / (s[0] + s[1]), abs=1e-15)
    assert r["gates"][0][0] == pytest.approx(0.50479, abs=1e-5)


# ---------------------------------------------------------------------------
# sigmoid closed forms
# ---------------------------------------------------------------------------
def test_sigmoid_closed_forms():
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    assert oracle.sigmoid(np.array([math.log(3.0)]))[0] == pytest.approx(0.75, abs=1e-15)
    z = np.linspace(-20, 20, 101)
    np.testing.assert_allclose(oracle.sigmoid(z) + oracle.sigmoid(-z), 1.0, atol=1e-15)


# ---------------------------------------------------------------------------
# top-k: brute force over all subsets, tie rule, shared experts never candidates
# ---------------------------------------------------------------------------
def test_topk_bruteforce_all_subsets():
    """8 routed experts, top-3 (the size of the §02f widget): the kept set is
    the subset with the largest total selection score, for every token."""
    E, k, T = 8, 3, 200
    z = _z(T, E + 2, seed=3)
    b = mi.uniform_f32(E, 3, mi.STREAM_B, -0.1, 0.1)
    r = oracle.route(z, b, k, E, 2)
    sel = 1 / (1 + np.exp(-z[:, :E])) + b.astype(np.float64)
    subsets = list(itertools.combinations(range(E), k))
    for t in range(T):
        best = max(subsets, key=lambda S: sum(sel[t, i] for i in S))
        assert set(r["topk_idx"][t]) == set(best)
        # order: descending selection score
        assert all(sel[t, r["topk_idx"][t][j]] >= sel[t, r["topk_idx"][t][j + 1]] for j in range(k - 1))


def test_topk_against_repeated_argmax():
    """256 routed, top-6 against an independent selection: k rounds of
    'largest remaining score, lowest index among equals'."""
    E, k, T = 256, 6, 64
    z = _z(T, E + 2, seed=5)
    b = mi.uniform_f32(E, 5, mi.STREAM_B, -0.05, 0.05)
    r = oracle.route(z, b, k, E, 2)
    for t in range(T):
        sel = [1 / (1 + math.exp(-z[t, i])) + float(b[i]) for i in range(E)]
        chosen = []
        for _ in range(k):
            best = None
            for i in range(E):
                if i in chosen:
                    continue
                if best is None or sel[i] > sel[best]:
                    best = i
            chosen.append(best)
        assert list(r["topk_idx"][t]) == chosen


def test_topk_ties_go_to_lower_index():
    z = np.zeros((1, 10))
    z[0, [1, 4, 6, 7]] = 1.0   # four equal scores, keep 3
    r = oracle.route(z, np.zeros(8, np.float32), 3, 8, 2)
    assert list(r["topk_idx"][0]) == [1, 4, 6]
    assert r["margin"][0] == 0.0


def test_shared_experts_are_never_candidates():
    T, E = 32, 16
    z = _z(T, E + 2, seed=11)
    z[:, E:] = 30.0  # shared experts score far above everything
    r = oracle.route(z, np.zeros(E, np.float32), 4, E, 2)
    assert (r["topk_idx"] < E).all()
    assert (r["gates"][:, 4:] > r["gates"][:, :4].max(axis=1, keepdims=True)).all()


# ---------------------------------------------------------------------------
# joint normalisation
# ---------------------------------------------------------------------------
def test_gates_sum_to_one():
    z = _z(500, 258, seed=13)
    b = mi.uniform_f32(256, 13, mi.STREAM_B, -0.1, 0.1)
    r = oracle.route(z, b, 6, 256, 2)
    np.testing.assert_allclose(r["gates"].sum(axis=1), 1.0, atol=1e-12)
    assert r["gates"].shape == (500, 8)


def test_gates_closed_form_when_all_selected():
    """k = n_routed, no shared experts: g = s / sum(s) over all experts."""
    E = 16
    z = _z(40, E, seed=17)
    r = oracle.route(z, np.zeros(E, np.float32), E, E, 0)
    s = 1 / (1 + np.exp(-z))
    g_sorted = np.take_along_axis(s / s.sum(axis=1, keepdims=True), r["topk_idx"].astype(np.int64), axis=1)
    np.testing.assert_allclose(r["gates"], g_sorted, rtol=1e-14)


def test_gates_include_shared_in_denominator():
    """k routed + 2 shared: each gate is s_i over the sum of the 8 contributors' s."""
    z = _z(50, 258, seed=19)
    r = oracle.route(z, np.zeros(256, np.float32), 6, 256, 2)
    s = 1 / (1 + np.exp(-z))
    for t in range(50):
        ids = list(r["topk_idx"][t]) + [256, 257]
        den = sum(s[t, i] for i in ids)
        np.testing.assert_allclose(r["gates"][t], [s[t, i] / den for i in ids], rtol=1e-14)


def test_bias_steers_selection_but_never_gates():
    """§02b / §02e: b appears in the top-6 and nowhere else."""
    T = 400
    z = _z(T, 258, seed=23)
    b0 = np.zeros(256, np.float32)
    b1 = mi.uniform_f32(256, 23, mi.STREAM_B, -0.05, 0.05)
    r0 = oracle.route(z, b0, 6, 256, 2)
    r1 = oracle.route(z, b1, 6, 256, 2)
    same = np.array([set(a) == set(c) for a, c in zip(r0["topk_idx"], r1["topk_idx"])])
    assert (~same).any() and same.any()
    s = 1 / (1 + np.exp(-z))
    for t in range(T):
        if same[t]:
            # same set: identical gate per expert id, bit for bit
            g0 = dict(zip(r0["contrib"][t], r0["gates"][t]))
            g1 = dict(zip(r1["contrib"][t], r1["gates"][t]))
            assert g0 == g1
        else:
            ids = r1["contrib"][t]
            np.testing.assert_allclose(r1["gates"][t], s[t, ids] / s[t, ids].sum(), rtol=1e-14)


# ---------------------------------------------------------------------------
# loads and the bias controller (§02e)
# ---------------------------------------------------------------------------
def test_load_counts_bruteforce():
    idx = (mi.words(300 * 6, 1, mi.STREAM_TEST_TOPK) % 256).reshape(300, 6)
    c = oracle.load_counts(idx, 256)
    for e in range(256):
        assert c[e] == sum(1 for t in range(300) for j in range(6) if idx[t, j] == e)


def test_bias_update_closed_forms():
    T, k, n = 256, 6, 256          # Lbar = 6 exactly
    b = np.full(n, 0.25, np.float32)
    counts = np.full(n, 6, np.int32)
    counts[0], counts[1] = 7, 5
    nb = oracle.bias_update(counts, b, T, k, 0.01)
    assert nb[0] == np.float32(np.float32(0.25) - np.float32(0.01))    # overloaded: lowered
    assert nb[1] == np.float32(np.float32(0.25) + np.float32(0.01))    # underloaded: raised
    assert (nb[2:] == np.float32(0.25)).all()                          # sign(0) = 0
    # non-integer Lbar: T=100, k=6 -> Lbar = 600/256 = 2.34375
    c2 = np.array([2, 3] + [0] * 254, np.int32)
    nb2 = oracle.bias_update(c2, np.zeros(256, np.float32), 100, 6, 1e-3)
    assert nb2[0] == np.float32(1e-3) and nb2[1] == np.float32(-1e-3)


def test_bias_accumulates_as_the_page_says():
    g = _golden("bias_accumulation.json")
    b = np.zeros(256, np.float32)
    counts = np.zeros(256, np.int32)
    counts[0] = 100  # expert 0 far above the mean load every batch
    for _ in range(g["batches"]):
        b = oracle.bias_update(counts, b, T=10, k=6, gamma=g["gamma"])
    assert b[0] == pytest.approx(g["expected_bias"], abs=1e-6)


# ---------------------------------------------------------------------------
# dispatch (grouping by expert, stable by token)
# ---------------------------------------------------------------------------
def _random_topk(T, k, E, seed):
    w = mi.words(T * E, seed, mi.STREAM_TEST_TOPK).reshape(T, E)
    return np.argsort(w, axis=1, kind="stable")[:, :k].astype(np.int32)


def test_dispatch_bruteforce():
    T, k, E = 37, 3, 8
    idx = _random_topk(T, k, E, 2)
    dp = oracle.dispatch(idx, E)
    for e in range(E):
        expected = [t for t in range(T) if e in idx[t]]
        assert list(dp["row_token"][dp["offsets"][e]:dp["offsets"][e + 1]]) == expected
    for t in range(T):
        for j in range(k):
            r = dp["token_row"][t, j]
            assert dp["row_token"][r] == t
            assert dp["offsets"][idx[t, j]] <= r < dp["offsets"][idx[t, j] + 1]


# ---------------------------------------------------------------------------
# expert MLP and GELU
# ---------------------------------------------------------------------------
def test_gelu_tanh_against_torch_and_identities():
    import torch

    u = np.linspace(-8, 8, 2001)
    ref = torch.nn.functional.gelu(torch.from_numpy(u), approximate="tanh").numpy()
    np.testing.assert_allclose(oracle.gelu_tanh(u), ref, rtol=1e-13, atol=1e-15)
    assert oracle.gelu_tanh(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(oracle.gelu_tanh(u) - oracle.gelu_tanh(-u), u, atol=1e-13)


def _perm_matrix(rows, cols, seed):
    """rows x cols 0/1 matrix with one 1 per row, at a seeded column."""
    w = mi.words(rows, seed, mi.STREAM_TEST_ROWS)
    col = (w % cols).astype(np.int64)
    m = np.zeros((rows, cols))
    m[np.arange(rows), col] = 1.0
    return m, col


def test_expert_with_selection_matrices():
    """W1 and W2 picking one input each: y[i] = c * gelu(a * x[p(q(i))]).
    Catches a transposed or swapped operand (d != d_ff)."""
    d, f, n = 64, 48, 5
    x = mi.normal_bf16(n * d, 4, mi.STREAM_X).reshape(n, d)
    P, p = _perm_matrix(f, d, 31)     # W1 [f, d]: h_j uses x[p(j)]
    Q, q = _perm_matrix(d, f, 32)     # W2 [d, f]: y_i uses h[q(i)]
    a, c = 2.0, 0.5
    w1 = mi.f32_to_bf16_bits((a * P).astype(np.float32))
    w2 = mi.f32_to_bf16_bits((c * Q).astype(np.float32))
    y = oracle.expert(x, w1, w2)
    xf = mi.bf16_to_f64(x)
    expect = c * oracle.gelu_tanh(a * xf[:, p[q]])
    np.testing.assert_allclose(y, expect, rtol=1e-15, atol=0)


def test_expert_zero_and_scaling():
    d, f, n = 32, 32, 4
    x = mi.normal_bf16(n * d, 9, mi.STREAM_X).reshape(n, d)
    w1 = mi.normal_bf16(f * d, 9, mi.STREAM_W1, std=0.2).reshape(f, d)
    w2 = mi.normal_bf16(d * f, 9, mi.STREAM_W2, std=0.2).reshape(d, f)
    assert (oracle.expert(x, w1, np.zeros_like(w2)) == 0).all()
    y = oracle.expert(x, w1, w2)
    w2x2 = mi.f32_to_bf16_bits(2 * mi.bf16_to_f64(w2).astype(np.float32))
    np.testing.assert_array_equal(oracle.expert(x, w1, w2x2), 2 * y)   # exact in fp64


def test_expert_identity_is_gelu():
    d = 64
    x = mi.normal_bf16(3 * d, 10, mi.STREAM_X).reshape(3, d)
    eye = mi.f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    np.testing.assert_allclose(oracle.expert(x, eye, eye), oracle.gelu_tanh(mi.bf16_to_f64(x)), rtol=1e-15)


# ---------------------------------------------------------------------------
# combine and the whole layer
# ---------------------------------------------------------------------------
def test_combine_one_hot_and_identical_rows():
    T, k, d = 20, 3, 16
    idx = _random_topk(T, k, 8, 4)
    dp = oracle.dispatch(idx, 8)
    y = mi.normal_f64(T * k * d, 4, mi.STREAM_TEST_ROWS).reshape(T * k, d)
    ysh = mi.normal_f64(2 * T * d, 4, mi.STREAM_TEST_SHARED).reshape(2, T, d)
    g = np.zeros((T, k + 2))
    g[:, 1] = 1.0
    np.testing.assert_array_equal(oracle.combine(y, dp["token_row"], g, ysh), y[dp["token_row"][:, 1]])
    g = np.zeros((T, k + 2))
    g[:, k + 1] = 1.0
    np.testing.assert_array_equal(oracle.combine(y, dp["token_row"], g, ysh), ysh[1])
    # identical contributor outputs and gates summing to one reproduce that output
    same = np.tile(y[:1], (T * k, 1))
    g = np.abs(mi.normal_f64(T * (k + 2), 5, mi.STREAM_TEST_GATES).reshape(T, k + 2))
    g /= g.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(oracle.combine(same, dp["token_row"], g, np.tile(y[:1], (2, T, 1))),
                               np.tile(y[:1], (T, 1)), rtol=1e-14)


def test_layer_with_identical_experts_is_that_expert():
    """All 258 experts equal: the output is that expert applied to x, whatever
    the routing (the gates of the 8 contributors sum to one)."""
    w = mi.WORKLOADS["tiny"]
    w1 = mi.host_w1(w, 0)
    w2 = mi.host_w2(w, 0)
    weights = {"w1": np.broadcast_to(w1, (w.n_experts,) + w1.shape),
               "w2": np.broadcast_to(w2, (w.n_experts,) + w2.shape)}
    tokens = np.arange(0, w.T, 17)
    r = oracle.forward_tokens(w, tokens, mi.host_bias(w), weights=weights)
    ref = oracle.expert(mi.host_x(w, tokens), w1, w2)
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-14)


def test_layer_is_the_gate_weighted_sum_of_eight_experts():
    """Zeroing every expert but one leaves exactly that expert's gated share:
    each token's output is g_e * E_e(x) for the one surviving expert e."""
    w = mi.WORKLOADS["tiny"]
    w1 = mi.host_w1_all(w)
    w2 = mi.host_w2_all(w).copy()
    keep = 256  # first shared expert, which every token uses
    w2_only = np.zeros_like(w2)
    w2_only[keep] = w2[keep]
    tokens = np.arange(10)
    r = oracle.forward_tokens(w, tokens, mi.host_bias(w), weights={"w1": w1, "w2": w2_only})
    y = oracle.expert(mi.host_x(w, tokens), w1[keep], w2[keep])
    np.testing.assert_allclose(r["out"], r["gates"][:, w.k:w.k + 1] * y, rtol=1e-14)


def test_sampled_tokens_match_full_batch():
    """Tokens are independent: routing a subset gives the same answer per token."""
    w = mi.WORKLOADS["tiny"]
    b = mi.host_bias(w)
    full = oracle.route_workload(w, b)
    sub = np.array([0, 5, 77, 255])
    part = oracle.route_workload(w, b, tokens=sub)
    np.testing.assert_array_equal(full["topk_idx"][sub], part["topk_idx"])
    np.testing.assert_array_equal(full["gates"][sub], part["gates"])


@pytest.mark.slow
def test_skew_offset_calibration():
    """The stored beta gives the skewed workload ~30% of assignments on its top 8 experts."""
    w = mi.WORKLOADS["skew"]
    r = oracle.route_workload(w, np.zeros(256, np.float32), logit_offset=mi.host_logit_offset(w))
    c = np.sort(oracle.load_counts(r["topk_idx"], 256))[::-1]
    assert abs(c[:8].sum() / c.sum() - 0.30) <= 0.005


@pytest.mark.parametrize("T,d,E", [(1, 64, 258), (37, 256, 258), (5, 7168, 9), (300, 32, 64)])
def test_logits_against_numpy_matmul(T, d, E):
    """The router logits z = x W_r^T (§02b) against numpy's fp64 matrix product of the same
    exactly widened bf16 values; and a hand case with one-hot rows picks out W_r's columns."""
    x = mi.normal_bf16(T * d, 12, mi.STREAM_X).reshape(T, d)
    wr = mi.normal_bf16(E * d, 12, mi.STREAM_WR, std=d ** -0.5).reshape(E, d)
    z = oracle.logits(x, wr)
    ref = mi.bf16_to_f64(x) @ mi.bf16_to_f64(wr).T
    np.testing.assert_allclose(z, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    onehot = mi.f32_to_bf16_bits(np.eye(min(d, 8), d, dtype=np.float32))
    np.testing.assert_array_equal(oracle.logits(onehot, wr), mi.bf16_to_f64(wr)[:, :min(d, 8)].T)
