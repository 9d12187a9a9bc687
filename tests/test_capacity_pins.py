"""Pins of the oracle's expert capacity, drop accounting and Router Balance Lab
loop ("Inkling, Dissected" §02d "The rich-get-richer problem", §02g "the Router
Balance Lab") to a hand-worked example, the counting definition, closed forms
and the lab results the page reports (no GPU)."""
import json
import os

import numpy as np
import pytest

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _distinct_topk(T, k, E, seed):
    """Random top-k rows with k distinct experts each (seeded, from the generator's words)."""
    u = mi.words(T * E, seed, mi.STREAM_TEST_TOPK).reshape(T, E)
    return np.argsort(u, axis=1, kind="stable")[:, :k].astype(np.int32)


def test_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "capacity_example.json")))
    topk = np.array(g["topk_idx"], dtype=np.int32)
    keep = oracle.capacity_keep(topk, g["capacity"], g["n_routed"])
    assert keep.tolist() == g["keep"]
    L = oracle.load_counts(topk, g["n_routed"])
    assert L.tolist() == g["counts"]
    m = oracle.load_metrics(L, g["capacity"], len(topk), g["top_k"])
    assert m["dropped"] == g["dropped"]
    assert m["drop_rate"] == pytest.approx(g["drop_rate"], abs=1e-15)
    assert m["max_vio"] == pytest.approx(g["max_vio"], abs=1e-12)


@pytest.mark.parametrize("T,k,E,cap", [(300, 6, 16, 100), (513, 3, 8, 150), (64, 8, 64, 7), (257, 1, 4, 30)])
def test_keep_is_counting_definition(T, k, E, cap):
    """keep[t, j] <=> fewer than `cap` earlier tokens picked the same expert
    (counted with a cumulative one-hot sum, not a queue)."""
    topk = _distinct_topk(T, k, E, seed=T + E)
    onehot = np.zeros((T, E), dtype=np.int64)
    np.put_along_axis(onehot, topk.astype(np.int64), 1, axis=1)
    before = np.cumsum(onehot, axis=0) - onehot  # picks of each expert by tokens < t
    expect = np.take_along_axis(before, topk.astype(np.int64), axis=1) < cap
    assert np.array_equal(oracle.capacity_keep(topk, cap, E), expect)


def test_keep_invariants():
    T, k, E = 1000, 6, 32
    topk = _distinct_topk(T, k, E, seed=3)
    L = oracle.load_counts(topk, E)
    for cap in [0, 1, 50, 187, int(L.max()) - 1, int(L.max()), 10 ** 6]:
        keep = oracle.capacity_keep(topk, cap, E)
        served = np.bincount(topk[keep], minlength=E)
        assert np.array_equal(served, np.minimum(L, cap)), cap
        m = oracle.load_metrics(L, cap, T, k)
        assert m["dropped"] == int((~keep).sum())
    assert oracle.capacity_keep(topk, int(L.max()), E).all()
    assert not oracle.capacity_keep(topk, 0, E).any()


def test_dispatch_with_drops():
    """Only served pairs get rows: expert e has min(L_e, C) rows, its earliest
    tokens, in token order; dropped pairs point nowhere; with every pair served
    the layout is the uncapped dispatch."""
    g = json.load(open(os.path.join(GOLDEN, "capacity_example.json")))
    topk = np.array(g["topk_idx"], dtype=np.int32)
    keep = np.array(g["keep"])
    r = oracle.dispatch(topk, g["n_routed"], keep)
    assert r["offsets"].tolist() == [0, 2, 4, 6]
    assert r["row_token"].tolist() == [0, 1, 0, 1, 2, 3]
    assert r["token_row"].tolist() == [[0, 2], [3, 1], [-1, 4], [5, -1], [-1, -1]]
    T, k, E = 700, 6, 32
    topk = _distinct_topk(T, k, E, seed=11)
    full = oracle.dispatch(topk, E)
    same = oracle.dispatch(topk, E, np.ones((T, k), dtype=bool))
    for key in full:
        assert np.array_equal(full[key], same[key])
    cap = 100
    r = oracle.dispatch(topk, E, oracle.capacity_keep(topk, cap, E))
    L = oracle.load_counts(topk, E)
    assert np.array_equal(np.diff(r["offsets"]), np.minimum(L, cap))
    for e in range(E):
        rows = r["row_token"][r["offsets"][e]:r["offsets"][e + 1]]
        assert np.array_equal(rows, np.nonzero((topk == e).any(axis=1))[0][:cap])


def test_capacity_for():
    assert oracle.capacity_for(1.25, 2048, 6, 64) == 240      # lab: 1.25 x 192
    assert oracle.capacity_for(1.25, 65536, 6, 256) == 1920   # 1.25 x 1536
    assert oracle.capacity_for(1.25, 100, 6, 64) == 11        # 11.71875 rounds down
    assert oracle.capacity_for(1.0, 256, 6, 256) == 6         # exactly the ideal load
    assert oracle.capacity_for(1.1, 1000, 1, 10) == 110       # 1.1 read as 11/10, not its binary neighbour


def test_metrics_closed_forms():
    # perfectly balanced loads: no violation, nothing dropped at any capacity >= the ideal load
    T, k, E = 4096, 6, 256
    L = np.full(E, k * T // E, dtype=np.int32)
    m = oracle.load_metrics(L, k * T // E, T, k)
    assert m["max_vio"] == 0.0 and m["dropped"] == 0
    # every token on one expert (k = 1): MaxVio = E - 1, drop rate = (T - C) / T
    T, k, E, C = 1000, 1, 8, 150
    L = np.zeros(E, dtype=np.int32)
    L[3] = T
    m = oracle.load_metrics(L, C, T, k)
    assert m["max_vio"] == pytest.approx(E - 1, abs=1e-12)
    assert m["drop_rate"] == pytest.approx((T - C) / T, abs=1e-15)


def test_forward_with_drops_identical_experts():
    """All experts equal: out_t = (sum of the gates of the contributors actually
    served) * E(x_t); a token that loses a routed expert loses exactly its gate."""
    w = mi.WORKLOADS["tiny"]
    tokens = np.arange(0, 40)
    e1, e2 = mi.host_w1(w, 5), mi.host_w2(w, 5)
    weights = {"w1": np.broadcast_to(e1, (w.n_experts,) + e1.shape),
               "w2": np.broadcast_to(e2, (w.n_experts,) + e2.shape)}
    bias = mi.host_bias(w)
    keep = np.ones((len(tokens), w.k), dtype=bool)
    keep[::3, 0] = False
    keep[1::4, 2:5] = False
    keep[7] = False
    r = oracle.forward_tokens(w, tokens, bias, weights=weights, keep=keep)
    ex = oracle.expert(mi.host_x(w, tokens), e1, e2)
    served = np.where(keep, r["gates"][:, :w.k], 0.0).sum(axis=1) + r["gates"][:, w.k:].sum(axis=1)
    np.testing.assert_allclose(r["out"], served[:, None] * ex, rtol=1e-12, atol=1e-12)
    full = oracle.forward_tokens(w, tokens, bias, weights=weights)
    same = oracle.forward_tokens(w, tokens, bias, weights=weights, keep=np.ones_like(keep))
    assert np.array_equal(full["out"], same["out"])


@pytest.fixture(scope="module")
def lab_runs():
    return {g: oracle.lab_run(mi.LAB, g) for g in mi.LAB.gammas}


def test_lab_reproduces_page_findings(lab_runs):
    """§02g's three results, as shapes rather than digits (the lab's own code and
    token stream are not on the page): without balancing the hottest expert stays
    near twice its share and several percent of slots drop; gamma = 0.01 brings
    MaxVio to about a quarter with essentially no drops; gamma = 0.05 slips back
    to a few percent of drops, still fewer than no balancing."""
    late = slice(50, None)
    none, good, hot = (lab_runs[g] for g in mi.LAB.gammas)
    assert none["capacity"] == 240
    assert none["max_vio"][late].mean() > 0.8 and none["max_vio"][late].min() > 0.6
    assert 0.03 < none["drop_rate"][late].mean() < 0.15
    assert good["max_vio"][late].mean() < 0.4
    assert good["drop_rate"][late].mean() < 0.005
    assert 0.01 < hot["drop_rate"][late].mean() < 0.10
    assert good["drop_rate"][late].mean() < hot["drop_rate"][late].mean() < none["drop_rate"][late].mean()
    assert good["max_vio"][late].mean() < hot["max_vio"][late].mean() < none["max_vio"][late].mean()


def test_lab_bias_moves_against_load(lab_runs):
    """The controller's direction (§02e): after each step, experts loaded above
    the ideal lose gamma, those below gain it, those exactly at it keep b."""
    r = lab_runs[0.01]
    w = mi.LAB
    for st in (0, 1, 37, 99):
        L = r["counts"][st].astype(np.int64)
        step = r["bias"][st + 1].astype(np.float64) - r["bias"][st].astype(np.float64)
        over, under = w.k * w.T < w.n_routed * L, w.k * w.T > w.n_routed * L
        assert (step[over] < 0).all() and (step[under] > 0).all()
        assert (step[~over & ~under] == 0).all()
        np.testing.assert_allclose(np.abs(step[over | under]), 0.01, rtol=1e-4)
    # no balancing: the bias never moves
    assert (lab_runs[0.0]["bias"] == 0).all()
