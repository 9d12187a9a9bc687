"""Expert capacity on the GPU ("Inkling, Dissected" §02d: overflow assignments
are dropped; §02g: the Router Balance Lab) against the oracle: the capped
dispatch bit-exact, the load statistics exact, the layer output with drops,
and the lab's 100-step balancing loop per step."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from parity import MARGIN, check_output, dev_bf16, host_bf16_bits, host_bf16_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if torch.cuda.is_available():
    import sparse_moe_layer_joint_b200 as moe


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _topk(T, k, E, seed, skew=0.0):
    """Seeded top-k rows with distinct experts; skew > 0 favours low expert ids."""
    u = mi.words(T * E, seed, mi.STREAM_TEST_TOPK).reshape(T, E).astype(np.float64) / 2 ** 32
    score = u - skew * np.log1p(np.arange(E))[None, :]
    return np.argsort(-score, axis=1, kind="stable")[:, :k].astype(np.int32)


def _permute_capped(topk, x, cap, n_routed):
    T, k = topk.shape
    d = x.shape[1]
    R = T * k
    off = torch.full((n_routed + 1,), -5, dtype=torch.int32, device="cuda")
    xp = torch.full((max(R, 1), d), float("nan"), dtype=torch.bfloat16, device="cuda")
    rt = torch.full((max(R, 1),), -5, dtype=torch.int32, device="cuda")
    tr = torch.full((T, k), -5, dtype=torch.int32, device="cuda")
    nb = moe.moe_permute_scratch_bytes(T, n_routed)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    counts = oracle.load_counts(topk, n_routed)
    moe.moe_permute_capped(dev_bf16(x), _i32(topk), _i32(counts), T, d, n_routed, k, cap, off, xp, rt, tr,
                           scratch, nb)
    assert moe.moe_get_status() == 0
    return off.cpu().numpy(), rt.cpu().numpy(), tr.cpu().numpy(), host_bf16_bits(xp)


@pytest.mark.parametrize("T,k,E,d,cap,skew", [
    (1, 6, 256, 64, 0, 0.0), (1, 6, 256, 64, 1, 0.0), (255, 6, 256, 64, 3, 0.5), (256, 6, 64, 72, 24, 0.3),
    (1000, 8, 256, 128, 30, 0.2), (2048, 6, 64, 32, 240, 0.1), (4097, 6, 256, 256, 120, 0.05),
    (3000, 1, 16, 8, 150, 1.0), (777, 3, 8, 16, 10 ** 6, 0.5),
])
@pytest.mark.parametrize("one_chunk", ["1", "0"])
def test_permute_capped_parity(T, k, E, d, cap, skew, one_chunk, monkeypatch):
    monkeypatch.setenv("MOE_PERMUTE_ONE_CHUNK", one_chunk)  # batches of <= 256 tokens: both index paths
    topk = _topk(T, k, E, T + E, skew)
    x = mi.normal_bf16(T * d, 5, mi.STREAM_X).reshape(T, d)
    keep = oracle.capacity_keep(topk, cap, E)
    ref = oracle.dispatch(topk, E, keep)
    off, rt, tr, xp = _permute_capped(topk, x, cap, E)
    n = int(ref["offsets"][-1])
    np.testing.assert_array_equal(off, ref["offsets"])
    np.testing.assert_array_equal(tr, ref["token_row"])
    np.testing.assert_array_equal(rt[:n], ref["row_token"])
    np.testing.assert_array_equal(xp[:n], x[ref["row_token"]])
    # rows past the served ones are left alone
    assert (rt[n:] == -5).all()


def test_permute_capped_without_overflow_is_permute():
    T, k, E, d = 1000, 6, 256, 64
    topk = _topk(T, k, E, 17)
    x = mi.normal_bf16(T * d, 6, mi.STREAM_X).reshape(T, d)
    L = oracle.load_counts(topk, E)
    ref = oracle.dispatch(topk, E)
    off, rt, tr, xp = _permute_capped(topk, x, int(L.max()), E)
    np.testing.assert_array_equal(off, ref["offsets"])
    np.testing.assert_array_equal(rt, ref["row_token"])
    np.testing.assert_array_equal(tr, ref["token_row"])


@pytest.mark.parametrize("E,cap,skew", [(256, 0, 0.0), (256, 20, 0.3), (64, 240, 0.1), (1, 5, 0.0), (200, 10 ** 6, 0.2)])
def test_load_stats_exact(E, cap, skew):
    T, k = 2048, min(6, E)
    topk = _topk(T, k, E, E + 3, skew)
    L = oracle.load_counts(topk, E)
    st = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    mt = torch.full((2,), -1, dtype=torch.float32, device="cuda")
    moe.moe_load_stats(_i32(L), E, T, k, cap, st, mt)
    got = st.cpu().numpy()
    m = oracle.load_metrics(L, cap, T, k)
    assert got[0] == m["max_load"] and got[1] == m["dropped"]
    # MaxVio and the drop rate: the oracle's fp64 values rounded once to fp32
    np.testing.assert_array_equal(mt.cpu().numpy(), np.array([m["max_vio"], m["drop_rate"]], dtype=np.float32))


def _layer_with_capacity(name, factor, tokens):
    w = mi.WORKLOADS[name]
    t = mi.torch_workload(w)
    layer = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f, w.n_routed, w.n_shared, w.k), capacity_factor=factor)
    b_host = t["bias"].cpu().numpy()
    out = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    cap = oracle.capacity_for(factor, w.T, w.k, w.n_routed)
    assert layer.capacity == cap
    gpu_idx = layer.topk_idx.cpu().numpy()
    # the drops follow from the GPU's own routing (integer work: exact)
    keep = oracle.capacity_keep(gpu_idx, cap, w.n_routed)
    ref = oracle.dispatch(gpu_idx, w.n_routed, keep)
    np.testing.assert_array_equal(layer.offsets.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(layer.token_row.cpu().numpy(), ref["token_row"])
    bal = layer.balance()
    m = oracle.load_metrics(layer.counts.cpu().numpy(), cap, w.T, w.k)
    assert bal["dropped"] == m["dropped"] == int((~keep).sum()) and bal["max_load"] == m["max_load"]
    assert bal["max_vio"] == np.float32(m["max_vio"]) and bal["drop_rate"] == np.float32(m["drop_rate"])
    assert m["dropped"] > 0
    # the routing itself, and the output with the drops applied, against the oracle
    off = mi.host_logit_offset(w)
    r = oracle.forward_tokens(w, tokens, b_host, off, keep=keep[tokens])
    same = np.array([list(a) == list(b) for a, b in zip(gpu_idx[tokens], r["topk_idx"])])
    assert same.mean() > 0.9
    got = host_bf16_f64(out[torch.from_numpy(np.asarray(tokens)).cuda()])
    check_output(got[same], r["out"][same], f"{name} capacity {factor}")
    dropped_tokens = (~keep[tokens]).any(axis=1) & same
    assert dropped_tokens.any()
    return layer


def test_layer_tiny_with_capacity():
    """Capacity = the ideal load (6 tokens per expert): many drops; every token checked."""
    _layer_with_capacity("tiny", 1.0, np.arange(256))


@pytest.mark.slow
def test_layer_mid_with_capacity():
    _layer_with_capacity("mid", 1.0, np.arange(0, 4096, 41))


@pytest.mark.slow
def test_layer_skew_with_capacity():
    """Skewed routing at 1.25x capacity: the hot experts overflow."""
    _layer_with_capacity("skew", 1.25, np.arange(0, 16384, 601))


@pytest.mark.slow
def test_layer_prefill_with_capacity():
    """Full prefill size, capacity = the ideal load (1536 tokens per expert),
    sampled tokens (the GEMMs see the shortened groups; the combine skips the
    dropped slots)."""
    _layer_with_capacity("prefill", 1.0, np.array([0, 1, 2, 3, 4095, 30000, 65535]))


# ---------------------------------------------------------------------------
# Router Balance Lab: 100 steps per balancing arm, on the GPU
# ---------------------------------------------------------------------------
def _gpu_lab(w, gamma):
    """The lab loop through the C ABI; returns per-step GPU topk, counts, stats, bias."""
    cap = moe.capacity_for(w.capacity_factor, w.T, w.k, w.n_routed)
    xs = dev_bf16(mi.lab_x_all(w))                     # [steps, T, d]
    wr = dev_bf16(mi.lab_wr(w))
    b = torch.zeros(w.n_routed, dtype=torch.float32, device="cuda")
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    g = torch.empty((w.T, w.k), dtype=torch.float32, device="cuda")
    c = torch.empty(w.n_routed, dtype=torch.int32, device="cuda")
    off = torch.empty(w.n_routed + 1, dtype=torch.int32, device="cuda")
    rt = torch.empty(w.T * w.k, dtype=torch.int32, device="cuda")
    tr = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    nb = moe.moe_permute_scratch_bytes(w.T, w.n_routed)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    st = torch.empty(2, dtype=torch.int32, device="cuda")
    res = {"topk": [], "counts": [], "stats": [], "bias": [b.cpu().numpy()], "token_row": []}
    for s in range(w.steps):
        moe.moe_router_topk(xs[s], wr, b, None, w.T, w.d, w.n_routed, 0, w.k, 1.0, idx, g, c)
        moe.moe_permute_capped(None, idx, c, w.T, w.d, w.n_routed, w.k, cap, off, None, rt, tr, scratch, nb)
        moe.moe_load_stats(c, w.n_routed, w.T, w.k, cap, st)
        moe.moe_bias_update(c, w.n_routed, w.T, w.k, gamma, b)
        res["topk"].append(idx.cpu().numpy())
        res["counts"].append(c.cpu().numpy())
        res["stats"].append(st.cpu().numpy())
        res["token_row"].append(tr.cpu().numpy())
        res["bias"].append(b.cpu().numpy())
    assert moe.moe_get_status() == 0
    return res, cap


@pytest.mark.parametrize("gamma", mi.LAB.gammas)
def test_lab_loop_per_step(gamma):
    """Each step checked against the oracle from the GPU's own state: routing
    (near-tie exemption as everywhere), drops and stats exact, the bias update
    bit-exact; then the run's balance against the oracle's own 100-step run."""
    w = mi.LAB
    res, cap = _gpu_lab(w, gamma)
    wr = mi.lab_wr(w)
    max_vio, drop_rate = [], []
    for s in range(w.steps):
        b_prev = res["bias"][s]
        ref = oracle.route(oracle.logits(mi.lab_x(w, s), wr), b_prev, w.k, w.n_routed, 0)
        exempt = ref["margin"] < MARGIN
        same = np.array([set(a) == set(b) for a, b in zip(res["topk"][s], ref["topk_idx"])])
        assert (same | exempt).all(), (s, int((~same & ~exempt).sum()))
        L = res["counts"][s]
        np.testing.assert_array_equal(L, oracle.load_counts(res["topk"][s], w.n_routed))
        keep = oracle.capacity_keep(res["topk"][s], cap, w.n_routed)
        np.testing.assert_array_equal(res["token_row"][s] >= 0, keep)
        m = oracle.load_metrics(L, cap, w.T, w.k)
        assert list(res["stats"][s]) == [m["max_load"], m["dropped"]]
        nb = oracle.bias_update(L, b_prev, w.T, w.k, gamma)
        np.testing.assert_array_equal(res["bias"][s + 1].view(np.uint32), nb.view(np.uint32))
        max_vio.append(m["max_vio"])
        drop_rate.append(m["drop_rate"])
    ref_run = oracle.lab_run(w, gamma)
    late = slice(50, None)
    assert abs(np.mean(max_vio[late]) - ref_run["max_vio"][late].mean()) < 0.05
    assert abs(np.mean(drop_rate[late]) - ref_run["drop_rate"][late].mean()) < 0.005


@pytest.mark.slow
def test_layer_inkling_decode_with_capacity():
    """Capacity with the released configuration (SwiGLU experts, route_scale 8) at decode scale."""
    w = mi.WORKLOADS["inkling_decode"]
    t = mi.torch_workload(w)
    layer = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f, w.n_routed, w.n_shared, w.k), capacity_factor=1.0,
                         activation=w.activation, route_scale=w.gate_scale)
    b_host = t["bias"].cpu().numpy()
    out = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    gpu_idx = layer.topk_idx.cpu().numpy()
    keep = oracle.capacity_keep(gpu_idx, layer.capacity, w.n_routed)
    assert layer.capacity == 1 and (~keep).any()        # 64 * 6 / 256 = 1.5 -> 1 token per expert
    tokens = np.array([0, 5, 63])
    r = oracle.forward_tokens(w, tokens, b_host, keep=keep[tokens])
    same = np.array([list(a) == list(b) for a, b in zip(gpu_idx[tokens], r["topk_idx"])])
    got = host_bf16_f64(out[torch.from_numpy(tokens).cuda()])
    check_output(got[same], r["out"][same], "inkling_decode capacity")
