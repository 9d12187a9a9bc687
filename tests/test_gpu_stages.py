"""GPU parity of each C-ABI call against the CPU oracle, on seeded synthetic
inputs (both sides read the same generated tensors), at sizes that span
several tiles and ragged tails, plus the edge cases."""
import json
import os

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from parity import GATE_ATOL, check_output, check_routing, dev_bf16, host_bf16_bits, host_bf16_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if torch.cuda.is_available():
    import sparse_moe_layer_joint_b200 as moe


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _random_topk(T, k, E, seed):
    w = mi.words(T * E, seed, mi.STREAM_TEST_TOPK).reshape(T, E)
    return np.argsort(w, axis=1, kind="stable")[:, :k].astype(np.int32)


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------
@pytest.fixture(params=["default", "tensor", "small", "cluster"])
def router_path(request, monkeypatch):
    """Every router kernel on the same cases: the path the library picks, the tcgen05 router
    (forced), and the small-batch CUDA-core routers forced at any T: the one-CTA kernel (narrow
    rows) and the cluster kernel."""
    monkeypatch.delenv("MOE_ROUTER_SINGLE", raising=False)
    if request.param == "default":
        monkeypatch.delenv("MOE_ROUTER_SMALL", raising=False)
    else:
        monkeypatch.setenv("MOE_ROUTER_SMALL", "0" if request.param == "tensor" else "1")
    if request.param == "cluster":
        monkeypatch.setenv("MOE_ROUTER_SINGLE", "0")
    return request.param


def _run_router(x_u16, wr_u16, bias, k, n_routed, n_shared, offset=None, scores=False):
    T, d = x_u16.shape
    x = dev_bf16(x_u16)
    wr = dev_bf16(wr_u16)
    b = _f32(bias)
    off = None if offset is None else _f32(offset)
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    g = torch.full((T, k + n_shared), float("nan"), dtype=torch.float32, device="cuda")
    c = torch.full((n_routed,), 12345, dtype=torch.int32, device="cuda")
    sc = torch.empty((T, n_routed + n_shared), dtype=torch.float32, device="cuda") if scores else None
    moe.moe_router_topk(x, wr, b, off, T, d, n_routed, n_shared, k, 1.0, idx, g, c, sc)
    torch.cuda.synchronize()
    out = (idx.cpu().numpy(), g.cpu().numpy().astype(np.float64), c.cpu().numpy())
    return out + ((sc.cpu().numpy(),) if scores else ())


@pytest.mark.parametrize("case", ["no_bias", "with_bias"])
def test_router_worked_example(case, router_path):
    """The §02c hand example through the GPU: 4 routed experts, top-2, logits
    z fed as x = e_0 and W_r[:, 0] = z (z rounded to bf16, which keeps the order)."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "worked_example_routing.json")) as fh:
        g = json.load(fh)
    d = 64
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    wr = np.zeros((4, d), np.float32)
    wr[:, 0] = g["z"]
    c = g[case]
    idx, gates, counts = _run_router(mi.f32_to_bf16_bits(x), mi.f32_to_bf16_bits(wr), np.array(c["bias"]), 2, 4, 0)
    assert list(idx[0] + 1) == c["selected_1based"]
    np.testing.assert_allclose(gates[0], c["gates_3dp"], atol=1e-3)
    assert list(counts) == [1 if i + 1 in c["selected_1based"] else 0 for i in range(4)]


@pytest.mark.parametrize("T,d,n_routed,n_shared,k", [
    (1, 64, 256, 2, 6), (7, 128, 256, 2, 6), (300, 256, 256, 2, 6), (1000, 512, 256, 2, 6),
    (200, 64, 8, 2, 3), (130, 192, 64, 0, 2), (129, 128, 256, 8, 8), (256, 64, 16, 1, 1),
    # widths that are not a multiple of 64 (the last K block is read as zeros past d)
    (2048, 32, 64, 0, 6), (300, 96, 256, 2, 6), (129, 8, 16, 2, 4), (1000, 200, 256, 2, 6),
])
def test_router_parity(T, d, n_routed, n_shared, k, router_path):
    E = n_routed + n_shared
    x = mi.normal_bf16(T * d, 1, mi.STREAM_X).reshape(T, d)
    wr = mi.normal_bf16(E * d, 1, mi.STREAM_WR, std=1 / np.sqrt(d)).reshape(E, d)
    b = mi.uniform_f32(n_routed, 1, mi.STREAM_B, -0.05, 0.05)
    ref = oracle.route(oracle.logits(x, wr), b, k, n_routed, n_shared)
    idx, gates, counts, scores = _run_router(x, wr, b, k, n_routed, n_shared, scores=True)
    check_routing(idx, gates, counts, ref, k, n_routed, n_shared)
    np.testing.assert_allclose(scores, ref["s"], atol=2e-6)


def test_router_logit_offset_and_ties(router_path):
    """A logit offset enters the affinity (and so the gates); exact ties keep the lower index."""
    T, d, n_routed, k = 64, 64, 32, 4
    x = np.zeros((T, d), np.float32)
    x[:, 0] = 1.0
    wr = np.zeros((n_routed + 2, d), np.float32)      # every logit 0: all scores tie
    off = np.zeros(n_routed, np.float32)
    off[[5, 9]] = 1.0                                   # two experts lifted
    xb, wb = mi.f32_to_bf16_bits(x), mi.f32_to_bf16_bits(wr)
    idx, gates, counts = _run_router(xb, wb, np.zeros(n_routed), k, n_routed, 2, offset=off)
    assert (idx == np.array([5, 9, 0, 1])).all()
    ref = oracle.route(oracle.logits(xb, wb), np.zeros(n_routed, np.float32), k, n_routed, 2, off)
    np.testing.assert_allclose(gates, ref["gates"], atol=1e-6)


def test_router_bias_never_touches_gates(router_path):
    """Same token, two biases: where the kept set is the same, the gates are bit-identical."""
    T, d = 512, 256
    x = mi.normal_bf16(T * d, 2, mi.STREAM_X).reshape(T, d)
    wr = mi.normal_bf16(258 * d, 2, mi.STREAM_WR, std=1 / 16).reshape(258, d)
    i0, g0, _ = _run_router(x, wr, np.zeros(256), 6, 256, 2)
    i1, g1, _ = _run_router(x, wr, mi.uniform_f32(256, 2, mi.STREAM_B, -0.05, 0.05), 6, 256, 2)
    same = np.array([set(a) == set(b) for a, b in zip(i0, i1)])
    assert same.any() and (~same).any()
    for t in np.nonzero(same)[0]:
        m0 = dict(zip(list(i0[t]) + [256, 257], g0[t]))
        m1 = dict(zip(list(i1[t]) + [256, 257], g1[t]))
        assert m0 == m1


def test_router_zero_tokens_zeroes_counts(router_path):
    c = torch.full((256,), 99, dtype=torch.int32, device="cuda")
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((258, 64), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(256, dtype=torch.float32, device="cuda")
    idx = torch.zeros((1, 6), dtype=torch.int32, device="cuda")
    g = torch.zeros((1, 8), dtype=torch.float32, device="cuda")
    moe.moe_router_topk(x, w, b, None, 0, 64, 256, 2, 6, 1.0, idx, g, c)
    torch.cuda.synchronize()
    assert (c.cpu().numpy() == 0).all()


# ---------------------------------------------------------------------------
# permute (dispatch): integer work, bit-exact
# ---------------------------------------------------------------------------
@pytest.fixture(params=["one_chunk", "chunked"])
def permute_path(request, monkeypatch):
    """Batches of at most 256 tokens: the single-CTA index kernel (default) and the three chunked launches."""
    monkeypatch.setenv("MOE_PERMUTE_ONE_CHUNK", "1" if request.param == "one_chunk" else "0")
    return request.param


@pytest.mark.parametrize("T,k,n_routed,d", [
    (1, 6, 256, 64), (7, 2, 8, 16), (255, 6, 256, 128), (256, 6, 256, 64), (257, 3, 64, 72),
    (1000, 8, 256, 256), (4096, 6, 256, 2048), (3000, 1, 16, 8),
])
def test_permute_parity(T, k, n_routed, d, permute_path):
    topk = _random_topk(T, k, n_routed, T + k)
    x = mi.normal_bf16(T * d, 3, mi.STREAM_X).reshape(T, d)
    ref = oracle.dispatch(topk, n_routed)
    counts = oracle.load_counts(topk, n_routed)
    R = T * k
    off = torch.full((n_routed + 1,), -5, dtype=torch.int32, device="cuda")
    xp = torch.full((R, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    rt = torch.full((R,), -5, dtype=torch.int32, device="cuda")
    tr = torch.full((T, k), -5, dtype=torch.int32, device="cuda")
    nb = moe.moe_permute_scratch_bytes(T, n_routed)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    moe.moe_permute(dev_bf16(x), _i32(topk), _i32(counts), T, d, n_routed, k, off, xp, rt, tr, scratch, nb)
    assert moe.moe_get_status() == 0
    np.testing.assert_array_equal(off.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(rt.cpu().numpy(), ref["row_token"])
    np.testing.assert_array_equal(tr.cpu().numpy(), ref["token_row"])
    np.testing.assert_array_equal(host_bf16_bits(xp), x[ref["row_token"]])


def test_permute_indices_only():
    """x_perm = NULL: the same offsets / row_token / token_row, no row copy."""
    T, k, n = 1000, 6, 256
    topk = _random_topk(T, k, n, 21)
    ref = oracle.dispatch(topk, n)
    off = torch.full((n + 1,), -5, dtype=torch.int32, device="cuda")
    rt = torch.full((T * k,), -5, dtype=torch.int32, device="cuda")
    tr = torch.full((T, k), -5, dtype=torch.int32, device="cuda")
    nb = moe.moe_permute_scratch_bytes(T, n)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    moe.moe_permute(None, _i32(topk), None, T, 64, n, k, off, None, rt, tr, scratch, nb)
    assert moe.moe_get_status() == 0
    np.testing.assert_array_equal(off.cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(rt.cpu().numpy(), ref["row_token"])
    np.testing.assert_array_equal(tr.cpu().numpy(), ref["token_row"])


@pytest.mark.parametrize("T", [300, 200])
def test_permute_reports_bad_inputs(T):
    k, n = 2, 16
    topk = _random_topk(T, k, n, 5)
    wrong = oracle.load_counts(topk, n)
    wrong[3] += 1
    nb = moe.moe_permute_scratch_bytes(T, n)
    bufs = dict(off=torch.zeros(n + 1, dtype=torch.int32, device="cuda"),
                xp=torch.zeros((T * k, 8), dtype=torch.bfloat16, device="cuda"),
                rt=torch.zeros(T * k, dtype=torch.int32, device="cuda"),
                tr=torch.zeros((T, k), dtype=torch.int32, device="cuda"),
                sc=torch.empty(nb, dtype=torch.uint8, device="cuda"))
    x = torch.zeros((T, 8), dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(x, _i32(topk), _i32(wrong), T, 8, n, k, bufs["off"], bufs["xp"], bufs["rt"], bufs["tr"],
                    bufs["sc"], nb)
    assert moe.moe_get_status() == moe.MOE_STATUS_COUNT_MISMATCH
    topk_bad = topk.copy()
    topk_bad[10, 1] = 999
    moe.moe_permute(x, _i32(topk_bad), None, T, 8, n, k, bufs["off"], bufs["xp"], bufs["rt"], bufs["tr"],
                    bufs["sc"], nb)
    assert moe.moe_get_status() & moe.MOE_STATUS_BAD_EXPERT
    assert bufs["tr"].cpu().numpy()[10, 1] == -1
    with pytest.raises(moe.MoEError):
        moe.moe_permute(x, _i32(topk), None, T, 8, n, k, bufs["off"], bufs["xp"], bufs["rt"], bufs["tr"],
                        bufs["sc"], 8)


# ---------------------------------------------------------------------------
# grouped expert MLPs (tcgen05)
# ---------------------------------------------------------------------------
def _ffn_weights(E, d, f, seed):
    w1 = mi.normal_bf16(E * f * d, seed, mi.STREAM_W1, std=1 / np.sqrt(d)).reshape(E, f, d)
    w2 = mi.normal_bf16(E * d * f, seed, mi.STREAM_W2, std=1 / np.sqrt(f)).reshape(E, d, f)
    return w1, w2


@pytest.fixture(params=["pair", "pair4", "wide", "wide3", "nohalf", "nmajor", "tails", "single"])
def gemm_variant(request, monkeypatch):
    """Every grouped-GEMM kernel: CTA pairs on 256 x 256 tiles with six pipeline stages (short
    launches) and with four (long launches), pairs on 256 x 512 tiles with four stages (the default for
    pair launches with the GELU and plain epilogues; SwiGLU launches keep 256-wide tiles) and with
    three, the wide pairs without half (M = 128) tiles for the groups' last rows, pairs walking small groups
    column-tile-major, pairs on each group's whole 256-row blocks followed by single CTAs on the rows
    past them, and single CTAs."""
    monkeypatch.setenv("MOE_GEMM_NMAJOR", "4" if request.param == "nmajor" else "0")
    monkeypatch.setenv("MOE_GEMM_TAILS", "1" if request.param == "tails" else "0")
    monkeypatch.setenv("MOE_GEMM_CTA", "1" if request.param == "single" else "2")
    if request.param in ("pair4", "wide3"):
        monkeypatch.setenv("MOE_GEMM_STAGES", "4,4" if request.param == "pair4" else "3,3")
    else:
        monkeypatch.delenv("MOE_GEMM_STAGES", raising=False)
    monkeypatch.setenv("MOE_GEMM_WIDE", "1" if request.param.startswith("wide") or request.param == "nohalf" else "0")
    monkeypatch.setenv("MOE_GEMM_HALF", "0" if request.param == "nohalf" else "1")
    return request.param


@pytest.mark.parametrize("sizes,d,f", [
    ([0, 1, 127, 128, 129, 300, 0, 5], 256, 128),
    ([200, 37, 0, 513], 512, 768),
    ([64] * 16, 128, 256),
    ([1000], 1024, 512),
    ([3, 0, 0, 0, 250, 7], 2048, 1024),
    ([129, 255, 256, 257, 0, 511, 1], 256, 256),
])
def test_grouped_ffn_parity(sizes, d, f, gemm_variant):
    G = len(sizes)
    n = int(sum(sizes))
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows = mi.normal_bf16(n * d, 4, mi.STREAM_TEST_ROWS).reshape(n, d)
    base = 3
    w1, w2 = _ffn_weights(G + base, d, f, 4)
    h = torch.empty((n, f), dtype=torch.bfloat16, device="cuda")
    y = torch.full((n, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_ffn(dev_bf16(rows), _i32(offsets), G, n, base, dev_bf16(w1), dev_bf16(w2), d, f,
                        moe.MOE_ACT_GELU_TANH, h, y)
    assert moe.moe_get_status() == 0
    yg = host_bf16_f64(y)
    for g in range(G):
        a, b = offsets[g], offsets[g + 1]
        if a == b:
            continue
        ref = oracle.expert(rows[a:b], w1[base + g], w2[base + g])
        check_output(yg[a:b], ref, f"group {g}")


@pytest.mark.parametrize("n,G,d,f", [(1, 2, 64, 64), (300, 2, 256, 128), (1030, 3, 512, 256)])
def test_grouped_ffn_identity_groups(n, G, d, f, gemm_variant):
    """offsets = NULL: every group (expert) sees all rows, as the shared experts do."""
    rows = mi.normal_bf16(n * d, 6, mi.STREAM_TEST_ROWS).reshape(n, d)
    w1, w2 = _ffn_weights(G + 5, d, f, 6)
    h = torch.empty((G, n, f), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((G, n, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_ffn(dev_bf16(rows), None, G, n, 5, dev_bf16(w1), dev_bf16(w2), d, f, moe.MOE_ACT_GELU_TANH, h, y)
    yg = host_bf16_f64(y)
    for g in range(G):
        check_output(yg[g], oracle.expert(rows, w1[5 + g], w2[5 + g]), f"group {g}")


def test_grouped_ffn_special_weights(gemm_variant):
    """W2 = 0 gives exactly 0; W1 = W2 = I (d = d_ff) gives bf16(gelu(x))."""
    n, d = 260, 128
    rows = mi.normal_bf16(n * d, 7, mi.STREAM_TEST_ROWS).reshape(n, d)
    eye = mi.f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    w1 = np.stack([eye, eye])
    w2 = np.stack([np.zeros_like(eye), eye])
    off = _i32([0, 100, n])
    h = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_ffn(dev_bf16(rows), off, 2, n, 0, dev_bf16(w1), dev_bf16(w2), d, d, 0, h, y)
    yg = host_bf16_f64(y)
    assert (yg[:100] == 0).all()
    ref = oracle.gelu_tanh(mi.bf16_to_f64(rows[100:]))
    np.testing.assert_allclose(yg[100:], ref, rtol=2 ** -7, atol=2e-3)


@pytest.mark.parametrize("T,n_routed,n_shared,k,d,f", [
    (300, 16, 2, 3, 256, 128), (1000, 8, 2, 2, 512, 256), (64, 64, 2, 6, 256, 256), (700, 4, 0, 2, 128, 128),
    (129, 0, 2, 1, 128, 192),
])
@pytest.mark.parametrize("gather", [False, True])
def test_experts_ffn_parity(T, n_routed, n_shared, k, d, f, gemm_variant, gather):
    """Routed experts on dispatched rows (copied by moe_permute, or gathered by the GEMM
    itself through row_token) and shared experts on all tokens, one pair of launches."""
    E = n_routed + n_shared
    x = mi.normal_bf16(T * d, 11, mi.STREAM_X).reshape(T, d)
    w1, w2 = _ffn_weights(E, d, f, 11)
    R = T * k
    h = torch.empty((R + n_shared * T, f), dtype=torch.bfloat16, device="cuda")
    y_perm = torch.full((max(R, 1), d), float("nan"), dtype=torch.bfloat16, device="cuda")
    y_sh = torch.full((max(n_shared, 1), T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    if n_routed:
        topk = _random_topk(T, k, n_routed, 12)
        dp = oracle.dispatch(topk, n_routed)
        xp = x[dp["row_token"]]
        moe.moe_experts_ffn(dev_bf16(x), None if gather else dev_bf16(xp), _i32(dp["row_token"]),
                            _i32(dp["offsets"]), T, n_routed, n_shared, k, dev_bf16(w1), dev_bf16(w2), d, f,
                            moe.MOE_ACT_GELU_TANH, h, y_perm, y_sh)
    else:
        moe.moe_experts_ffn(dev_bf16(x), None, None, None, T, 0, n_shared, k, dev_bf16(w1), dev_bf16(w2), d, f,
                            moe.MOE_ACT_GELU_TANH, h, y_perm, y_sh)
    assert moe.moe_get_status() == 0
    if n_routed:
        yp = host_bf16_f64(y_perm)
        off = dp["offsets"]
        for e in range(n_routed):
            if off[e] < off[e + 1]:
                check_output(yp[off[e]:off[e + 1]], oracle.expert(xp[off[e]:off[e + 1]], w1[e], w2[e]), f"routed {e}")
    ys = host_bf16_f64(y_sh)
    for sidx in range(n_shared):
        check_output(ys[sidx], oracle.expert(x, w1[n_routed + sidx], w2[n_routed + sidx]), f"shared {sidx}")


# ---------------------------------------------------------------------------
# SwiGLU experts (the released configuration: "Under the hood", SwiGLU FFNs)
# ---------------------------------------------------------------------------
def _swiglu_weights(E, d, f, seed):
    w1 = mi.normal_bf16(E * 2 * f * d, seed, mi.STREAM_W1, std=1 / np.sqrt(d)).reshape(E, 2 * f, d)
    w2 = mi.normal_bf16(E * d * f, seed, mi.STREAM_W2, std=1 / np.sqrt(f)).reshape(E, d, f)
    return w1, w2


@pytest.mark.parametrize("sizes,d,f", [
    ([0, 1, 127, 128, 129, 300, 0, 5], 256, 128),
    ([200, 37, 0, 513], 512, 192),          # d_ff not a multiple of 128: a half-width last tile
    ([64] * 16, 128, 64),
    ([1000], 1024, 512),
    ([129, 255, 256, 257, 0, 511, 1], 256, 384),
])
def test_grouped_ffn_swiglu_parity(sizes, d, f, gemm_variant):
    G = len(sizes)
    n = int(sum(sizes))
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows = mi.normal_bf16(n * d, 14, mi.STREAM_TEST_ROWS).reshape(n, d)
    base = 2
    w1, w2 = _swiglu_weights(G + base, d, f, 14)
    h = torch.full((n, f), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((n, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_ffn(dev_bf16(rows), _i32(offsets), G, n, base, dev_bf16(w1), dev_bf16(w2), d, f,
                        moe.MOE_ACT_SWIGLU, h, y)
    assert moe.moe_get_status() == 0
    yg = host_bf16_f64(y)
    for g in range(G):
        a, b = offsets[g], offsets[g + 1]
        if a == b:
            continue
        ref = oracle.expert_swiglu(rows[a:b], w1[base + g], w2[base + g])
        check_output(yg[a:b], ref, f"group {g}")


def test_swiglu_special_weights(gemm_variant):
    """Wg = I, Wu = I, W2 = I (d = d_ff): y = bf16(silu(x) * x); Wu = 0 gives exactly 0."""
    n, d = 300, 128
    rows = mi.normal_bf16(n * d, 15, mi.STREAM_TEST_ROWS).reshape(n, d)
    eye = mi.f32_to_bf16_bits(np.eye(d, dtype=np.float32))
    zero = np.zeros_like(eye)
    w1 = np.stack([np.concatenate([eye, eye]), np.concatenate([eye, zero])])
    w2 = np.stack([eye, eye])
    off = _i32([0, 200, n])
    h = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((n, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_ffn(dev_bf16(rows), off, 2, n, 0, dev_bf16(w1), dev_bf16(w2), d, d, moe.MOE_ACT_SWIGLU, h, y)
    yg = host_bf16_f64(y)
    xr = mi.bf16_to_f64(rows[:200])
    np.testing.assert_allclose(yg[:200], oracle.silu(xr) * xr, rtol=2 ** -6, atol=2e-3)
    assert (yg[200:] == 0).all()


@pytest.mark.parametrize("T,n_routed,n_shared,k,d,f", [
    (300, 16, 2, 3, 256, 128), (64, 64, 2, 6, 384, 192), (700, 4, 0, 2, 128, 128), (129, 0, 2, 1, 128, 256),
])
def test_experts_ffn_swiglu_parity(T, n_routed, n_shared, k, d, f, gemm_variant):
    E = n_routed + n_shared
    x = mi.normal_bf16(T * d, 16, mi.STREAM_X).reshape(T, d)
    w1, w2 = _swiglu_weights(E, d, f, 16)
    R = T * k
    h = torch.empty((R + n_shared * T, f), dtype=torch.bfloat16, device="cuda")
    y_perm = torch.full((max(R, 1), d), float("nan"), dtype=torch.bfloat16, device="cuda")
    y_sh = torch.full((max(n_shared, 1), T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    xp = None
    if n_routed:
        topk = _random_topk(T, k, n_routed, 17)
        dp = oracle.dispatch(topk, n_routed)
        xp = x[dp["row_token"]]
        moe.moe_experts_ffn(dev_bf16(x), dev_bf16(xp), _i32(dp["row_token"]), _i32(dp["offsets"]), T, n_routed,
                            n_shared, k, dev_bf16(w1), dev_bf16(w2), d, f, moe.MOE_ACT_SWIGLU, h, y_perm, y_sh)
    else:
        moe.moe_experts_ffn(dev_bf16(x), None, None, None, T, 0, n_shared, k, dev_bf16(w1), dev_bf16(w2), d, f,
                            moe.MOE_ACT_SWIGLU, h, y_perm, y_sh)
    assert moe.moe_get_status() == 0
    if n_routed:
        yp = host_bf16_f64(y_perm)
        off = dp["offsets"]
        for e in range(n_routed):
            if off[e] < off[e + 1]:
                check_output(yp[off[e]:off[e + 1]], oracle.expert_swiglu(xp[off[e]:off[e + 1]], w1[e], w2[e]),
                             f"routed {e}")
    ys = host_bf16_f64(y_sh)
    for sidx in range(n_shared):
        check_output(ys[sidx], oracle.expert_swiglu(x, w1[n_routed + sidx], w2[n_routed + sidx]), f"shared {sidx}")


@pytest.mark.parametrize("scale", [8.0, 2.83])
def test_router_route_scale(scale, router_path):
    """Joint weights times route_scale x global_scale: sums equal the scale, values the
    oracle's scaled weights, selection unchanged."""
    T, d = 700, 256
    x = mi.normal_bf16(T * d, 9, mi.STREAM_X).reshape(T, d)
    wr = mi.normal_bf16(258 * d, 9, mi.STREAM_WR, std=1 / 16).reshape(258, d)
    b = mi.uniform_f32(256, 9, mi.STREAM_B, -0.05, 0.05)
    ref = oracle.route(oracle.logits(x, wr), b, 6, 256, 2, route_scale=scale)
    xd, wd, bd = dev_bf16(x), dev_bf16(wr), _f32(b)
    idx = torch.empty((T, 6), dtype=torch.int32, device="cuda")
    g = torch.empty((T, 8), dtype=torch.float32, device="cuda")
    c = torch.empty(256, dtype=torch.int32, device="cuda")
    moe.moe_router_topk(xd, wd, bd, None, T, d, 256, 2, 6, scale, idx, g, c)
    g1 = torch.empty_like(g)
    moe.moe_router_topk(xd, wd, bd, None, T, d, 256, 2, 6, 1.0, idx, g1, c)
    torch.cuda.synchronize()
    check_routing(idx.cpu().numpy(), g.cpu().numpy().astype(np.float64), c.cpu().numpy(), ref, 6, 256, 2,
                  gate_scale=scale)
    # the scale is one fp32 multiply after the normalisation
    np.testing.assert_array_equal(g.cpu().numpy(), (g1.cpu().numpy() * np.float32(scale)).astype(np.float32))


# ---------------------------------------------------------------------------
# combine
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,k,ns,d", [(1, 6, 2, 64), (333, 6, 2, 256), (1024, 2, 0, 128), (100, 8, 8, 72)])
def test_combine_parity(T, k, ns, d):
    topk = _random_topk(T, k, 64, 8)
    dp = oracle.dispatch(topk, 64)
    y = mi.normal_bf16(T * k * d, 8, mi.STREAM_TEST_ROWS).reshape(T * k, d)
    ysh = mi.normal_bf16(max(ns, 1) * T * d, 8, mi.STREAM_TEST_SHARED).reshape(max(ns, 1), T, d)
    g = np.abs(mi.normal_f32(T * (k + ns), 8, mi.STREAM_TEST_GATES)).reshape(T, k + ns)
    g /= g.sum(axis=1, keepdims=True)
    g = g.astype(np.float32)
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(dev_bf16(y), _i32(dp["token_row"]), _f32(g), dev_bf16(ysh) if ns else None, T, d, k, ns, out)
    ref = oracle.combine(mi.bf16_to_f64(y), dp["token_row"], g.astype(np.float64),
                         mi.bf16_to_f64(ysh[:ns]) if ns else None)
    got = host_bf16_f64(out)
    np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-5)


# ---------------------------------------------------------------------------
# bias update: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T,k,n,gamma", [(256, 6, 256, 1e-3), (4096, 6, 256, 1e-3), (100, 6, 256, 0.01),
                                         (1000, 3, 64, 0.05)])
def test_bias_update_bit_exact(T, k, n, gamma):
    mean = k * T // n
    w = mi.words(n, T, mi.STREAM_TEST_TOPK)
    counts = (mean + (w % 5).astype(np.int64) - 2).clip(0).astype(np.int32)   # includes counts == mean
    b = mi.uniform_f32(n, T, mi.STREAM_B, -0.1, 0.1)
    bd = _f32(b)
    moe.moe_bias_update(_i32(counts), n, T, k, gamma, bd)
    ref = oracle.bias_update(counts, b, T, k, gamma)
    np.testing.assert_array_equal(bd.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ---------------------------------------------------------------------------
# failure path: a bounded device wait gives up and reports, the context lives on
# ---------------------------------------------------------------------------
def test_bounded_wait_times_out_and_reports():
    assert moe.moe_get_status() == 0
    moe.moe_debug_bounded_wait(50_000_000)     # 50 ms on a barrier nothing completes
    st = moe.moe_get_status()
    assert st & moe.MOE_STATUS_TIMEOUT
    assert moe.moe_get_status() == 0           # cleared by the read
    # the context still works
    idx, gates, counts = _run_router(mi.normal_bf16(64 * 64, 1, 1).reshape(64, 64),
                                     mi.normal_bf16(258 * 64, 1, 2, std=0.125).reshape(258, 64),
                                     np.zeros(256), 6, 256, 2)
    assert counts.sum() == 64 * 6


def test_debug_sync_reports_the_failing_call(monkeypatch):
    """With the debug-sync check on, a device-side timeout raises at the call that timed out,
    also when that call ran on a stream other than the current one."""
    assert moe.moe_get_status() == 0
    monkeypatch.setattr(moe, "_DEBUG_SYNC", True)
    side = torch.cuda.Stream()
    with pytest.raises(moe.MoEError) as err:
        moe.moe_debug_bounded_wait(20_000_000, stream=side)
    assert "moe_debug_bounded_wait" in str(err.value) and err.value.code == moe.MOE_ERR_TIMEOUT
    moe.moe_permute_scratch_bytes(64, 256)          # a call that does not check the status
    assert moe.moe_get_status() == 0                 # the debug check read and cleared the bit


def test_generator_device_matches_host():
    """The device generator writes the same bits as the host generator."""
    w = mi.WORKLOADS["tiny"]
    t = mi.torch_workload(w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16_bits(t["x"]), mi.host_x(w))
    np.testing.assert_array_equal(host_bf16_bits(t["w_r"]), mi.host_wr(w))
    np.testing.assert_array_equal(host_bf16_bits(t["w1"][17]), mi.host_w1(w, 17))
    np.testing.assert_array_equal(host_bf16_bits(t["w2"][257]), mi.host_w2(w, 257))
    np.testing.assert_array_equal(t["bias"].cpu().numpy(), mi.host_bias(w))
    n = 1 << 20
    a = torch.empty(n, dtype=torch.float32, device="cuda")
    mi.gpu_normal_f32(a.data_ptr(), n, 9, 3, 12345, 0.5, torch.cuda.current_stream().cuda_stream)
    np.testing.assert_array_equal(a.cpu().numpy(), mi.normal_f32(n, 9, 3, 12345, 0.5))
