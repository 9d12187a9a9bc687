"""The whole layer on the GPU (router -> permute -> routed and shared experts
-> combine -> bias update, through the C ABI) against the oracle on the
workloads' seeded inputs: all tokens where the oracle finishes in seconds,
sampled tokens at the full sizes (tokens are independent, so a sample is
checked exactly), plus properties that hold at any size."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from parity import check_output, check_routing, host_bf16_bits, host_bf16_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if torch.cuda.is_available():
    import sparse_moe_layer_joint_b200 as moe


def _layer(w, with_weights=True, fused=True, gather=False):
    t = mi.torch_workload(w, with_weights=with_weights)
    layer = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f, w.n_routed, w.n_shared, w.k), fused_experts=fused,
                         gather_rows=gather, activation=w.activation, route_scale=w.gate_scale)
    return t, layer


def _check_dispatch_properties(layer, x_bits, T, k, n_routed):
    """Dispatch invariants at any size: offsets scan the counts, every (token,
    slot) row holds that token's x, rows of an expert are in token order."""
    off = layer.offsets.cpu().numpy().astype(np.int64)
    counts = layer.counts.cpu().numpy()
    idx = layer.topk_idx.cpu().numpy()
    tr = layer.token_row.cpu().numpy()
    rt = layer.row_token.cpu().numpy()
    assert off[0] == 0 and (np.diff(off) == counts).all() and off[-1] == T * k
    np.testing.assert_array_equal(rt[tr.reshape(-1)], np.repeat(np.arange(T), k))
    seg = np.searchsorted(off, tr.reshape(-1), side="right") - 1
    np.testing.assert_array_equal(seg, idx.reshape(-1))
    for e in range(n_routed):
        r = rt[off[e]:off[e + 1]]
        assert (np.diff(r) > 0).all()
    if not layer.gather_rows:  # the rows were copied (otherwise the GEMM gathers them itself)
        sample = np.linspace(0, T * k - 1, min(T * k, 512)).astype(np.int64)
        xp = host_bf16_bits(layer.x_perm[torch.from_numpy(sample).cuda()])
        np.testing.assert_array_equal(xp, x_bits[rt[sample]])


def _check_expert_groups(w, layer, t, x_bits, experts, shared_tokens=None):
    """Whole row groups of the expert GEMMs at full size: every y_perm row of each
    listed expert (its ragged last tile included) against the oracle's expert on
    the token that row holds; optionally the shared experts' rows of some tokens."""
    off = layer.offsets.cpu().numpy().astype(np.int64)
    rt = layer.row_token.cpu().numpy()
    fn = oracle.expert_for(w)
    for e in experts:
        lo, hi = int(off[e]), int(off[e + 1])
        assert hi > lo
        got = host_bf16_f64(layer.y_perm[lo:hi])
        ref = fn(x_bits[rt[lo:hi]], host_bf16_bits(t["w1"][e]), host_bf16_bits(t["w2"][e]))
        check_output(got, ref, f"{w.name} expert {e} rows {lo}..{hi}")
    if shared_tokens is not None:
        for s_i in range(w.n_shared):
            e = w.n_routed + s_i
            got = host_bf16_f64(layer.y_shared[s_i][torch.from_numpy(shared_tokens).cuda()])
            ref = fn(x_bits[shared_tokens], host_bf16_bits(t["w1"][e]), host_bf16_bits(t["w2"][e]))
            check_output(got, ref, f"{w.name} shared expert {e}")


def _run_and_check(name, tokens=None, check_all_routing=True, fused=True, gather=False, expert_groups=None,
                   shared_tokens=None):
    w = mi.WORKLOADS[name]
    t, layer = _layer(w, fused=fused, gather=gather)
    bias0 = t["bias"].clone()
    out = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
    layer.bias_update(t["bias"], w.gamma)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    b_host = bias0.cpu().numpy()
    off = mi.host_logit_offset(w)
    x_bits = host_bf16_bits(t["x"])
    # routing of every token
    if check_all_routing:
        ref = oracle.route_workload(w, b_host, logit_offset=off, x=x_bits)
        same = check_routing(layer.topk_idx.cpu().numpy(), layer.gates.cpu().numpy().astype(np.float64),
                             layer.counts.cpu().numpy(), ref, w.k, w.n_routed, w.n_shared, w.gate_scale)
        # the bias update, bit-exact whenever the counts agree with the oracle's
        ref_counts = oracle.load_counts(ref["topk_idx"], w.n_routed)
        if (layer.counts.cpu().numpy() == ref_counts).all():
            nb = oracle.bias_update(ref_counts, b_host, w.T, w.k, w.gamma)
            np.testing.assert_array_equal(t["bias"].cpu().numpy().view(np.uint32), nb.view(np.uint32))
    _check_dispatch_properties(layer, x_bits, w.T, w.k, w.n_routed)
    if callable(expert_groups):  # chosen from the routed counts
        expert_groups = expert_groups(layer.counts.cpu().numpy())
    if expert_groups is not None:
        _check_expert_groups(w, layer, t, x_bits, expert_groups, shared_tokens)
    # layer output on the sampled tokens
    if tokens is None:
        tokens = np.arange(w.T)
    r = oracle.forward_tokens(w, tokens, b_host, off)
    gpu_idx = layer.topk_idx.cpu().numpy()[tokens]
    same_t = np.array([set(a) == set(b) for a, b in zip(gpu_idx, r["topk_idx"])])
    assert same_t.mean() > 0.9
    got = host_bf16_f64(out[torch.from_numpy(tokens).cuda()])
    return check_output(got[same_t], r["out"][same_t], name)


def test_layer_tiny_all_tokens():
    _run_and_check("tiny")


def test_layer_tiny_two_streams():
    """The shared experts on a second stream (two moe_grouped_ffn calls) instead of the fused launch."""
    _run_and_check("tiny", fused=False)


def test_layer_tiny_gathered_rows():
    """Fused experts gathering the routed rows from x (TMA row gathers) instead of reading copied rows."""
    _run_and_check("tiny", gather=True)


@pytest.mark.slow
def test_layer_mid_gathered_rows():
    _run_and_check("mid", tokens=np.arange(0, 4096, 97), gather=True)


@pytest.mark.slow
def test_layer_mid_sampled():
    _run_and_check("mid", tokens=np.arange(0, 4096, 37))


@pytest.mark.slow
def test_layer_decode_sampled():
    _run_and_check("decode", tokens=np.arange(0, 64, 5))


@pytest.mark.slow
def test_layer_prefill_full_routing_and_groups():
    """Prefill size (65536 tokens, d 7168): every token's routing and gates, the counts
    and the bias update against the oracle; the complete row groups of the first, a
    middle and the last routed expert, and 512 tokens of both shared experts, from the
    full-size GEMM launches; the layer output on sampled tokens."""
    _run_and_check("prefill", tokens=np.array([0, 1, 4095, 30000, 65535]), expert_groups=[0, 128, 255],
                   shared_tokens=np.arange(65536 - 512, 65536))


def test_layer_inkling_decode_sampled():
    """The released configuration (SwiGLU experts, d 6144, d_ff 3072, route_scale 8) at decode scale."""
    _run_and_check("inkling_decode", tokens=np.arange(0, 64, 9))


@pytest.mark.slow
def test_layer_inkling_full_routing_and_groups():
    """The released configuration at prefill scale (65536 tokens, about 29 GB of expert
    weights): all tokens' routing (route_scale 8), counts and bias update; whole row
    groups of three routed experts and 256 tokens of the shared experts."""
    _run_and_check("inkling", tokens=np.array([0, 7, 40000, 65535]), expert_groups=[0, 131, 255],
                   shared_tokens=np.arange(0, 65536, 256))


@pytest.mark.slow
def test_layer_skew_sampled_and_bias_trajectory():
    """Skewed routing: full layer once on sampled tokens, then 20 rounds of
    route -> count -> bias update on the same tokens, compared per round with
    the oracle's own 20 rounds (routing with the exemption rule; b bit-exact
    while the counts agree)."""
    w = mi.WORKLOADS["skew"]

    def groups(counts):
        # the busiest expert, the smallest non-empty one, and two whose last 256-row tile holds at most 128
        # rows (run as half tiles at this size)
        nz = np.flatnonzero(counts)
        half = [int(e) for e in nz if 0 < counts[e] % 256 <= 128 and counts[e] > 256][:2]
        return sorted({int(np.argmax(counts)), int(nz[np.argmin(counts[nz])]), *half})

    _run_and_check("skew", tokens=np.arange(0, w.T, 509), expert_groups=groups,
                   shared_tokens=np.arange(0, w.T, 997))
    t, layer = _layer(w, with_weights=False)
    off = mi.host_logit_offset(w)
    x_bits = host_bf16_bits(t["x"])
    z = oracle.logits(x_bits, mi.host_wr(w))
    b_ref = mi.host_bias(w)
    agree = True
    maxvio = []
    s = w
    for it in range(w.bias_iters):
        moe.moe_router_topk(t["x"], t["w_r"], t["bias"], t["logit_offset"], s.T, s.d, s.n_routed, s.n_shared, s.k,
                            1.0, layer.topk_idx, layer.gates, layer.counts)
        torch.cuda.synchronize()
        ref = oracle.route(z, b_ref, s.k, s.n_routed, s.n_shared, off)
        check_routing(layer.topk_idx.cpu().numpy(), layer.gates.cpu().numpy().astype(np.float64),
                      layer.counts.cpu().numpy(), ref, s.k, s.n_routed, s.n_shared)
        ref_counts = oracle.load_counts(ref["topk_idx"], s.n_routed)
        agree = agree and bool((layer.counts.cpu().numpy() == ref_counts).all())
        moe.moe_bias_update(layer.counts, s.n_routed, s.T, s.k, s.gamma, t["bias"])
        b_ref = oracle.bias_update(ref_counts, b_ref, s.T, s.k, s.gamma)
        if agree:
            np.testing.assert_array_equal(t["bias"].cpu().numpy().view(np.uint32), b_ref.view(np.uint32))
        maxvio.append(ref_counts.max() / (s.k * s.T / s.n_routed) - 1)
    # the controller lowers the hottest expert's load (qualitative, §02e)
    assert maxvio[-1] < maxvio[0]


def test_layer_is_deterministic_and_writes_every_row():
    w = mi.WORKLOADS["tiny"]
    t, layer = _layer(w, gather=False)
    layer.out.fill_(float("nan"))
    layer.x_perm.fill_(float("nan"))
    o1 = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"]).clone()
    xp1 = layer.x_perm.clone()
    o2 = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"]).clone()
    torch.cuda.synchronize()
    assert not torch.isnan(o1.float()).any() and not torch.isnan(xp1.float()).any()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(xp1.view(torch.int16), layer.x_perm.view(torch.int16))


def test_layer_ragged_token_counts():
    """T not a multiple of any tile size, and T = 1."""
    for T in (1, 77, 300):
        w = mi.Workload("ragged", T, 256, 128, b_half_width=0.1)
        _run_and_check_w(w)


def _run_and_check_w(w):
    t, layer = _layer(w)
    out = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"])
    torch.cuda.synchronize()
    b = t["bias"].cpu().numpy()
    r = oracle.forward_tokens(w, np.arange(w.T), b)
    same = check_routing(layer.topk_idx.cpu().numpy(), layer.gates.cpu().numpy().astype(np.float64),
                         layer.counts.cpu().numpy(), r, w.k, w.n_routed, w.n_shared)
    check_output(host_bf16_f64(out)[same], r["out"][same], w.name)


def test_layer_identical_experts_give_that_expert():
    """All 258 experts equal: out = E(x) whatever the routing."""
    w = mi.WORKLOADS["tiny"]
    t, layer = _layer(w)
    t["w1"][:] = t["w1"][0]
    t["w2"][:] = t["w2"][0]
    out = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"])
    ref = oracle.expert(mi.host_x(w), mi.host_w1(w, 0), mi.host_w2(w, 0))
    check_output(host_bf16_f64(out), ref, "identical experts")


def test_layer_step_replays_as_cuda_graph():
    """The whole step (router -> ... -> combine -> bias update) captured as one CUDA graph
    replays bit-identically to the eager calls (no host work, allocation or sync inside)."""
    w = mi.WORKLOADS["tiny"]
    t, layer = _layer(w)
    b0 = t["bias"].clone()
    outs = []
    for _ in range(2):
        layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
        layer.bias_update(t["bias"], w.gamma)
        outs.append((layer.out.clone(), t["bias"].clone()))
    torch.cuda.synchronize()
    t["bias"].copy_(b0)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
        layer.bias_update(t["bias"], w.gamma)
    t["bias"].copy_(b0)  # capture ran nothing; start the replays from the same bias
    for out, bias in outs:
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(layer.out, out)
        assert torch.equal(t["bias"], bias)
    assert moe.moe_get_status() == 0
