"""NVFP4 routed experts on the GPU ("Under the hood", "Quantization: BF16 vs
NVFP4": FP4 weights and activations, blocks of 16, FP8 scales) against the
oracle: weight and activation quantization bit-exact, the block-scaled grouped
GEMM on the oracle's quantized operands, and the layer with NVFP4 experts."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from oracle import nvfp4
from parity import check_output, check_routing, dev_bf16, host_bf16_bits, host_bf16_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if torch.cuda.is_available():
    import sparse_moe_layer_joint_b200 as moe


# the documented device layouts, written out for the tests
def _unpack_codes(b):
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 15
    out[..., 1::2] = b >> 4
    return out


def _pack_codes(c):
    c = np.asarray(c, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def _sf_index(R, K):
    r = np.arange(R)[:, None]
    b = np.arange(K // 16)[None, :]
    return (((r // 128) * (K // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4)


def _sf_logical(buf, R, K):
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[_sf_index(R, K)]


def _sf_tiled(s, R, K):
    out = np.zeros(R * K // 16, dtype=np.uint8)
    out[_sf_index(R, K)] = s
    return out


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("G,N,K,std", [(3, 256, 512, 0.05), (2, 128, 256, 30.0), (1, 384, 768, 1e-3)])
def test_quantize_weights_bit_exact(G, N, K, std):
    w = mi.normal_bf16(G * N * K, 21, mi.STREAM_W1, std=std).reshape(G, N, K)
    if G > 1:
        w[1] = 0                                              # an all-zero matrix: g = 0, codes 0
    q = torch.empty((G, N, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((G, N * K // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(G, dtype=torch.float32, device="cuda")
    moe.moe_nvfp4_quantize_weights(dev_bf16(w), G, N, K, q, sf, g)
    assert moe.moe_get_status() == 0
    qh, sfh, gh = q.cpu().numpy(), sf.cpu().numpy(), g.cpu().numpy()
    for i in range(G):
        rq, rs, rg = nvfp4.quantize_weight(mi.bf16_to_f64(w[i]).astype(np.float32))
        assert gh[i] == rg
        np.testing.assert_array_equal(_unpack_codes(qh[i]), rq)
        np.testing.assert_array_equal(_sf_logical(sfh[i], N, K), rs)


def _dispatch(T, k, E, d, seed, cap=None):
    x = mi.normal_bf16(T * d, seed, mi.STREAM_X).reshape(T, d)
    u = mi.words(T * E, seed, mi.STREAM_TEST_TOPK).reshape(T, E).astype(np.float64)
    topk = np.argsort(-(u - 2e9 * np.log1p(np.arange(E))[None, :] / 10), axis=1, kind="stable")[:, :k].astype(np.int32)
    keep = oracle.capacity_keep(topk, cap, E) if cap is not None else None
    dp = oracle.dispatch(topk, E, keep)
    rows_cap = moe.moe_nvfp4_rows_capacity(T, E, k)
    xq = torch.zeros((rows_cap, d // 2), dtype=torch.uint8, device="cuda")
    xsf = torch.zeros((rows_cap * d // 16,), dtype=torch.uint8, device="cuda")
    trp = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    offp = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    moe.moe_nvfp4_dispatch(dev_bf16(x), _i32(topk), _i32(dp["token_row"]), _i32(dp["offsets"]), T, d, E, k, xq, xsf,
                           trp, offp)
    assert moe.moe_get_status() == 0
    return x, topk, dp, rows_cap, xq, xsf, trp, offp


@pytest.mark.parametrize("T,k,E,d,cap", [(300, 6, 16, 512, None), (1, 6, 256, 256, None), (1000, 2, 64, 768, 40),
                                         (513, 8, 8, 256, None)])
def test_dispatch_quant_bit_exact(T, k, E, d, cap):
    x, topk, dp, rows_cap, xq, xsf, trp, offp = _dispatch(T, k, E, d, T + E, cap)
    counts = np.diff(dp["offsets"])
    off_pad = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)])
    np.testing.assert_array_equal(offp.cpu().numpy(), off_pad)
    # the padded row of (t, j): same place in its expert's rows as in the unpadded layout
    tr = dp["token_row"]
    e_of = topk.astype(np.int64)
    expect = np.where(tr >= 0, tr - dp["offsets"][e_of] + off_pad[e_of], -1)
    np.testing.assert_array_equal(trp.cpu().numpy(), expect)
    q_ref, s_ref = nvfp4.quantize_activation(mi.bf16_to_f64(x).astype(np.float32))
    codes = _unpack_codes(xq.cpu().numpy())
    sfs = _sf_logical(xsf.cpu().numpy(), rows_cap, d)
    t_idx, j_idx = np.nonzero(expect >= 0)
    rows = expect[t_idx, j_idx]
    np.testing.assert_array_equal(codes[rows], q_ref[t_idx])
    np.testing.assert_array_equal(sfs[rows], s_ref[t_idx])


def _tie_rows(n_rows, K):
    """Rows of K values made of blocks whose quotients x / s are exact E2M1 midpoints
    (bf16-exact; see the oracle pin of the same name): scales 15/16 * 2^e."""
    out = np.zeros((n_rows, K), dtype=np.float32)
    for r in range(n_rows):
        for b in range(K // 16):
            s = 0.9375 * 2.0 ** ((r + 3 * b) % 9 - 5)
            v = np.array([6, 1.25, 2.5, 5, -1.25, -2.5, -5, 0.25, 1.75, 3.5, 0.75, 0, 0, 0, 0, 0]) * s
            out[r, 16 * b:16 * b + 16] = np.roll(v, (r + b) % 16)
    bits = out.view(np.uint32)
    assert ((bits & 0xFFFF) == 0).all()                      # every value is a bf16
    return (bits >> 16).astype(np.uint16)


def test_quantize_at_exact_ties_divides():
    """Weights and the FP4 dispatch on blocks whose values over their scale are exact
    E2M1 midpoints: the codes are the even ones, as the oracle's division gives."""
    N, K = 128, 256
    w = _tie_rows(N, K)
    w[5, 7] = np.uint16(np.float32(448 * 6 * 2.0 ** -4).view(np.uint32) >> 16)   # g = 2^-4
    q = torch.empty((1, N, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((1, N * K // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    moe.moe_nvfp4_quantize_weights(dev_bf16(w[None]), 1, N, K, q, sf, g)
    assert moe.moe_get_status() == 0
    rq, rs, rg = nvfp4.quantize_weight(mi.bf16_to_f64(w).astype(np.float32))
    assert g.cpu().numpy()[0] == rg
    np.testing.assert_array_equal(_unpack_codes(q.cpu().numpy()[0]), rq)
    np.testing.assert_array_equal(_sf_logical(sf.cpu().numpy()[0], N, K), rs)

    T, k, E = 64, 2, 4
    x = _tie_rows(T, K)
    topk = np.stack([np.arange(T) % E, (np.arange(T) + 1) % E], axis=1).astype(np.int32)
    dp = oracle.dispatch(topk, E)
    rows_cap = moe.moe_nvfp4_rows_capacity(T, E, k)
    xq = torch.zeros((rows_cap, K // 2), dtype=torch.uint8, device="cuda")
    xsf = torch.zeros((rows_cap * K // 16,), dtype=torch.uint8, device="cuda")
    trp = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    offp = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    moe.moe_nvfp4_dispatch(dev_bf16(x), _i32(topk), _i32(dp["token_row"]), _i32(dp["offsets"]), T, K, E, k, xq, xsf,
                           trp, offp)
    assert moe.moe_get_status() == 0
    q_ref, s_ref = nvfp4.quantize_activation(mi.bf16_to_f64(x).astype(np.float32))
    rows = trp.cpu().numpy()
    codes = _unpack_codes(xq.cpu().numpy())
    sfs = _sf_logical(xsf.cpu().numpy(), rows_cap, K)
    for j in range(k):
        np.testing.assert_array_equal(codes[rows[:, j]], q_ref)
        np.testing.assert_array_equal(sfs[rows[:, j]], s_ref)


@pytest.fixture(params=["tn128", "tn256", "pair128", "pair256"])
def fp4_tile(request, monkeypatch):
    """Every FP4 GEMM tile, each forced: one CTA per 128 x 128 or 128 x 256 tile (256 where N is a
    multiple of 256, the default for short groups), a CTA pair per 256 x 128 or 256 x 256 tile (the
    default for long groups)."""
    monkeypatch.setenv("MOE_FP4_TN", request.param[-3:])
    monkeypatch.setenv("MOE_FP4_PAIR", "1" if request.param.startswith("pair") else "0")
    return request.param


def _gemm_inputs(sizes, N, K, seed):
    """A (activations) and W quantized by the oracle, laid out as the device expects."""
    G = len(sizes)
    off_pad = np.concatenate([[0], np.cumsum([(n + 127) // 128 * 128 for n in sizes])]).astype(np.int32)
    rows_cap = max(int(off_pad[-1]), 128)
    a = (mi.normal_f64(rows_cap * K, seed, mi.STREAM_TEST_ROWS).reshape(rows_cap, K)).astype(np.float32)
    aq, as_ = nvfp4.quantize_activation(a)
    w = mi.normal_bf16(G * N * K, seed, mi.STREAM_W1, std=K ** -0.5).reshape(G, N, K)
    wq = [nvfp4.quantize_weight(mi.bf16_to_f64(w[g]).astype(np.float32)) for g in range(G)]
    dev = {
        "aq": _u8(_pack_codes(aq)), "asf": _u8(_sf_tiled(as_, rows_cap, K)), "off_pad": _i32(off_pad),
        "wq": _u8(np.stack([_pack_codes(q) for q, _, _ in wq])),
        "wsf": _u8(np.stack([_sf_tiled(s, N, K) for _, s, _ in wq])),
        "g": torch.tensor([gg for _, _, gg in wq], dtype=torch.float32, device="cuda"),
    }
    return aq, as_, wq, off_pad, rows_cap, dev


@pytest.mark.parametrize("sizes,N,K", [([130, 0, 1, 300], 256, 512), ([128] * 3, 128, 256), ([700], 384, 1024),
                                       ([5, 260, 17, 0, 129, 64, 1, 1], 128, 768)])
def test_gemm_bf16_out_matches_oracle(sizes, N, K, fp4_tile):
    aq, as_, wq, off_pad, rows_cap, dev = _gemm_inputs(sizes, N, K, len(sizes) + N)
    G = len(sizes)
    # unpadded output rows through offsets_out
    off_out = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(off_out[-1])
    out = torch.full((max(R, 1), N), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_nvfp4_grouped_gemm(dev["aq"], dev["asf"], dev["off_pad"], G, rows_cap, dev["wq"], dev["wsf"], dev["g"],
                               N, K, moe.MOE_NVFP4_EPI_BF16, None, None, out, _i32(off_out), R)
    assert moe.moe_get_status() == 0
    got = host_bf16_f64(out)
    for g in range(G):
        if sizes[g] == 0:
            continue
        a0 = off_pad[g]
        ref = nvfp4.gemm(aq[a0:a0 + sizes[g]], as_[a0:a0 + sizes[g]], *wq[g])
        check_output(got[off_out[g]:off_out[g + 1]], ref, f"group {g}")
        np.testing.assert_allclose(got[off_out[g]:off_out[g + 1]], ref, rtol=2 ** -7, atol=1e-3 * np.abs(ref).max())


@pytest.mark.parametrize("sizes,real_rows", [([300, 77, 128], False), ([1, 5, 33, 64, 100, 129, 0, 2], True)])
def test_gemm_gelu_fp4_out_matches_oracle(sizes, real_rows, fp4_tile):
    """GEMM1's epilogue: g * acc, GELU, FP4 re-quantization.  The codes decide on
    fp32 values that differ from the oracle's by the accumulation order, so a code
    or scale may sit on the other side of a rounding boundary: at most 0.1% may
    differ, and the dequantized hidden rows agree to the usual tolerance.  With the
    groups' real row counts given, only those rows are loaded (padding rows are
    then not meaningful and not compared)."""
    N, K = 512, 768
    aq, as_, wq, off_pad, rows_cap, dev = _gemm_inputs(sizes, N, K, 5)
    G = len(sizes)
    hq = torch.zeros((rows_cap, N // 2), dtype=torch.uint8, device="cuda")
    hsf = torch.zeros((rows_cap * N // 16,), dtype=torch.uint8, device="cuda")
    off_real = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    moe.moe_nvfp4_grouped_gemm(dev["aq"], dev["asf"], dev["off_pad"], G, rows_cap, dev["wq"], dev["wsf"], dev["g"],
                               N, K, moe.MOE_NVFP4_EPI_GELU_FP4, hq, hsf, None,
                               _i32(off_real) if real_rows else None, int(off_real[-1]) if real_rows else 0)
    assert moe.moe_get_status() == 0
    codes = _unpack_codes(hq.cpu().numpy())
    sfs = _sf_logical(hsf.cpu().numpy(), rows_cap, N)
    n_code = n_sf = 0
    for g in range(G):
        a0, n = off_pad[g], sizes[g]
        pre = nvfp4.gemm(aq[a0:a0 + n], as_[a0:a0 + n], *wq[g])
        h = oracle.gelu_tanh(pre)
        rq, rs = nvfp4.quantize_activation(h.astype(np.float32))
        n_code += int((codes[a0:a0 + n] != rq).sum())
        n_sf += int((sfs[a0:a0 + n] != rs).sum())
        check_output(nvfp4.dequantize(codes[a0:a0 + n], sfs[a0:a0 + n]), nvfp4.dequantize(rq, rs), f"h {g}")
    total = sum(sizes) * N
    assert n_code <= 1e-3 * total and n_sf <= 1e-3 * total / 16, (n_code, n_sf)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_gemm_swiglu_fp4_out_matches_oracle(pair, monkeypatch):
    """The SwiGLU first GEMM: gate and up rows of one quantized W1 [2N, K] side by side in a
    256-wide tile (on a CTA pair: the gate rows in one CTA, the up rows in the other),
    silu(g * gate) * (g * up), FP4 out; the same acceptance as the GELU epilogue."""
    monkeypatch.setenv("MOE_FP4_PAIR", pair)
    sizes, N, K = [1, 77, 128, 300], 256, 512
    G = len(sizes)
    off_pad = np.concatenate([[0], np.cumsum([(n + 127) // 128 * 128 for n in sizes])]).astype(np.int32)
    rows_cap = int(off_pad[-1])
    a = (mi.normal_f64(rows_cap * K, 31, mi.STREAM_TEST_ROWS).reshape(rows_cap, K)).astype(np.float32)
    aq, as_ = nvfp4.quantize_activation(a)
    w = mi.normal_bf16(G * 2 * N * K, 31, mi.STREAM_W1, std=K ** -0.5).reshape(G, 2 * N, K)
    wq = [nvfp4.quantize_weight(mi.bf16_to_f64(w[g]).astype(np.float32)) for g in range(G)]
    hq = torch.zeros((rows_cap, N // 2), dtype=torch.uint8, device="cuda")
    hsf = torch.zeros((rows_cap * N // 16,), dtype=torch.uint8, device="cuda")
    off_real = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    moe.moe_nvfp4_grouped_gemm(_u8(_pack_codes(aq)), _u8(_sf_tiled(as_, rows_cap, K)), _i32(off_pad), G, rows_cap,
                               _u8(np.stack([_pack_codes(q) for q, _, _ in wq])),
                               _u8(np.stack([_sf_tiled(s, 2 * N, K) for _, s, _ in wq])),
                               torch.tensor([gg for _, _, gg in wq], dtype=torch.float32, device="cuda"), N, K,
                               moe.MOE_NVFP4_EPI_SWIGLU_FP4, hq, hsf, None, _i32(off_real), int(off_real[-1]))
    assert moe.moe_get_status() == 0
    codes = _unpack_codes(hq.cpu().numpy())
    sfs = _sf_logical(hsf.cpu().numpy(), rows_cap, N)
    n_code = n_sf = 0
    for g in range(G):
        a0, n = off_pad[g], sizes[g]
        pre = nvfp4.gemm(aq[a0:a0 + n], as_[a0:a0 + n], *wq[g])
        gate, up = pre[:, :N], pre[:, N:]
        h = gate / (1.0 + np.exp(-gate)) * up
        rq, rs = nvfp4.quantize_activation(h.astype(np.float32))
        n_code += int((codes[a0:a0 + n] != rq).sum())
        n_sf += int((sfs[a0:a0 + n] != rs).sum())
        check_output(nvfp4.dequantize(codes[a0:a0 + n], sfs[a0:a0 + n]), nvfp4.dequantize(rq, rs), f"h {g}")
    total = sum(sizes) * N
    assert n_code <= 1e-3 * total and n_sf <= 1e-3 * total / 16, (n_code, n_sf)


def _nvfp4_expert_groups(w, layer, t, experts):
    """Whole row groups of the NVFP4 expert GEMMs at full size: every y_perm row of each listed expert
    (its ragged last tile included) against the NVFP4 oracle's expert on the token that row holds.  The
    hidden layer's FP4 codes decide on fp32 sums in a different order, so a few codes may sit on the
    other side of a rounding boundary; the rows meet the usual output bar."""
    off = layer.offsets.cpu().numpy().astype(np.int64)
    rt = layer.row_token.cpu().numpy()
    x_bits = host_bf16_bits(t["x"])
    fn = nvfp4.expert_swiglu if w.activation == "swiglu" else nvfp4.expert
    for e in experts:
        lo, hi = int(off[e]), int(off[e + 1])
        assert hi > lo
        w1 = nvfp4.quantize_weight(mi.bf16_to_f64(host_bf16_bits(t["w1"][e])).astype(np.float32))
        w2 = nvfp4.quantize_weight(mi.bf16_to_f64(host_bf16_bits(t["w2"][e])).astype(np.float32))
        ref = fn(mi.bf16_to_f64(x_bits[rt[lo:hi]]).astype(np.float32), w1, w2)["y"]
        check_output(host_bf16_f64(layer.y_perm[lo:hi]), ref, f"{w.name} nvfp4 expert {e} rows {lo}..{hi}")


def _nvfp4_layer(name, tokens, cap=None, expert_groups=None):
    w = mi.WORKLOADS[name]
    t = mi.torch_workload(w)
    layer = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f, w.n_routed, w.n_shared, w.k), precision="nvfp4",
                         capacity_factor=cap, activation=w.activation, route_scale=w.gate_scale)
    layer.set_nvfp4_weights(t["w1"], t["w2"])
    b_host = t["bias"].cpu().numpy()
    out = layer.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"], t["logit_offset"])
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    if expert_groups is not None:
        _nvfp4_expert_groups(w, layer, t, expert_groups)
    gpu_idx = layer.topk_idx.cpu().numpy()
    keep = None
    if cap is not None:
        keep = oracle.capacity_keep(gpu_idx, layer.capacity, w.n_routed)[tokens]
    r = nvfp4.forward_tokens(w, tokens, b_host, keep=keep)
    same = np.array([list(a) == list(b) for a, b in zip(gpu_idx[tokens], r["topk_idx"])])
    assert same.mean() > 0.8
    got = host_bf16_f64(out[torch.from_numpy(np.asarray(tokens)).cuda()])
    check_output(got[same], r["out"][same], f"{name} nvfp4")
    # the cost of the format: the bf16 layer's output on the same tokens, for the record
    ref_bf16 = oracle.forward_tokens(w, tokens, b_host, mi.host_logit_offset(w), keep=keep)["out"]
    rel = np.linalg.norm(got[same] - ref_bf16[same]) / np.linalg.norm(ref_bf16[same])
    assert rel < (0.4 if w.activation == "swiglu" else 0.25)   # two quantized projections multiply in SwiGLU
    return rel


def test_layer_nvfp4_mid_sampled():
    _nvfp4_layer("mid", np.arange(0, 4096, 211))


@pytest.mark.slow
def test_layer_nvfp4_decode_sampled():
    _nvfp4_layer("decode", np.array([0, 31, 63]))


@pytest.mark.slow
def test_layer_nvfp4_mid_with_capacity():
    _nvfp4_layer("mid", np.arange(0, 4096, 301), cap=1.0)


@pytest.mark.slow
def test_layer_nvfp4_prefill_sampled():
    """Full prefill size (65536 tokens, 256 experts of d 7168 / d_ff 2048) with NVFP4 experts: sampled
    tokens through the whole layer, and every row of the first, a middle and the last expert."""
    _nvfp4_layer("prefill", np.array([0, 40000, 65535]), expert_groups=[0, 128, 255])


def test_nvfp4_zero_tokens_and_empty_experts():
    """T = 0: the dispatch still writes the (all-zero) padded offsets; the GEMMs then have no tiles."""
    E, d, k = 16, 256, 2
    x = torch.zeros((1, d), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, k), dtype=torch.int32, device="cuda")
    off = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    xq = torch.zeros((128, d // 2), dtype=torch.uint8, device="cuda")
    xsf = torch.zeros((128 * d // 16,), dtype=torch.uint8, device="cuda")
    trp = torch.zeros((1, k), dtype=torch.int32, device="cuda")
    offp = torch.full((E + 1,), -3, dtype=torch.int32, device="cuda")
    moe.moe_nvfp4_dispatch(x, idx, idx, off, 0, d, E, k, xq, xsf, trp, offp)
    assert (offp.cpu().numpy() == 0).all()
    w = torch.zeros((E, 128, d), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((E, 128, d // 2), dtype=torch.uint8, device="cuda")
    wsf = torch.zeros((E, 128 * d // 16), dtype=torch.uint8, device="cuda")
    g = torch.zeros(E, dtype=torch.float32, device="cuda")
    moe.moe_nvfp4_quantize_weights(w, E, 128, d, wq, wsf, g)
    y = torch.full((1, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_nvfp4_grouped_gemm(xq, xsf, offp, E, 128, wq, wsf, g, 128, d, moe.MOE_NVFP4_EPI_BF16, None, None, y,
                               off, 0)
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    assert (y.float().cpu().numpy() == 7.0).all()      # nothing written
    assert (g.cpu().numpy() == 0).all()                 # all-zero weights: tensor scale 0


@pytest.mark.slow
def test_layer_nvfp4_inkling_decode_sampled():
    """The released configuration in NVFP4 (SwiGLU experts, route_scale 8) at decode scale."""
    _nvfp4_layer("inkling_decode", np.array([0, 40]))
