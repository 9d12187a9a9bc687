"""Pins of the oracle's NVFP4 quantization ("Under the hood", "Quantization: BF16
vs NVFP4": FP4 weights and activations, blocks of 16, FP8 block scales) to the
OCP Microscaling format definitions, a library FP8 conversion, exact round
trips and error bounds (no GPU)."""
import numpy as np
import pytest

import moe_inputs as mi
from oracle import nvfp4

torch = pytest.importorskip("torch")


def test_e2m1_table_and_round_trip():
    mags = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    np.testing.assert_array_equal(nvfp4.e2m1_decode(np.arange(8)), mags)
    np.testing.assert_array_equal(nvfp4.e2m1_decode(np.arange(8, 16)), [-m for m in mags])
    codes = np.arange(16)
    back = nvfp4.e2m1_encode(nvfp4.e2m1_decode(codes))
    np.testing.assert_array_equal(back, np.where(codes == 8, 0, codes))   # -0 is written as +0


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.2500001, 1), (0.75, 2), (0.7499, 1), (1.25, 2), (1.2501, 3), (1.75, 4), (2.5, 4), (2.51, 5),
    (3.5, 6), (3.49, 5), (5.0, 6), (5.01, 7), (6.0, 7), (7.0, 7), (1e30, 7), (-0.1, 0), (-0.3, 9), (-5.0, 14),
    (-9.0, 15),
])
def test_e2m1_ties_to_even_and_saturation(v, code):
    assert int(nvfp4.e2m1_encode(np.array([v]))[0]) == code


def test_e4m3_known_codes():
    np.testing.assert_array_equal(nvfp4.e4m3_decode(np.array([0x38, 0x7E, 0x01, 0x08, 0x07, 0x77, 0x00])),
                                  [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, 0.875 * 2.0 ** -6, 240.0, 0.0])


def test_e4m3_encoder_matches_torch_float8_cast():
    """Round to nearest even on the E4M3 grid, against torch's float8_e4m3fn conversion:
    a dense log-spaced sweep plus every exact midpoint between neighbouring values."""
    table = nvfp4.e4m3_decode(np.arange(127))
    mids = (table[:-1] + table[1:]) / 2
    v = np.concatenate([np.geomspace(2.0 ** -12, 448.0, 20001), mids, table, [0.0, 2.0 ** -11, 447.9]])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(nvfp4.e4m3_encode_nonneg(v32), ref)
    assert int(nvfp4.e4m3_encode_nonneg(np.array([1e9]))[0]) == 0x7E       # saturates


def test_activation_round_trip_of_representable_blocks():
    """Blocks built from E2M1 codes times an E4M3 scale, with a block maximum of
    magnitude 6, are quantized back to exactly those codes and scales."""
    rng_codes = mi.words(64 * 64, 3, mi.STREAM_TEST_ROWS) % 16
    q = rng_codes.reshape(64, 64).astype(np.uint8)
    q[:, ::16] = 7                                          # every block holds a +6
    s = (mi.words(64 * 4, 4, mi.STREAM_TEST_ROWS) % 100 + 20).reshape(64, 4).astype(np.uint8)
    x = nvfp4.dequantize(q, s).astype(np.float32)
    q2, s2 = nvfp4.quantize_activation(x)
    np.testing.assert_array_equal(s2, s)
    np.testing.assert_array_equal(nvfp4.e2m1_decode(q2), nvfp4.e2m1_decode(q))


def test_weight_round_trip_with_tensor_scale():
    q = (mi.words(32 * 128, 5, mi.STREAM_TEST_ROWS) % 16).reshape(32, 128).astype(np.uint8)
    q[:, ::16] = 7
    s = (mi.words(32 * 8, 6, mi.STREAM_TEST_ROWS) % 90 + 30).reshape(32, 8).astype(np.uint8)
    s[0, 0] = 0x7E                                          # the matrix maximum uses the largest scale
    g = 2.0 ** -10
    w = nvfp4.dequantize(q, s, g).astype(np.float32)
    q2, s2, g2 = nvfp4.quantize_weight(w)
    assert g2 == np.float32(g)
    np.testing.assert_array_equal(s2, s)
    np.testing.assert_array_equal(nvfp4.e2m1_decode(q2), nvfp4.e2m1_decode(q))


def test_activation_codes_are_nearest_grid_points():
    x = (mi.normal_f64(300 * 64, 7, mi.STREAM_TEST_ROWS).reshape(300, 64) * 3).astype(np.float32)
    q, s = nvfp4.quantize_activation(x)
    sd = nvfp4.e4m3_decode(s)
    r = x.reshape(300, 4, 16) / sd[..., None]
    got = nvfp4.e2m1_decode(q).reshape(300, 4, 16)
    grid = np.concatenate([-nvfp4.E2M1_MAGNITUDE[::-1], nvfp4.E2M1_MAGNITUDE])
    best = np.abs(r[..., None] - grid).min(axis=-1)
    assert (np.abs(r - got) <= best + 1e-6).all()
    # the block scale is amax/6 to within E4M3's half-step (relative 1/16), so the block maximum maps to 4 or 6
    amax = np.abs(x.reshape(300, 4, 16)).max(axis=-1)
    np.testing.assert_allclose(sd, amax / 6, rtol=1 / 16 + 1e-7)
    assert set(np.unique(np.abs(got).max(axis=-1))) <= {4.0, 6.0}


def _tie_blocks():
    """Blocks whose quotients x / s are exact E2M1 midpoints.  Each block's first
    value is 6 s, so its scale is s = E4M3(6 s / 6); the others are m s for the
    midpoints m in {1.25, 2.5, 5}, which round to the lower, even code (1, 2, 4).
    With s = 15/16 * 2^e the fp32 reciprocal of s is inexact, and m s times it
    rounds to just above m, which would give the upper code."""
    scales = [0.9375 * 2.0 ** e for e in (-5, -2, 0, 1, 3)]
    blocks = []
    for s in scales:
        b = np.zeros(16, dtype=np.float64)
        b[0] = 6 * s
        b[1:4] = [1.25 * s, 2.5 * s, 5 * s]
        b[4:7] = [-1.25 * s, -2.5 * s, -5 * s]
        b[7:10] = [0.25 * s, 1.75 * s, 3.5 * s]      # ties that go up (0.75, 1.75, 3.5) or to 0
        b[10] = 0.75 * s
        blocks.append(b)
    return np.array(scales), np.array(blocks).astype(np.float32)


TIE_CODES = [7, 2, 4, 6, 10, 12, 14, 0, 4, 6, 2, 0, 0, 0, 0, 0]


def test_codes_are_rounded_quotients_at_exact_ties():
    """A code is the E2M1 rounding (ties to even) of the exact quotient x / s: at a
    midpoint the even code wins.  Checked on blocks where a product with the fp32
    reciprocal of s lands just past the midpoint."""
    scales, x = _tie_blocks()
    inv = (np.float32(1) / scales.astype(np.float32)).astype(np.float32)
    assert (((x[:, 1] * inv).astype(np.float32)) > np.float32(1.25)).all()   # the reciprocal form would round up
    q, s = nvfp4.quantize_activation(x)
    np.testing.assert_array_equal(nvfp4.e4m3_decode(s)[:, 0], scales)
    np.testing.assert_array_equal(q, np.tile(TIE_CODES, (len(scales), 1)))
    # weights: the same blocks with a power-of-two tensor scale (the quotient is unchanged)
    w = np.concatenate([x, np.full((1, 16), 448 * 6 * 2.0 ** -4, np.float32)])
    qw, sw, g = nvfp4.quantize_weight(w)
    assert g == np.float32(2.0 ** -4)
    np.testing.assert_array_equal(qw[:-1], np.tile(TIE_CODES, (len(scales), 1)))


def test_codes_equal_fp64_quotients_rounded_to_fp32():
    """The fp32 quotient equals the fp64 quotient of the same fp32 operands rounded
    to fp32 (a correctly rounded division, by the double-rounding bound for
    division); the codes then follow from the E2M1 rounding of that value."""
    x = (mi.normal_f64(500 * 64, 9, mi.STREAM_TEST_ROWS).reshape(500, 64) * 2).astype(np.float32)
    q, s = nvfp4.quantize_activation(x)
    sd = nvfp4.e4m3_decode(s)
    r = (x.reshape(500, 4, 16).astype(np.float64) / sd[..., None]).astype(np.float32)
    np.testing.assert_array_equal(q.reshape(500, 4, 16), np.where(sd[..., None] > 0, nvfp4.e2m1_encode(r), 0))
    w = (mi.normal_f64(64 * 256, 10, mi.STREAM_TEST_ROWS).reshape(64, 256) * 0.02).astype(np.float32)
    qw, sw, g = nvfp4.quantize_weight(w)
    den = (nvfp4.e4m3_decode(sw).astype(np.float32) * g).astype(np.float32)
    rw = (w.reshape(64, 16, 16).astype(np.float64) / den[..., None]).astype(np.float32)
    np.testing.assert_array_equal(qw.reshape(64, 16, 16), np.where(den[..., None] > 0, nvfp4.e2m1_encode(rw), 0))


def test_scale_invariance_by_powers_of_two():
    x = (mi.normal_f64(40 * 32, 8, mi.STREAM_TEST_ROWS).reshape(40, 32)).astype(np.float32)
    q, s = nvfp4.quantize_activation(x)
    q4, s4 = nvfp4.quantize_activation(x * np.float32(4))
    np.testing.assert_array_equal(q4, q)
    np.testing.assert_array_equal(s4.astype(int), s.astype(int) + 2 * 8)   # exponent field + 2


def test_gemm_orientation():
    """dq(A) dq(B)^T with B = c * identity reproduces c * dq(A): the weight rows
    are the output features (a transposed operand fails).  c = 6 * 448 * 2^-10, so
    the tensor scale is a power of two and c is exact."""
    K = 64
    x = mi.normal_f64(10 * K, 9, mi.STREAM_TEST_ROWS).reshape(10, K).astype(np.float32)
    xq, xs = nvfp4.quantize_activation(x)
    w = np.zeros((48, K), np.float32)
    c = 6 * 448 * 2.0 ** -10
    w[np.arange(48), np.arange(48)] = c                     # 48 outputs read the first 48 inputs
    wq, ws, g = nvfp4.quantize_weight(w)
    assert g == np.float32(2.0 ** -10)
    np.testing.assert_allclose(nvfp4.gemm(xq, xs, wq, ws, g), c * nvfp4.dequantize(xq, xs)[:, :48],
                               rtol=1e-14, atol=0)


def test_layer_composition_with_identical_experts():
    """All routed experts equal (and both shared experts equal): every routed
    contributor gives the same NVFP4 expert output Y4 and every shared one the same
    bf16 output Y, so out = (sum of routed gates) * Y4 + (sum of shared gates) * Y."""
    import oracle

    w = mi.Workload("pin", 12, 256, 256, b_half_width=0.1)
    tokens = np.arange(12)
    w1r, w2r = mi.host_w1(w, 3), mi.host_w2(w, 3)
    w1s, w2s = mi.host_w1(w, 256), mi.host_w2(w, 256)

    import moe_inputs

    orig = (moe_inputs.host_w1, moe_inputs.host_w2)
    try:
        moe_inputs.host_w1 = lambda ww, e: w1r if e < ww.n_routed else w1s
        moe_inputs.host_w2 = lambda ww, e: w2r if e < ww.n_routed else w2s
        bias = mi.host_bias(w)
        r = nvfp4.forward_tokens(w, tokens, bias)
    finally:
        moe_inputs.host_w1, moe_inputs.host_w2 = orig
    x = mi.host_x(w, tokens)
    wq1 = nvfp4.quantize_weight(mi.bf16_to_f64(w1r).astype(np.float32))
    wq2 = nvfp4.quantize_weight(mi.bf16_to_f64(w2r).astype(np.float32))
    y4 = nvfp4.expert(mi.bf16_to_f64(x).astype(np.float32), wq1, wq2)["y"]
    ybf = oracle.expert(x, w1s, w2s)
    g = r["gates"]
    expect = g[:, :w.k].sum(axis=1, keepdims=True) * y4 + g[:, w.k:].sum(axis=1, keepdims=True) * ybf
    np.testing.assert_allclose(r["out"], expect, rtol=1e-12, atol=1e-12)


def test_swiglu_expert_special_case():
    """Representable operands: x a block of +-3 and +-2, Wg = c * I and Wu = c/4 * I (c = 6 * 448 *
    2^-10, so the tensor scale is a power of two), W2 = c * I: the hidden layer is
    silu(c x) * (c x / 4) exactly before its own quantization (the gate rows come first: swapped
    halves give silu(c x / 4) * c x), and y = c * dq(quantize(h))."""
    from scipy.special import expit

    d = 64
    x = np.tile(np.array([6.0, -4.0, 4.0, -6.0] * 4, np.float32), (3, 4))[:, :d] * np.float32(0.5)
    c = 6 * 448 * 2.0 ** -10
    eye = np.eye(d, dtype=np.float32) * np.float32(c)
    w1 = nvfp4.quantize_weight(np.concatenate([eye, eye / np.float32(4)]))
    assert w1[2] == np.float32(2.0 ** -10)
    w2 = nvfp4.quantize_weight(eye)
    r = nvfp4.expert_swiglu(x, w1, w2)
    z = c * x.astype(np.float64)
    h = z * expit(z) * (z / 4)
    np.testing.assert_allclose(r["h"], h, rtol=1e-12)
    hq, hs = nvfp4.quantize_activation(h.astype(np.float32))
    np.testing.assert_allclose(r["y"], c * nvfp4.dequantize(hq, hs), rtol=1e-12)
