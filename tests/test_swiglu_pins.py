"""Pins of the oracle's gated (SwiGLU) expert and of the gate scale of the
released configuration ("Under the hood": SwiGLU experts of intermediate width
3072; routing weights scaled by route_scale times a learned global scale),
against library routines, special cases and invariants (no GPU)."""
import numpy as np
import pytest
from scipy.special import expit

import moe_inputs as mi
import oracle


def test_silu_is_u_times_logistic():
    u = np.concatenate([np.linspace(-40, 40, 4001), [0.0, 1e-300, -1e-300, 700.0, -700.0]])
    np.testing.assert_allclose(oracle.silu(u), u * expit(u), rtol=1e-14, atol=1e-300)


def test_swiglu_special_case_elementwise():
    """Wg = I, Wu = 2I, W2 = I (d = d_ff): y = silu(x) * 2x elementwise -- the gate
    branch carries the SiLU, the up branch is linear, so swapping them
    (silu(2x) * x) or dropping a branch fails."""
    d = 16
    x = mi.normal_f64(5 * d, 3, mi.STREAM_TEST_ROWS).reshape(5, d) * 2
    eye = np.eye(d)
    w1 = np.concatenate([eye, 2 * eye])
    y = oracle.expert_swiglu_f64(x, w1, eye)
    np.testing.assert_allclose(y, 2 * x * x * expit(x), rtol=1e-13, atol=1e-15)
    assert not np.allclose(y, x * 2 * x * expit(2 * x))


def test_swiglu_linear_in_up_and_down_and_zero_gate():
    d, f, n = 24, 40, 7
    x = mi.normal_f64(n * d, 4, mi.STREAM_TEST_ROWS).reshape(n, d)
    wg = mi.normal_f64(f * d, 4, mi.STREAM_W1).reshape(f, d) / np.sqrt(d)
    wu = mi.normal_f64(f * d, 5, mi.STREAM_W1).reshape(f, d) / np.sqrt(d)
    w2 = mi.normal_f64(d * f, 4, mi.STREAM_W2).reshape(d, f) / np.sqrt(f)
    y = oracle.expert_swiglu_f64(x, np.concatenate([wg, wu]), w2)
    np.testing.assert_allclose(oracle.expert_swiglu_f64(x, np.concatenate([wg, -3 * wu]), w2), -3 * y,
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.expert_swiglu_f64(x, np.concatenate([wg, wu]), 0.5 * w2), 0.5 * y,
                               rtol=1e-12, atol=1e-12)
    assert not oracle.expert_swiglu_f64(x, np.concatenate([np.zeros_like(wg), wu]), w2).any()
    # one hidden unit, one token: y = W2[:, j] * silu(g) * u with g, u the two dot products
    j = 11
    mask = np.zeros((f, 1))
    mask[j] = 1.0
    y1 = oracle.expert_swiglu_f64(x[:1], np.concatenate([wg * mask, wu * mask]), w2)
    g, u = float(wg[j] @ x[0]), float(wu[j] @ x[0])
    np.testing.assert_allclose(y1[0], w2[:, j] * g * expit(g) * u, rtol=1e-12, atol=1e-14)


def test_swiglu_bf16_entry_matches_f64_entry():
    d, f, n = 64, 96, 9
    x = mi.normal_bf16(n * d, 6, mi.STREAM_TEST_ROWS).reshape(n, d)
    w1 = mi.normal_bf16(2 * f * d, 6, mi.STREAM_W1, std=d ** -0.5).reshape(2 * f, d)
    w2 = mi.normal_bf16(d * f, 6, mi.STREAM_W2, std=f ** -0.5).reshape(d, f)
    a = oracle.expert_swiglu(x, w1, w2)
    b = oracle.expert_swiglu_f64(mi.bf16_to_f64(x), mi.bf16_to_f64(w1), mi.bf16_to_f64(w2))
    np.testing.assert_array_equal(a, b)


def test_route_scale_scales_the_joint_weights():
    """The gates of a token sum to the scale, and scaling changes nothing else
    (selection, order, ratios): the scale is applied after the joint normalisation."""
    T, E = 300, 258
    z = mi.normal_f64(T * E, 8, mi.STREAM_TEST_ROWS).reshape(T, E)
    b = mi.uniform_f32(256, 8, mi.STREAM_B, -0.05, 0.05)
    r1 = oracle.route(z, b, 6, 256, 2)
    r8 = oracle.route(z, b, 6, 256, 2, route_scale=8.0)
    assert np.array_equal(r1["topk_idx"], r8["topk_idx"])
    np.testing.assert_array_equal(r8["gates"], 8.0 * r1["gates"])   # a power of two: exact
    np.testing.assert_allclose(r8["gates"].sum(axis=1), 8.0, rtol=1e-14)
    r3 = oracle.route(z, b, 6, 256, 2, route_scale=2.83)
    np.testing.assert_allclose(r3["gates"].sum(axis=1), 2.83, rtol=1e-14)


def test_inkling_workload_shapes():
    w = mi.WORKLOADS["inkling"]
    assert (w.d, w.f, w.n_routed, w.n_shared, w.k) == (6144, 3072, 256, 2, 6)
    assert w.w1_rows == 6144 and w.gate_scale == 8.0
    # 6 routed + 2 shared experts of width 3072 = the dense intermediate width 24576 of the same config
    assert (w.k + w.n_shared) * w.f == 24576
    rows = w.T * (w.k + w.n_shared)
    assert w.flops() == pytest.approx(2 * w.T * w.d * 258 + 6 * rows * w.d * w.f)
    small = mi.Workload("s", 4, 64, 32, activation="swiglu")
    assert mi.host_w1(small, 3).shape == (64, 64)
