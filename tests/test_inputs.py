"""The seeded input generator: published Philox test vectors, accuracy of its
own log/sin/cos against libm, distribution moments, slicing consistency."""
import math

import numpy as np
import pytest

import moe_inputs as mi


# Known-answer vectors for Philox-4x32-10 published with the Random123 library
# (Salmon et al., SC'11): (counter, key) -> output.
KAT = [
    ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
    ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
    ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
     [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
]


@pytest.mark.parametrize("ctr,key,out", KAT)
def test_philox_known_answers(ctr, key, out):
    assert list(mi.philox_raw(ctr, key)) == out


def test_box_muller_matches_libm():
    """Our series-based ln and sincos(2 pi u) reproduce libm's Box-Muller to ~1e-15."""
    n = 4096
    w = mi.words(n, 0, mi.STREAM_X)          # words of blocks 0..1023 in order
    z = mi.normal_f64(n, 0, mi.STREAM_X)
    for i in range(0, n, 4):
        for p in range(2):
            u1 = (float(w[i + 2 * p]) + 0.5) / 2.0**32
            u2 = float(w[i + 2 * p + 1]) / 2.0**32
            rad = math.sqrt(-2.0 * math.log(u1))
            ref_c, ref_s = rad * math.cos(2 * math.pi * u2), rad * math.sin(2 * math.pi * u2)
            assert z[i + 2 * p] == pytest.approx(ref_c, abs=1e-13)
            assert z[i + 2 * p + 1] == pytest.approx(ref_s, abs=1e-13)


def test_normal_moments():
    z = mi.normal_f64(1 << 21, 0, mi.STREAM_W1)
    assert abs(z.mean()) < 3e-3
    assert abs(z.std() - 1) < 3e-3
    assert abs((z ** 4).mean() - 3) < 3e-2


def test_uniform_range_and_mean():
    u = mi.uniform_f32(1 << 20, 0, mi.STREAM_B, -0.05, 0.05)
    assert u.min() > -0.05 and u.max() < 0.05
    assert abs(u.mean()) < 2e-4


def test_bf16_rounding_matches_torch():
    import torch

    f = mi.normal_f32(1 << 16, 3, mi.STREAM_X, std=3.0)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mi.f32_to_bf16_bits(f), ref)
    np.testing.assert_array_equal(mi.normal_bf16(1 << 16, 3, mi.STREAM_X, std=3.0), ref)


def test_slices_agree_with_whole_tensors():
    w = mi.WORKLOADS["tiny"]
    w1 = mi.host_w1_all(w)
    w2 = mi.host_w2_all(w)
    for e in (0, 17, 256, 257):
        np.testing.assert_array_equal(mi.host_w1(w, e), w1[e])
        np.testing.assert_array_equal(mi.host_w2(w, e), w2[e])
    x = mi.host_x(w)
    np.testing.assert_array_equal(mi.host_x(w, [3, 200]), x[[3, 200]])


def test_thread_count_does_not_change_values():
    a = mi.normal_bf16(300_001, 1, mi.STREAM_W2, 0, 0.1, nthreads=1)
    b = mi.normal_bf16(300_001, 1, mi.STREAM_W2, 0, 0.1, nthreads=7)
    np.testing.assert_array_equal(a, b)


def test_workload_flop_counts():
    w = mi.WORKLOADS["prefill"]
    assert w.flops() == pytest.approx(31.03e12, rel=1e-3)
    assert w.flops() / w.T == pytest.approx(473.5e6, rel=1e-3)


def test_lab_generator_recipe():
    """The Router Balance Lab inputs follow their stated recipe: specialties Zipf-distributed with
    expert 0 about 30 times as common as expert 63, tokens at their specialty's center plus
    N(0, sigma^2 / d) jitter, router rows alpha * center."""
    w = mi.LAB
    spec = np.concatenate([mi.lab_specialty(w, s) for s in range(w.steps)])
    counts = np.bincount(spec, minlength=w.n_routed)
    assert 30 * 0.8 < counts[0] / counts[-1] < 30 * 1.25
    assert (np.diff(counts[:8]) < 0).all()                  # the most common specialties in Zipf order
    c = mi.lab_centers(w)
    np.testing.assert_array_equal(mi.lab_wr(w), mi.f32_to_bf16_bits((w.alpha * c).astype(np.float32)))
    x = mi.bf16_to_f64(mi.lab_x(w, 7))
    jit = x - c[mi.lab_specialty(w, 7)]
    assert abs(jit.mean()) < 0.005
    np.testing.assert_allclose(jit.std(), w.sigma / np.sqrt(w.d), rtol=0.03)
    # steps draw fresh batches
    assert not np.array_equal(mi.lab_x(w, 0), mi.lab_x(w, 1))
