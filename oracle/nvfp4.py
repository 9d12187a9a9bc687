"""NVFP4 part of the CPU oracle -- TEST INFRASTRUCTURE ONLY.

"Under the hood" (huggingface.co blog), "Quantization: BF16 vs NVFP4": the
released NVFP4 checkpoint quantizes weights and activations to FP4 in blocks of
16 values, each block with an FP8 scale ("group_size": 16, dynamic block scales),
for Blackwell's FP4 tensor cores (W4A4).  Only the routed experts are quantized
here; the router and the shared experts stay bf16.

Formats (Open Compute Project "OCP Microscaling Formats (MX) v1.0"):

* E2M1 (FP4): sign, 2 exponent bits (bias 1), 1 mantissa bit; the magnitudes
  are 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7, sign in bit 3);
* E4M3 (FP8, the block scale): 4 exponent bits (bias 7), 3 mantissa bits,
  subnormals down to 2^-9, largest finite 448; a scale is never negative.

Recipe (this oracle's reading; the page gives only the block size and the FP8
scales): every conversion rounds to nearest, ties to even, and saturates to the
largest finite value.  A weight matrix W gets one fp32 scale g = amax|W| / (6 * 448)
and per 16-block scales s_b = E4M3(fl32(amax_b / 6) / g); its codes are
q = E2M1(fl32(w / fl32(s_b * g))).  An activation block (dynamic, no tensor
scale) gets s_b = E4M3(fl32(amax_b / 6)) and q = E2M1(fl32(x / s_b)).  A value
is divided by its block's scale, as the format's definition puts it (an element
stands for its code times the scale, so the code is the value over the scale),
each division correctly rounded to fp32.  A block whose scale rounds to 0 has
all codes 0.  Every quantity that decides a code or a scale is one fp32 operation
on fp32 operands, in the order written.

The expert (§02 of "Inkling, Dissected": two matmuls with a nonlinearity, GELU
tanh form here) on quantized operands: h = gelu(g1 * sum(dq(x) dq(W1))),
h is quantized like any activation, y = g2 * sum(dq(h) dq(W2)); the sums are
fp64 over the exact dequantized values.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

E2M1_MAGNITUDE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0
E4M3_MAX = 448.0
BLOCK = 16


# ---------------------------------------------------------------------------
# element formats
# ---------------------------------------------------------------------------
def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    mag = E2M1_MAGNITUDE[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 value, ties to the even code (mantissa bit 0), saturating at
    +-6; values that round to zero magnitude get code 0 (no negative zero)."""
    v = np.asarray(v, dtype=np.float64)
    m = np.abs(v)
    # midpoints between neighbouring magnitudes, and which side a tie goes to:
    # 0.25 (0|0.5 -> 0), 0.75 (0.5|1 -> 1), 1.25 (1|1.5 -> 1), 1.75 (1.5|2 -> 2),
    # 2.5 (2|3 -> 2), 3.5 (3|4 -> 4), 5 (4|6 -> 4): the even codes are 0, 2, 4, 6
    code = np.full(m.shape, 7, dtype=np.int64)
    for c in range(6, -1, -1):
        lo, hi = E2M1_MAGNITUDE[c], E2M1_MAGNITUDE[c + 1]
        mid = 0.5 * (lo + hi)
        take_lower = (m < mid) | ((m == mid) & (c % 2 == 0))
        code = np.where(take_lower, c, code)
    code = np.where((code > 0) & (v < 0), code | 8, code)
    return code.astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    e = (c >> 3) & 15
    mnt = c & 7
    val = np.where(e == 0, mnt / 8.0 * 2.0 ** -6, (1.0 + mnt / 8.0) * 2.0 ** (e - 7))
    return np.where(c & 128, -val, val)


def _e4m3_table() -> np.ndarray:
    return e4m3_decode(np.arange(0, 127))  # 0x00 .. 0x7E: every finite non-negative value, increasing


def e4m3_encode_nonneg(v: np.ndarray) -> np.ndarray:
    """Nearest non-negative E4M3 value to v >= 0, ties to the even code,
    saturating at 448."""
    v = np.asarray(v, dtype=np.float64)
    table = _e4m3_table()
    v = np.minimum(v, E4M3_MAX)
    hi = np.searchsorted(table, v, side="left")            # first value >= v
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = v - table[lo]
    d_hi = table[hi] - v
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(table[hi] == v, hi, np.where(pick_hi, hi, lo))
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# quantization (blocks of 16 along the last axis)
# ---------------------------------------------------------------------------
def _blocks(a: np.ndarray) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    assert a.shape[-1] % BLOCK == 0
    return a.reshape(a.shape[:-1] + (a.shape[-1] // BLOCK, BLOCK))


def quantize_activation(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Dynamic block quantization of activations (fp32 values, [..., K]):
    codes [..., K] (unpacked E2M1), scale codes [..., K/16] (E4M3)."""
    b = _blocks(x)
    amax = np.abs(b).max(axis=-1)
    s_code = e4m3_encode_nonneg((amax / np.float32(6.0)).astype(np.float32))
    s = e4m3_decode(s_code).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (b / s[..., None]).astype(np.float32)
    q = np.where(s[..., None] > 0, e2m1_encode(r), 0).astype(np.uint8)
    return q.reshape(np.shape(x)), s_code


def quantize_weight(w: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.float32]:
    """Two-level quantization of one weight matrix [N, K] (fp32 values):
    codes [N, K], block scale codes [N, K/16], tensor scale g (fp32)."""
    w = np.asarray(w, dtype=np.float32)
    g = np.float32(np.abs(w).max() / np.float32(6.0 * 448.0)) if w.size else np.float32(0)
    b = _blocks(w)
    amax = np.abs(b).max(axis=-1)
    if g == 0:
        return np.zeros(w.shape, np.uint8), np.zeros(amax.shape, np.uint8), np.float32(0)
    s_code = e4m3_encode_nonneg(((amax / np.float32(6.0)).astype(np.float32) / g).astype(np.float32))
    denom = (e4m3_decode(s_code).astype(np.float32) * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (b / denom[..., None]).astype(np.float32)
    q = np.where(denom[..., None] > 0, e2m1_encode(r), 0).astype(np.uint8)
    return q.reshape(w.shape), s_code, g


def dequantize(q: np.ndarray, s_code: np.ndarray, g: float = 1.0) -> np.ndarray:
    """Exact values (fp64) of codes with their block scales (and tensor scale)."""
    v = e2m1_decode(q)
    v = v.reshape(v.shape[:-1] + (v.shape[-1] // BLOCK, BLOCK)) * e4m3_decode(s_code)[..., None]
    return v.reshape(np.shape(q)) * float(g)


# ---------------------------------------------------------------------------
# the expert on NVFP4 operands
# ---------------------------------------------------------------------------
def gemm(a_q, a_s, b_q, b_s, g_b) -> np.ndarray:
    """g_b * (dq(A) @ dq(B)^T) in fp64; A [M, K] activations, B [N, K] weights."""
    return dequantize(a_q, a_s) @ dequantize(b_q, b_s).T * float(g_b)


def expert_swiglu(x_f32: np.ndarray, w1: tuple, w2: tuple) -> dict:
    """One SwiGLU expert ("Under the hood", "MoE: the expert configuration") on NVFP4
    operands: W1 [2 d_ff, d] (gate rows, then up rows) is one quantized matrix (one
    tensor scale g1); h = silu(g1 * sum(dq(x) dq(Wg))) * (g1 * sum(dq(x) dq(Wu))),
    quantized like any activation; y = g2 * sum(dq(h) dq(W2))."""
    q1, s1, g1 = w1
    f = q1.shape[0] // 2
    xq, xs = quantize_activation(x_f32)
    pre = gemm(xq, xs, q1, s1, g1)          # [n, 2 d_ff]: gate columns, then up columns
    gate, up = pre[:, :f], pre[:, f:]
    h = gate / (1.0 + np.exp(-gate)) * up
    hq, hs = quantize_activation(h.astype(np.float32))
    y = gemm(hq, hs, *w2)
    return {"xq": xq, "xs": xs, "pre": pre, "h": h, "hq": hq, "hs": hs, "y": y}


def expert(x_f32: np.ndarray, w1: tuple, w2: tuple) -> dict:
    """One GELU expert on NVFP4 operands.  x_f32 [n, d] (the bf16 inputs as fp32);
    w1 = (q [f, d], s, g), w2 = (q [d, f], s, g) from ``quantize_weight``.
    Returns the quantized input, the pre-activation, h and its quantization, y."""
    from oracle import gelu_tanh

    xq, xs = quantize_activation(x_f32)
    pre = gemm(xq, xs, *w1)
    h = gelu_tanh(pre)
    hq, hs = quantize_activation(h.astype(np.float32))
    y = gemm(hq, hs, *w2)
    return {"xq": xq, "xs": xs, "pre": pre, "h": h, "hq": hq, "hs": hs, "y": y}


# ---------------------------------------------------------------------------
# the layer with NVFP4 routed experts (router and shared experts in bf16)
# ---------------------------------------------------------------------------
def forward_tokens(w, tokens, bias, keep=None, cache=None) -> dict:
    """The layer's forward for the given tokens of workload w with the routed
    experts on NVFP4 operands (weights quantized by ``quantize_weight``, each
    token's activations by ``quantize_activation``) and the shared experts as
    in the bf16 layer; gates, routing and the combine as ``oracle.forward_tokens``.
    ``cache`` (dict) keeps quantized expert weights between calls."""
    import moe_inputs as mi
    import oracle

    cache = {} if cache is None else cache
    tokens = np.asarray(tokens, dtype=np.int64)
    x = mi.host_x(w, tokens)
    r = oracle.route_workload(w, bias, tokens, mi.host_logit_offset(w), x=x)
    contrib = r["contrib"]
    gates = r["gates"].copy()
    if keep is not None:
        gates[:, :w.k] = np.where(np.asarray(keep, dtype=bool), gates[:, :w.k], 0.0)
    xf = mi.bf16_to_f64(x).astype(np.float32)
    out = np.zeros((len(tokens), w.d), dtype=np.float64)
    for e in np.unique(contrib):
        e = int(e)
        rows, slots = np.nonzero(contrib == e)
        if e < w.n_routed:
            if e not in cache:
                cache[e] = (quantize_weight(mi.bf16_to_f64(mi.host_w1(w, e)).astype(np.float32)),
                            quantize_weight(mi.bf16_to_f64(mi.host_w2(w, e)).astype(np.float32)))
            fn = expert_swiglu if getattr(w, "activation", "gelu_tanh") == "swiglu" else expert
            y = fn(xf[rows], *cache[e])["y"]
        else:
            y = oracle.expert_for(w)(x[rows], mi.host_w1(w, e), mi.host_w2(w, e))
        out[rows] += gates[rows, slots][:, None] * y
    r["out"] = out
    r["tokens"] = tokens
    return r
