"""CPU oracle for the sparse MoE layer -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct fp64 restatement of the layer the pages
describe.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it.  It shares no code with the CUDA path
(``sparse_moe_layer_joint_b200``): the only module both sides use is
``moe_inputs``, which generates the seeded synthetic inputs and holds none of
the layer's arithmetic.

Sources (all on "Inkling, Dissected", engineermaxxing.com, unless noted):

* §02 "Anatomy of one MoE layer": 256 routed experts (each token uses exactly
  6), 2 shared experts that see every token, a router scoring the experts; the
  layer output is the weighted sum of the 8 contributing experts' outputs with
  one joint normalisation; an expert is two matmuls with a nonlinearity.
* §02b "Sigmoid, not softmax": s_i = sigmoid(x . w_i); keep the top 6 by
  s_i + b_i; g_i = s_i / sum over kept U shared of s_j; the per-token sketch
  orders the steps (scores for all 258, top-6 of the first 256 plus bias,
  append the shared indices 256 and 257, normalise, weighted sum).
* §02c "A routing decision, by hand": the worked 4-expert, top-2 example.
* §02e "The aux-loss-free bias": after each batch, b_i <- b_i + gamma *
  sign(Lbar - L_i), L_i = tokens that selected expert i, Lbar = total
  selections / 256.
* "Under the hood" (huggingface.co blog), "The routing strategy": scores cover
  256 + 2 experts with independent sigmoids, top-6 over routed experts only
  after adding the correction bias, shared experts join the normalisation but
  are never candidates.

Readings where the pages are silent:
ties in the top-k go to the lower expert index; the output order of the top-k
is descending biased score; sign(0) = 0; Lbar = k*T/n_routed compared in
integers; only routed experts are counted; the bias update follows the forward
(the forward uses the current b); route_scale is 1 (gates sum to 1); the
nonlinearity is GELU (tanh form); experts have no biases; no residual is added.

The functions follow the pages' order: ``route`` (scores, biased top-k, joint
gates), ``load_counts``, ``bias_update``, ``dispatch`` (grouping of the
(token, expert) pairs by expert), ``expert`` (one expert MLP), ``combine`` and
``forward_tokens`` (all of it for a set of tokens).  Further: expert capacity
and its metrics (``capacity_for``, ``capacity_keep``, ``load_metrics``, §02d),
the Router Balance Lab loop (``lab_run``, §02g), the SwiGLU expert of the
released configuration (``expert_swiglu``, "Under the hood") and, in
``oracle/nvfp4.py``, the NVFP4 quantization and experts.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np

import moe_inputs as mi

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.or_logits.argtypes = [vp, vp, i64, i64, i64, vp, i32]
        L.or_gelu_tanh.argtypes = [vp, i64, vp]
        L.or_expert_mlp.argtypes = [vp, i64, vp, vp, i64, i64, vp, i32]
        L.or_expert_mlp_f64.argtypes = [vp, i64, vp, vp, i64, i64, vp, i32]
        L.or_silu.argtypes = [vp, i64, vp]
        L.or_expert_swiglu.argtypes = [vp, i64, vp, vp, i64, i64, vp, i32]
        L.or_expert_swiglu_f64.argtypes = [vp, i64, vp, vp, i64, i64, vp, i32]
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
# router: §02b formula; "Under the hood", "The routing strategy", steps 1-4
# ---------------------------------------------------------------------------
def logits(x_bf16: np.ndarray, w_bf16: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """z[t, i] = x_t . w_i in fp64 for every expert row of w (bf16 bit patterns)."""
    x = _c(x_bf16, np.uint16)
    w = _c(w_bf16, np.uint16)
    T, d = x.shape
    E = w.shape[0]
    z = np.empty((T, E), dtype=np.float64)
    lib().or_logits(x.ctypes.data, w.ctypes.data, T, d, E, z.ctypes.data, nthreads)
    return z


def sigmoid(z: np.ndarray) -> np.ndarray:
    """The affinity s = sigma(z) = 1 / (1 + e^-z), independently per expert (§02b)."""
    return 1.0 / (1.0 + np.exp(-np.asarray(z, dtype=np.float64)))


def route(z: np.ndarray, bias: np.ndarray, k: int, n_routed: int, n_shared: int,
          logit_offset: Optional[np.ndarray] = None, route_scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Biased top-k selection and joint gates from router logits.

    z [T, n_routed + n_shared] fp64 logits; bias [n_routed] (fp32 values).
    ``logit_offset`` (workload input, routed experts only) is added to z before
    the sigmoid.

    Returns topk_idx [T, k] int32 (descending s_i + b_i, ties to the lower
    index), gates [T, k + n_shared] fp64 (the k routed in topk order, then the
    shared experts in index order), s [T, E], sel [T, n_routed] = s + b and
    margin [T] = sel of the k-th minus sel of the (k+1)-th candidate.

    ``route_scale``: the jointly normalised weights are multiplied by it ("Under
    the hood", "The routing strategy", step 5: route_scale times the learned
    global_scale; the caller passes the product).  1 leaves gates summing to 1.
    """
    z = np.array(z, dtype=np.float64)
    T, E = z.shape
    assert E == n_routed + n_shared and 1 <= k <= n_routed
    if logit_offset is not None:
        z[:, :n_routed] += np.asarray(logit_offset, dtype=np.float64)
    s = sigmoid(z)
    # the bias enters the selection score and nothing else (§02b, §02e)
    sel = s[:, :n_routed] + np.asarray(bias, dtype=np.float64)[None, :]
    # full sort of every token's candidates: descending sel, then ascending index
    index = np.broadcast_to(np.arange(n_routed), sel.shape)
    order = np.lexsort((index, -sel), axis=-1)
    topk = order[:, :k]
    if k < n_routed:
        rows = np.arange(T)
        margin = sel[rows, order[:, k - 1]] - sel[rows, order[:, k]]
    else:
        margin = np.full(T, np.inf)
    # joint normalisation over the kept routed experts and all shared experts
    contrib = np.concatenate([topk, np.broadcast_to(np.arange(n_routed, E), (T, n_shared))], axis=1)
    s_c = np.take_along_axis(s, contrib, axis=1)
    # the denominator is a sum over a set: add its terms in ascending expert
    # index, so the gates depend on which experts are kept, not on their rank
    den = np.take_along_axis(s, np.sort(contrib, axis=1), axis=1).sum(axis=1, keepdims=True)
    gates = s_c / den * float(route_scale)
    return {"topk_idx": topk.astype(np.int32), "gates": gates, "s": s, "sel": sel, "margin": margin,
            "contrib": contrib.astype(np.int32)}


# ---------------------------------------------------------------------------
# §02e: loads and the aux-loss-free bias controller
# ---------------------------------------------------------------------------
def load_counts(topk_idx: np.ndarray, n_routed: int) -> np.ndarray:
    """L_i: how many tokens selected routed expert i this batch (int32)."""
    return np.bincount(np.asarray(topk_idx).reshape(-1), minlength=n_routed).astype(np.int32)


def bias_update(counts: np.ndarray, bias: np.ndarray, T: int, k: int, gamma: float) -> np.ndarray:
    """b_i <- b_i + gamma * sign(Lbar - L_i) with Lbar = k*T / n_routed.

    The sign is taken in integers, sign(k*T - n_routed*L_i), so no rounding of
    Lbar enters; b is fp32, so the step is the fp32 sum of b_i and
    fl32(gamma) * sign, and sign(0) = 0 leaves b_i unchanged.
    """
    counts = np.asarray(counts, dtype=np.int64)
    n_routed = counts.shape[0]
    sgn = np.sign(np.int64(k) * np.int64(T) - np.int64(n_routed) * counts).astype(np.float32)
    b = np.asarray(bias, dtype=np.float32)
    return (b + np.float32(gamma) * sgn).astype(np.float32)


# ---------------------------------------------------------------------------
# §02d: expert capacity -- assignments past an expert's capacity are dropped
# ---------------------------------------------------------------------------
def capacity_for(factor: float, T: int, k: int, n_routed: int) -> int:
    """Capacity of every routed expert: ``factor`` times the ideal load k*T/n_routed,
    rounded down to a whole number of tokens (the page gives 1.25x the ideal load
    and no rounding; rounding down keeps the capacity at or below that bound).
    The factor is taken as the decimal number it prints as, so 1.25 is 5/4 exactly."""
    from fractions import Fraction
    return int((Fraction(repr(float(factor))) * k * T) // n_routed)


def capacity_keep(topk_idx: np.ndarray, capacity: int, n_routed: int) -> np.ndarray:
    """keep[t, j]: whether the assignment of token t to expert topk_idx[t, j] is served.

    Each expert serves at most ``capacity`` tokens per batch; its queue is filled
    in token order, and the assignments that arrive once the queue is full are
    the overflow, which is dropped (§02d).  A token never picks an expert twice,
    so within one token the slot order does not matter."""
    topk_idx = np.asarray(topk_idx)
    T, k = topk_idx.shape
    queued = [0] * n_routed
    keep = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for j in range(k):
            e = int(topk_idx[t, j])
            keep[t, j] = queued[e] < capacity
            queued[e] += 1
    return keep


def load_metrics(counts: np.ndarray, capacity: Optional[int], T: int, k: int) -> Dict[str, float]:
    """Balance metrics of one batch from the loads L_i (the demand: tokens that
    selected expert i, dropped or not).  MaxVio = max_i L_i / Lbar - 1 with
    Lbar = k*T/n_routed (the hottest expert's demand over the ideal, minus one);
    dropped = sum_i max(0, L_i - capacity); drop_rate = dropped / (k*T), the share
    of expert slots lost to overflow (§02g)."""
    L = np.asarray(counts, dtype=np.int64)
    n_routed = L.shape[0]
    ideal = k * T / n_routed
    dropped = int(np.maximum(L - capacity, 0).sum()) if capacity is not None else 0
    return {"max_load": int(L.max()) if L.size else 0, "max_vio": float(L.max() / ideal - 1.0) if T else 0.0,
            "dropped": dropped, "drop_rate": dropped / (k * T) if T else 0.0}


def lab_run(w: "mi.LabWorkload", gamma: float, steps: Optional[int] = None,
            bias0: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """The Router Balance Lab loop (§02g) for one balancing step size: per step,
    score the step's tokens with the frozen router, take the biased top-k, count
    the loads, apply the capacity, record MaxVio and the drop rate, then move the
    bias (§02e).  gamma = 0 is the lab's no-balancing arm."""
    steps = w.steps if steps is None else steps
    wr = mi.lab_wr(w)
    cap = capacity_for(w.capacity_factor, w.T, w.k, w.n_routed)
    b = np.zeros(w.n_routed, dtype=np.float32) if bias0 is None else np.asarray(bias0, dtype=np.float32)
    out = {"max_vio": [], "drop_rate": [], "dropped": [], "counts": [], "bias": [b.copy()], "capacity": cap}
    for st in range(steps):
        r = route(logits(mi.lab_x(w, st), wr), b, w.k, w.n_routed, w.n_shared)
        L = load_counts(r["topk_idx"], w.n_routed)
        m = load_metrics(L, cap, w.T, w.k)
        out["max_vio"].append(m["max_vio"])
        out["drop_rate"].append(m["drop_rate"])
        out["dropped"].append(m["dropped"])
        out["counts"].append(L)
        b = bias_update(L, b, w.T, w.k, gamma)
        out["bias"].append(b.copy())
    for key in ("max_vio", "drop_rate", "dropped", "counts", "bias"):
        out[key] = np.asarray(out[key])
    return out


# ---------------------------------------------------------------------------
# dispatch (§02: every token goes to exactly its 6 routed experts)
# ---------------------------------------------------------------------------
def dispatch(topk_idx: np.ndarray, n_routed: int, keep: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Group the T*k (token, slot) pairs by expert, each expert's rows in token order.

    offsets [n_routed + 1]: rows of expert e are offsets[e] .. offsets[e+1]-1;
    row_token [rows]: the token each row came from; token_row [T, k]: the row
    each (token, slot) pair went to.  With ``keep`` (from ``capacity_keep``) only
    the served pairs get rows and a dropped pair's token_row is -1.
    """
    topk_idx = np.asarray(topk_idx)
    T, k = topk_idx.shape
    flat = topk_idx.reshape(-1).astype(np.int64)
    served = np.ones(T * k, dtype=bool) if keep is None else np.asarray(keep, dtype=bool).reshape(-1)
    pairs = np.nonzero(served)[0]                              # served (token, slot) pairs, in token order
    order = pairs[np.argsort(flat[pairs], kind="stable")]      # by expert, then by (token, slot)
    counts = np.bincount(flat[pairs], minlength=n_routed)
    offsets = np.zeros(n_routed + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    row_token = (order // k).astype(np.int32)
    token_row = np.full(T * k, -1, dtype=np.int32)
    token_row[order] = np.arange(len(order), dtype=np.int32)
    return {"offsets": offsets.astype(np.int32), "row_token": row_token, "token_row": token_row.reshape(T, k)}


# ---------------------------------------------------------------------------
# experts (§02: two matmuls with a nonlinearity; GELU, tanh form)
# ---------------------------------------------------------------------------
def gelu_tanh(u: np.ndarray) -> np.ndarray:
    u = _c(u, np.float64)
    out = np.empty_like(u)
    lib().or_gelu_tanh(u.ctypes.data, u.size, out.ctypes.data)
    return out


def expert(xrows_bf16: np.ndarray, w1_bf16: np.ndarray, w2_bf16: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """y[r] = W2 . gelu(W1 . x_r) in fp64; x rows [n, d], W1 [d_ff, d], W2 [d, d_ff] (bf16 bits)."""
    x = _c(xrows_bf16, np.uint16)
    w1 = _c(w1_bf16, np.uint16)
    w2 = _c(w2_bf16, np.uint16)
    n, d = x.shape
    f = w1.shape[0]
    assert w1.shape == (f, d) and w2.shape == (d, f)
    y = np.zeros((n, d), dtype=np.float64)
    if n:
        lib().or_expert_mlp(x.ctypes.data, n, w1.ctypes.data, w2.ctypes.data, d, f, y.ctypes.data, nthreads)
    return y


def expert_f64(xrows: np.ndarray, w1: np.ndarray, w2: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """The same expert on fp64 operands (for pins with exact inputs)."""
    x = _c(xrows, np.float64)
    w1 = _c(w1, np.float64)
    w2 = _c(w2, np.float64)
    n, d = x.shape
    f = w1.shape[0]
    assert w1.shape == (f, d) and w2.shape == (d, f)
    y = np.zeros((n, d), dtype=np.float64)
    if n:
        lib().or_expert_mlp_f64(x.ctypes.data, n, w1.ctypes.data, w2.ctypes.data, d, f, y.ctypes.data, nthreads)
    return y


def silu(u: np.ndarray) -> np.ndarray:
    u = _c(u, np.float64)
    out = np.empty_like(u)
    lib().or_silu(u.ctypes.data, u.size, out.ctypes.data)
    return out


def expert_swiglu(xrows_bf16: np.ndarray, w1_bf16: np.ndarray, w2_bf16: np.ndarray, nthreads: int = 0) -> np.ndarray:
    """The gated expert of the released configuration ("Under the hood", "MoE: the
    expert configuration": SwiGLU experts), y[r] = W2 . (silu(Wg . x_r) * (Wu . x_r))
    in fp64; W1 [2 d_ff, d] holds Wg (rows 0..d_ff-1) then Wu, W2 [d, d_ff] (bf16 bits)."""
    x = _c(xrows_bf16, np.uint16)
    w1 = _c(w1_bf16, np.uint16)
    w2 = _c(w2_bf16, np.uint16)
    n, d = x.shape
    f = w2.shape[1]
    assert w1.shape == (2 * f, d) and w2.shape == (d, f)
    y = np.zeros((n, d), dtype=np.float64)
    if n:
        lib().or_expert_swiglu(x.ctypes.data, n, w1.ctypes.data, w2.ctypes.data, d, f, y.ctypes.data, nthreads)
    return y


def expert_swiglu_f64(xrows: np.ndarray, w1: np.ndarray, w2: np.ndarray, nthreads: int = 0) -> np.ndarray:
    x = _c(xrows, np.float64)
    w1 = _c(w1, np.float64)
    w2 = _c(w2, np.float64)
    n, d = x.shape
    f = w2.shape[1]
    assert w1.shape == (2 * f, d) and w2.shape == (d, f)
    y = np.zeros((n, d), dtype=np.float64)
    if n:
        lib().or_expert_swiglu_f64(x.ctypes.data, n, w1.ctypes.data, w2.ctypes.data, d, f, y.ctypes.data, nthreads)
    return y


def expert_for(w: "mi.Workload"):
    """The expert function of a workload's activation."""
    return expert_swiglu if getattr(w, "activation", "gelu_tanh") == "swiglu" else expert


# ---------------------------------------------------------------------------
# combine (§02: weighted sum of the 8 contributors, honest gates)
# ---------------------------------------------------------------------------
def combine(y_rows: np.ndarray, token_row: np.ndarray, gates: np.ndarray,
            y_shared: Optional[np.ndarray]) -> np.ndarray:
    """out[t] = sum_j g[t, j] y_rows[token_row[t, j]] + sum_s g[t, k+s] y_shared[s, t] (fp64)."""
    y_rows = np.asarray(y_rows, dtype=np.float64)
    gates = np.asarray(gates, dtype=np.float64)
    T, k = token_row.shape
    out = np.zeros((T, y_rows.shape[1]), dtype=np.float64)
    for j in range(k):
        out += gates[:, j:j + 1] * y_rows[token_row[:, j]]
    if y_shared is not None:
        y_shared = np.asarray(y_shared, dtype=np.float64)
        for s in range(y_shared.shape[0]):
            out += gates[:, k + s:k + s + 1] * y_shared[s]
    return out


# ---------------------------------------------------------------------------
# whole layer for a set of tokens of a workload (inputs from moe_inputs)
# ---------------------------------------------------------------------------
def route_workload(w: "mi.Workload", bias: np.ndarray, tokens: Optional[Sequence[int]] = None,
                   logit_offset: Optional[np.ndarray] = None, wr: Optional[np.ndarray] = None,
                   x: Optional[np.ndarray] = None, nthreads: int = 0) -> Dict[str, np.ndarray]:
    """Router output for all tokens (or the given ones) of workload w."""
    if x is None:
        x = mi.host_x(w, tokens)
    if wr is None:
        wr = mi.host_wr(w)
    z = logits(x, wr, nthreads)
    r = route(z, bias, w.k, w.n_routed, w.n_shared, logit_offset, route_scale=w.gate_scale)
    r["z"] = z
    return r


def forward_tokens(w: "mi.Workload", tokens: Sequence[int], bias: np.ndarray,
                   logit_offset: Optional[np.ndarray] = None, nthreads: int = 0,
                   weights: Optional[Dict[str, np.ndarray]] = None,
                   keep: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """The layer's forward for the given tokens of workload w, in fp64.

    Tokens are independent in this layer (each token's output depends only on
    its own x row), so the result for a sample of tokens is exactly the full
    layer's result on those tokens.  ``weights`` may hold host copies of
    w1 [E, f, d] and w2 [E, d, f]; otherwise each needed expert's matrices are
    generated on demand.

    ``keep`` [len(tokens), k] (from ``capacity_keep`` over the whole batch, since
    capacity couples the tokens): routed assignments marked False were dropped and
    contribute nothing; the other gates are left as they are (§02d: a dropped
    token simply does not get that expert's contribution).
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    x = mi.host_x(w, tokens)
    r = route_workload(w, bias, tokens, logit_offset, x=x, nthreads=nthreads)
    n = len(tokens)
    contrib = r["contrib"]           # [n, k + n_shared] expert ids
    gates = r["gates"].copy()
    if keep is not None:
        gates[:, :w.k] = np.where(np.asarray(keep, dtype=bool), gates[:, :w.k], 0.0)
    out = np.zeros((n, w.d), dtype=np.float64)
    for e in np.unique(contrib):
        rows, slots = np.nonzero(contrib == e)
        if weights is not None:
            w1, w2 = weights["w1"][e], weights["w2"][e]
        else:
            w1, w2 = mi.host_w1(w, int(e)), mi.host_w2(w, int(e))
        y = expert_for(w)(x[rows], w1, w2, nthreads)
        out[rows] += gates[rows, slots][:, None] * y
    r["out"] = out
    r["tokens"] = tokens
    return r
