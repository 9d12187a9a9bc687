"""Seeded synthetic inputs for the sparse MoE layer (input generation only).

This module is the one piece shared by the CPU oracle (``oracle/``) and the
CUDA path (``sparse_moe_layer_joint_b200``).  It holds none of the layer's
arithmetic: it turns (seed, stream id, element index) into numbers with the
distributions the workloads below state, bit-identically on the host (C++) and
on the device (CUDA) -- see ``csrc/gen_core.h`` for the generator
(Philox-4x32-10 + Box-Muller, both written from their published definitions).

Every tensor has its own stream id, so any slice of any tensor (one token's
row, one expert's weight matrix) can be produced on its own: the oracle
generates only the slices it needs, the GPU generates whole tensors in HBM.

Workloads (the layer of "Inkling, Dissected" §02 "Anatomy of one MoE layer":
256 routed + 2 shared experts, top-6, each expert a d -> d_ff -> d MLP):

=========  ======  ====  =====  ==================================================
name        T       d     d_ff   notes
=========  ======  ====  =====  ==================================================
tiny        256     256   128    b ~ U(-0.1, 0.1); one bias update, gamma 1e-3
mid         4096    2048  768    b = 0
skew        16384   4096  1024   Zipf(s=1.1)-ranked logit offset; 20 bias updates
decode      64      7168  2048   b ~ U(-0.05, 0.05); weight-streaming bound
prefill     65536   7168  2048   b ~ U(-0.05, 0.05); about 15 GB of expert weights
inkling     65536   6144  3072   SwiGLU experts, route_scale 8; about 29 GB of weights
inkling_decode 64   6144  3072   the same layer at decode scale
=========  ======  ====  =====  ==================================================

x ~ N(0, 1); router and first-layer expert weights ~ N(0, 1/d); second-layer
expert weights ~ N(0, 1/d_ff) (variance = 1/fan_in).  All bf16 except b (fp32).
"""
from __future__ import annotations

import ctypes
import json
import math
import os
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoeinputs.so")

# One Philox stream id per tensor.
STREAM_X = 1
STREAM_WR = 2
STREAM_W1 = 3
STREAM_W2 = 4
STREAM_B = 5
STREAM_PERM = 6
# Streams for stage-level test inputs (synthetic intermediate tensors).
STREAM_TEST_TOPK = 10
STREAM_TEST_ROWS = 11
STREAM_TEST_GATES = 12
STREAM_TEST_SHARED = 13
# Streams of the Router Balance Lab workload.
STREAM_LAB_CENTERS = 20
STREAM_LAB_SPECIALTY = 21
STREAM_LAB_JITTER = 22

N_ROUTED = 256
N_SHARED = 2
TOP_K = 6


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    f: int
    n_routed: int = N_ROUTED
    n_shared: int = N_SHARED
    k: int = TOP_K
    seed: int = 0
    b_half_width: float = 0.0   # b ~ U(-w, w); 0 means b = 0
    gamma: float = 1e-3
    bias_iters: int = 1
    skew: bool = False
    description: str = ""
    activation: str = "gelu_tanh"   # or "swiglu": W1 holds the gate rows, then the up rows
    route_scale: float = 1.0        # the released config's route_scale
    global_scale: float = 1.0       # its learned scalar (no trained value here: 1)

    @property
    def n_experts(self) -> int:
        return self.n_routed + self.n_shared

    @property
    def w1_rows(self) -> int:
        return 2 * self.f if self.activation == "swiglu" else self.f

    @property
    def gate_scale(self) -> float:
        return self.route_scale * self.global_scale

    @property
    def std_x(self) -> float:
        return 1.0

    @property
    def std_wr(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def std_w1(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def std_w2(self) -> float:
        return 1.0 / math.sqrt(self.f)

    def flops(self) -> float:
        """Algorithmic FLOPs of one layer forward: router GEMM + 2 expert GEMMs
        over the T*k routed and T*n_shared shared (token, expert) rows."""
        rows = self.T * (self.k + self.n_shared)
        mats = 3 if self.activation == "swiglu" else 2
        return 2.0 * self.T * self.d * self.n_experts + 2.0 * mats * self.d * self.f * rows


WORKLOADS = {
    "tiny": Workload("tiny", 256, 256, 128, b_half_width=0.1, gamma=1e-3, bias_iters=1,
                     description="tiny MoE layer: T=256, d=256, d_ff=128"),
    "mid": Workload("mid", 4096, 2048, 768, b_half_width=0.0,
                    description="uniform routing, mid-size: T=4096, d=2048, d_ff=768"),
    "skew": Workload("skew", 16384, 4096, 1024, b_half_width=0.0, gamma=1e-3, bias_iters=20, skew=True,
                     description="skewed routing (Zipf s=1.1 logit offset): T=16384, d=4096, d_ff=1024"),
    "decode": Workload("decode", 64, 7168, 2048, b_half_width=0.05,
                       description="decode-scale: T=64, d=7168, d_ff=2048"),
    "prefill": Workload("prefill", 65536, 7168, 2048, b_half_width=0.05,
                        description="prefill-scale: T=65536, d=7168, d_ff=2048"),
    # the released Inkling configuration ("Under the hood": hidden 6144, SwiGLU experts of
    # intermediate 3072, route_scale 8 times a learned global_scale)
    "inkling": Workload("inkling", 65536, 6144, 3072, b_half_width=0.05, activation="swiglu", route_scale=8.0,
                        description="Inkling config, prefill-scale: T=65536, d=6144, SwiGLU d_ff=3072, "
                                    "route_scale 8"),
    "inkling_decode": Workload("inkling_decode", 64, 6144, 3072, b_half_width=0.05, activation="swiglu",
                               route_scale=8.0,
                               description="Inkling config, decode-scale: T=64, d=6144, SwiGLU d_ff=3072, "
                                           "route_scale 8"),
}

ZIPF_S = 1.1


@dataclass(frozen=True)
class LabWorkload:
    """The Router Balance Lab ("Inkling, Dissected" §02g): a frozen router over 64
    experts, top-6, embedding width 32, batches of 2048 tokens for 100 routing
    steps, hard expert capacities of 1.25x the ideal load, tokens drawn from a
    Zipf distribution over expert specialties (expert 0's home cluster about 30
    times as common as expert 63's) and jittered.

    Generator (this module's reading; the lab's own code is not on the page):
    specialty centers c_i ~ N(0, I/d); router row i = alpha * c_i (bf16); token
    t of step s has specialty e ~ P(e) proportional to (e + 1)^-zs with
    64^zs = zipf_ratio, and x = c_e + sigma * N(0, I/d) (bf16).  alpha and sigma
    were chosen so that, with no balancing, the hottest expert sits near twice
    its fair share, as in the page's run."""
    name: str = "lab"
    T: int = 2048
    d: int = 32
    n_routed: int = 64
    n_shared: int = 0
    k: int = 6
    steps: int = 100
    capacity_factor: float = 1.25
    zipf_ratio: float = 30.0
    alpha: float = 4.0
    sigma: float = 0.75
    seed: int = 0
    gammas: tuple = (0.0, 0.01, 0.05)
    description: str = ("Router Balance Lab: 64 experts, top-6, d=32, 2048 tokens x 100 steps, "
                        "Zipf-lumpy tokens, capacity 1.25x ideal")

    @property
    def n_experts(self) -> int:
        return self.n_routed + self.n_shared


LAB = LabWorkload()

SKEW_BETA_PATH = os.path.join(_HERE, "skew_beta.json")


# --------------------------------------------------------------------------
# library loading
# --------------------------------------------------------------------------
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        u64, u32, i32, dbl, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.mi_host_philox_block.argtypes = [u64, u32, u64, vp]
        L.mi_host_philox_raw.argtypes = [vp, vp, vp]
        L.mi_host_words_u32.argtypes = [vp, u64, u64, u32, u64, i32]
        L.mi_host_normal_f64.argtypes = [vp, u64, u64, u32, u64, i32]
        L.mi_host_normal_bf16.argtypes = [vp, u64, u64, u32, u64, dbl, i32]
        L.mi_host_normal_f32.argtypes = [vp, u64, u64, u32, u64, dbl, i32]
        L.mi_host_uniform_f32.argtypes = [vp, u64, u64, u32, u64, dbl, dbl, i32]
        for name in ("mi_gpu_normal_bf16", "mi_gpu_normal_f32"):
            getattr(L, name).argtypes = [vp, u64, u64, u32, u64, dbl, vp]
            getattr(L, name).restype = i32
        L.mi_gpu_uniform_f32.argtypes = [vp, u64, u64, u32, u64, dbl, dbl, vp]
        L.mi_gpu_uniform_f32.restype = i32
        L.mi_gpu_words_u32.argtypes = [vp, u64, u64, u32, u64, vp]
        L.mi_gpu_words_u32.restype = i32
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# --------------------------------------------------------------------------
# host generation (numpy arrays)
# --------------------------------------------------------------------------
def philox_raw(ctr: Sequence[int], key: Sequence[int]) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().mi_host_philox_raw(_ptr(c), _ptr(k), _ptr(out))
    return out


def words(n: int, seed: int, stream: int, offset: int = 0, nthreads: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint32)
    lib().mi_host_words_u32(_ptr(out), n, seed, stream, offset, nthreads)
    return out


def normal_f64(n: int, seed: int, stream: int, offset: int = 0, nthreads: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().mi_host_normal_f64(_ptr(out), n, seed, stream, offset, nthreads)
    return out


def normal_bf16(n: int, seed: int, stream: int, offset: int = 0, std: float = 1.0,
                nthreads: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, std^2) samples."""
    out = np.empty(n, dtype=np.uint16)
    lib().mi_host_normal_bf16(_ptr(out), n, seed, stream, offset, std, nthreads)
    return out


def normal_f32(n: int, seed: int, stream: int, offset: int = 0, std: float = 1.0,
               nthreads: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().mi_host_normal_f32(_ptr(out), n, seed, stream, offset, std, nthreads)
    return out


def uniform_f32(n: int, seed: int, stream: int, lo: float, hi: float, offset: int = 0,
                nthreads: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().mi_host_uniform_f32(_ptr(out), n, seed, stream, offset, lo, hi, nthreads)
    return out


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


# --------------------------------------------------------------------------
# workload tensors, host side (slices on demand)
# --------------------------------------------------------------------------
def host_x(w: Workload, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """x [T, d] (or the given token rows) as bf16 bits."""
    if rows is None:
        return normal_bf16(w.T * w.d, w.seed, STREAM_X, 0, w.std_x).reshape(w.T, w.d)
    out = np.empty((len(rows), w.d), dtype=np.uint16)
    for i, t in enumerate(rows):
        out[i] = normal_bf16(w.d, w.seed, STREAM_X, int(t) * w.d, w.std_x, nthreads=1)
    return out


def host_wr(w: Workload) -> np.ndarray:
    """Router weight [n_routed + n_shared, d], bf16 bits; rows 0..255 routed, 256, 257 shared."""
    return normal_bf16(w.n_experts * w.d, w.seed, STREAM_WR, 0, w.std_wr).reshape(w.n_experts, w.d)


def host_w1(w: Workload, e: int) -> np.ndarray:
    """Expert e's first matrix [d_ff, d] (K-major), bf16 bits; [2 d_ff, d] (gate rows,
    then up rows) for SwiGLU experts."""
    r = w.w1_rows
    return normal_bf16(r * w.d, w.seed, STREAM_W1, e * r * w.d, w.std_w1).reshape(r, w.d)


def host_w2(w: Workload, e: int) -> np.ndarray:
    """Expert e's second matrix [d, d_ff] (K-major), bf16 bits."""
    return normal_bf16(w.d * w.f, w.seed, STREAM_W2, e * w.d * w.f, w.std_w2).reshape(w.d, w.f)


def host_w1_all(w: Workload) -> np.ndarray:
    r = w.w1_rows
    return normal_bf16(w.n_experts * r * w.d, w.seed, STREAM_W1, 0, w.std_w1).reshape(w.n_experts, r, w.d)


def host_w2_all(w: Workload) -> np.ndarray:
    return normal_bf16(w.n_experts * w.d * w.f, w.seed, STREAM_W2, 0, w.std_w2).reshape(w.n_experts, w.d, w.f)


def host_bias(w: Workload) -> np.ndarray:
    """Initial balancing bias b [n_routed] fp32."""
    if w.b_half_width == 0.0:
        return np.zeros(w.n_routed, dtype=np.float32)
    return uniform_f32(w.n_routed, w.seed, STREAM_B, -w.b_half_width, w.b_half_width)


def expert_ranks(w: Workload) -> np.ndarray:
    """Seeded permutation: rank r_i in 1..n_routed of each routed expert."""
    keys = words(w.n_routed, w.seed, STREAM_PERM).astype(np.int64)
    order = np.lexsort((np.arange(w.n_routed), keys))  # by key, ties by index
    ranks = np.empty(w.n_routed, dtype=np.int64)
    ranks[order] = np.arange(1, w.n_routed + 1)
    return ranks


def skew_beta() -> float:
    with open(SKEW_BETA_PATH) as fh:
        return float(json.load(fh)["beta"])


def zipf_offset(w: Workload, beta: float) -> np.ndarray:
    """Per-routed-expert logit offset o_i = -beta * s * ln(rank_i), s = 1.1, fp32."""
    r = expert_ranks(w).astype(np.float64)
    return (-beta * ZIPF_S * np.log(r)).astype(np.float32)


def host_logit_offset(w: Workload) -> Optional[np.ndarray]:
    if not w.skew:
        return None
    return zipf_offset(w, skew_beta())


# --------------------------------------------------------------------------
# device generation (fills caller-owned device buffers by pointer)
# --------------------------------------------------------------------------
def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with status {rc}")


def gpu_normal_bf16(ptr: int, n: int, seed: int, stream_id: int, offset: int, std: float, cuda_stream: int):
    _check(lib().mi_gpu_normal_bf16(ptr, n, seed, stream_id, offset, std, cuda_stream), "mi_gpu_normal_bf16")


def gpu_normal_f32(ptr: int, n: int, seed: int, stream_id: int, offset: int, std: float, cuda_stream: int):
    _check(lib().mi_gpu_normal_f32(ptr, n, seed, stream_id, offset, std, cuda_stream), "mi_gpu_normal_f32")


def gpu_uniform_f32(ptr: int, n: int, seed: int, stream_id: int, offset: int, lo: float, hi: float,
                    cuda_stream: int):
    _check(lib().mi_gpu_uniform_f32(ptr, n, seed, stream_id, offset, lo, hi, cuda_stream), "mi_gpu_uniform_f32")


def gpu_words_u32(ptr: int, n: int, seed: int, stream_id: int, offset: int, cuda_stream: int):
    _check(lib().mi_gpu_words_u32(ptr, n, seed, stream_id, offset, cuda_stream), "mi_gpu_words_u32")


def torch_workload(w: Workload, device="cuda", with_weights: bool = True):
    """Allocate and fill the workload's tensors in device memory (torch), using the
    device generator.  Returns a dict of torch tensors: x, w_r, w1, w2, bias,
    logit_offset (or None)."""
    import torch

    dev = torch.device(device)
    s = torch.cuda.current_stream(dev).cuda_stream
    out = {}
    x = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=dev)
    gpu_normal_bf16(x.data_ptr(), x.numel(), w.seed, STREAM_X, 0, w.std_x, s)
    out["x"] = x
    wr = torch.empty((w.n_experts, w.d), dtype=torch.bfloat16, device=dev)
    gpu_normal_bf16(wr.data_ptr(), wr.numel(), w.seed, STREAM_WR, 0, w.std_wr, s)
    out["w_r"] = wr
    if with_weights:
        w1 = torch.empty((w.n_experts, w.w1_rows, w.d), dtype=torch.bfloat16, device=dev)
        gpu_normal_bf16(w1.data_ptr(), w1.numel(), w.seed, STREAM_W1, 0, w.std_w1, s)
        w2 = torch.empty((w.n_experts, w.d, w.f), dtype=torch.bfloat16, device=dev)
        gpu_normal_bf16(w2.data_ptr(), w2.numel(), w.seed, STREAM_W2, 0, w.std_w2, s)
        out["w1"], out["w2"] = w1, w2
    b = torch.zeros(w.n_routed, dtype=torch.float32, device=dev)
    if w.b_half_width != 0.0:
        gpu_uniform_f32(b.data_ptr(), w.n_routed, w.seed, STREAM_B, 0, -w.b_half_width, w.b_half_width, s)
    out["bias"] = b
    off = host_logit_offset(w)
    out["logit_offset"] = None if off is None else torch.from_numpy(off).to(dev)
    return out


# --------------------------------------------------------------------------
# Router Balance Lab inputs (host side; the GPU path copies these bits)
# --------------------------------------------------------------------------
def lab_centers(w: LabWorkload) -> np.ndarray:
    """Specialty centers c [n_routed, d] (float64), c_i ~ N(0, I/d)."""
    return normal_f64(w.n_routed * w.d, w.seed, STREAM_LAB_CENTERS).reshape(w.n_routed, w.d) / math.sqrt(w.d)


def lab_wr(w: LabWorkload) -> np.ndarray:
    """Frozen router weight [n_routed, d] as bf16 bits: alpha * c."""
    return f32_to_bf16_bits((w.alpha * lab_centers(w)).astype(np.float32))


def lab_specialty(w: LabWorkload, step: int) -> np.ndarray:
    """Each token's specialty at a step: inverse-CDF draw from P(e) ~ (e+1)^-zs."""
    zs = math.log(w.zipf_ratio) / math.log(w.n_routed)
    p = np.arange(1, w.n_routed + 1, dtype=np.float64) ** -zs
    cdf = np.cumsum(p / p.sum())
    u = (words(w.T, w.seed, STREAM_LAB_SPECIALTY, step * w.T).astype(np.float64) + 0.5) / 4294967296.0
    return np.minimum(np.searchsorted(cdf, u, side="right"), w.n_routed - 1).astype(np.int64)


def lab_x(w: LabWorkload, step: int) -> np.ndarray:
    """Tokens [T, d] of a step as bf16 bits: c_e + sigma * N(0, I/d)."""
    c = lab_centers(w)
    jit = normal_f64(w.T * w.d, w.seed, STREAM_LAB_JITTER, step * w.T * w.d).reshape(w.T, w.d)
    x = c[lab_specialty(w, step)] + w.sigma * jit / math.sqrt(w.d)
    return f32_to_bf16_bits(x.astype(np.float32))


def lab_x_all(w: LabWorkload) -> np.ndarray:
    """Tokens of every step, [steps, T, d] bf16 bits."""
    return np.stack([lab_x(w, s) for s in range(w.steps)])
