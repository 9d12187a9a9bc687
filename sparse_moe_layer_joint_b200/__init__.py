"""Python binding of libmoe (the C ABI declared in include/moe.h).

Argument marshalling only: every step of the MoE layer runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (PyTorch supplies device memory
and streams, nothing else); each function takes the same arguments, in the same
order, as its C counterpart, with pointers replaced by tensors and the stream
defaulting to torch's current stream.  A non-zero return code raises MoEError.

Importing this module fails loudly if libmoe.so has not been built; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                      "(there is no non-CUDA implementation of this layer)")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_TIMEOUT = -4
MOE_ERR_DEVICE = -5
MOE_ERR_SCRATCH = -6
MOE_STATUS_TIMEOUT = 0x1
MOE_STATUS_BAD_EXPERT = 0x2
MOE_STATUS_COUNT_MISMATCH = 0x4
MOE_STATUS_RECV_OVERFLOW = 0x8
MOE_ACT_GELU_TANH = 0
MOE_ACT_SWIGLU = 1
MOE_NVFP4_EPI_GELU_FP4 = 0
MOE_NVFP4_EPI_BF16 = 1
MOE_NVFP4_EPI_SWIGLU_FP4 = 2

_vp, _i32, _u64, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_float, ctypes.c_size_t

_lib.moe_router_topk.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp, _vp]
_lib.moe_permute_scratch_bytes.argtypes = [_i32, _i32]
_lib.moe_permute_scratch_bytes.restype = _sz
_lib.moe_permute.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_permute_capped.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.moe_load_stats.argtypes = [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.moe_capacity_for.argtypes = [ctypes.c_longlong, ctypes.c_longlong, _i32, _i32, _i32]
_lib.moe_capacity_for.restype = ctypes.c_longlong
_lib.moe_permute_noalloc.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]
_lib.moe_grouped_ffn.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.moe_experts_ffn.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _vp, _vp,
                                 _vp, _vp]
_lib.moe_combine.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp]
_lib.moe_bias_update.argtypes = [_vp, _i32, _i32, _i32, _f32, _vp, _vp]
_i64 = ctypes.c_longlong
_lib.moe_nvfp4_quantize_weights.argtypes = [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp]
_lib.moe_nvfp4_rows_capacity.argtypes = [_i32, _i32, _i32]
_lib.moe_nvfp4_rows_capacity.restype = _i64
_lib.moe_nvfp4_dispatch.argtypes = [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]
_lib.moe_nvfp4_grouped_gemm.argtypes = [_vp, _vp, _vp, _i32, _i64, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp,
                                        _vp, _i64, _vp]
_lib.moe_ep_plan.argtypes = [_vp, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.moe_ep_dispatch.argtypes = [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp]
_lib.moe_ep_combine.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i64, _vp,
                                _vp]
_lib.moe_ipc_handle_bytes.argtypes = []
_lib.moe_ipc_get_handle.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_ulonglong)]
_lib.moe_ipc_open.argtypes = [_vp, ctypes.c_ulonglong, ctypes.POINTER(_vp)]
_lib.moe_ipc_close.argtypes = [_vp]
_lib.moe_status_string.argtypes = [_i32]
_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_get_status.argtypes = [_vp, ctypes.POINTER(_i32)]
_lib.moe_set_wait_timeout_ns.argtypes = [_u64]
_lib.moe_debug_bounded_wait.argtypes = [_u64, _vp]
for _f in ("moe_router_topk", "moe_permute", "moe_permute_capped", "moe_permute_noalloc", "moe_grouped_ffn",
           "moe_experts_ffn", "moe_combine", "moe_bias_update", "moe_load_stats", "moe_get_status",
           "moe_nvfp4_quantize_weights", "moe_nvfp4_dispatch", "moe_nvfp4_grouped_gemm",
           "moe_set_wait_timeout_ns", "moe_debug_bounded_wait", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_combine",
           "moe_ipc_handle_bytes", "moe_ipc_get_handle", "moe_ipc_open", "moe_ipc_close"):
    getattr(_lib, _f).restype = _i32


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code}: {status_string(code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    return _lib


def header_functions() -> list:
    """Names of the functions include/moe.h declares."""
    with open(HEADER_PATH) as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:[a-z_0-9]+\s+)*[a-z_0-9]+\s*\*?\s*(moe_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


def header_arity() -> dict:
    """Number of parameters of each function include/moe.h declares."""
    with open(HEADER_PATH) as fh:
        text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"(moe_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def status_string(code: int) -> str:
    return _lib.moe_status_string(int(code)).decode()


def _p(t) -> Optional[int]:
    """Device address of a tensor (or an int address); None for None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoEError(fn, rc)
    if _DEBUG_SYNC:
        _debug_sync(fn)


# MOE_DEBUG_SYNC=1: after every call, synchronise the device and read the device status word, so
# a device-side error is reported at the call that caused it (slow; off by default).
_DEBUG_SYNC = os.environ.get("MOE_DEBUG_SYNC") == "1"


def _debug_sync(fn: str):
    import torch

    # the call may have run on any stream (MoELayer uses a side stream too): wait for the whole
    # device, so the status read sees this call's kernels and its reset races no running kernel
    torch.cuda.synchronize()
    v = _i32(0)
    rc = _lib.moe_get_status(None, ctypes.byref(v))
    if rc != MOE_OK or v.value != 0:
        raise MoEError(f"{fn} (device status {v.value:#x})", rc if rc != MOE_OK else MOE_ERR_DEVICE)


# ---------------------------------------------------------------------------
# the five calls of the layer, same names and argument order as the C ABI
# ---------------------------------------------------------------------------
def moe_router_topk(x, w_router, bias, logit_offset, T: int, d: int, n_routed: int, n_shared: int, top_k: int,
                    route_scale: float, topk_idx, gates, counts, scores_out=None, stream=None):
    _check("moe_router_topk", _lib.moe_router_topk(
        _p(x), _p(w_router), _p(bias), _p(logit_offset), T, d, n_routed, n_shared, top_k, route_scale,
        _p(topk_idx), _p(gates), _p(counts), _p(scores_out), _stream(stream)))


def moe_permute_scratch_bytes(T: int, n_routed: int) -> int:
    return int(_lib.moe_permute_scratch_bytes(T, n_routed))


def moe_permute(x, topk_idx, counts, T: int, d: int, n_routed: int, top_k: int, offsets, x_perm, row_token,
                token_row, scratch, scratch_bytes: int, stream=None):
    _check("moe_permute", _lib.moe_permute(
        _p(x), _p(topk_idx), _p(counts), T, d, n_routed, top_k, _p(offsets), _p(x_perm), _p(row_token),
        _p(token_row), _p(scratch), scratch_bytes, _stream(stream)))


def moe_permute_capped(x, topk_idx, counts, T: int, d: int, n_routed: int, top_k: int, capacity: int, offsets,
                       x_perm, row_token, token_row, scratch, scratch_bytes: int, stream=None):
    _check("moe_permute_capped", _lib.moe_permute_capped(
        _p(x), _p(topk_idx), _p(counts), T, d, n_routed, top_k, capacity, _p(offsets), _p(x_perm), _p(row_token),
        _p(token_row), _p(scratch), scratch_bytes, _stream(stream)))


def moe_permute_noalloc(x, topk_idx, counts, T: int, d: int, n_routed: int, top_k: int, offsets, x_perm, row_token,
                        token_row, stream=None):
    """moe_permute without a scratch argument, for callers that cannot allocate
    device memory: the scratch is a fixed 1 MiB device array inside libmoe
    (limit: moe_permute_scratch_bytes(T, n_routed) <= 1 MiB).  Calls on one
    device share that array, so calls that could overlap on the GPU must be
    ordered; the first call on a device should come before any stream capture."""
    _check("moe_permute_noalloc", _lib.moe_permute_noalloc(
        _p(x), _p(topk_idx), _p(counts), T, d, n_routed, top_k, _p(offsets), _p(x_perm), _p(row_token),
        _p(token_row), _stream(stream)))


def moe_grouped_ffn(rows, offsets, n_groups: int, n_rows: int, expert_base: int, w1, w2, d: int, d_ff: int,
                    activation: int, h_scratch, y, stream=None):
    _check("moe_grouped_ffn", _lib.moe_grouped_ffn(
        _p(rows), _p(offsets), n_groups, n_rows, expert_base, _p(w1), _p(w2), d, d_ff, activation, _p(h_scratch),
        _p(y), _stream(stream)))


def moe_experts_ffn(x, x_perm, row_token, offsets, T: int, n_routed: int, n_shared: int, top_k: int, w1, w2, d: int,
                    d_ff: int, activation: int, h_scratch, y_perm, y_shared, stream=None):
    _check("moe_experts_ffn", _lib.moe_experts_ffn(
        _p(x), _p(x_perm), _p(row_token), _p(offsets), T, n_routed, n_shared, top_k, _p(w1), _p(w2), d, d_ff,
        activation, _p(h_scratch), _p(y_perm), _p(y_shared), _stream(stream)))


def moe_combine(y_perm, token_row, gates, y_shared, T: int, d: int, top_k: int, n_shared: int, out, stream=None):
    _check("moe_combine", _lib.moe_combine(
        _p(y_perm), _p(token_row), _p(gates), _p(y_shared), T, d, top_k, n_shared, _p(out), _stream(stream)))


def moe_bias_update(counts, n_routed: int, T: int, top_k: int, gamma: float, bias, stream=None):
    _check("moe_bias_update", _lib.moe_bias_update(_p(counts), n_routed, T, top_k, gamma, _p(bias), _stream(stream)))


def moe_load_stats(counts, n_routed: int, T: int, top_k: int, capacity: int, stats, metrics=None, stream=None):
    _check("moe_load_stats", _lib.moe_load_stats(_p(counts), n_routed, T, top_k, capacity, _p(stats), _p(metrics),
                                                 _stream(stream)))


def moe_capacity_for(factor_num: int, factor_den: int, T: int, top_k: int, n_routed: int) -> int:
    c = int(_lib.moe_capacity_for(int(factor_num), int(factor_den), T, top_k, n_routed))
    if c < 0:
        raise MoEError("moe_capacity_for", c)
    return c


def moe_nvfp4_quantize_weights(w, G: int, N: int, K: int, q, sf, gscale, stream=None):
    _check("moe_nvfp4_quantize_weights", _lib.moe_nvfp4_quantize_weights(
        _p(w), G, N, K, _p(q), _p(sf), _p(gscale), _stream(stream)))


def moe_nvfp4_rows_capacity(T: int, n_routed: int, top_k: int) -> int:
    return int(_lib.moe_nvfp4_rows_capacity(T, n_routed, top_k))


def moe_nvfp4_dispatch(x, topk_idx, token_row, offsets, T: int, d: int, n_routed: int, top_k: int, xq, xsf,
                       token_row_pad, offsets_pad, stream=None):
    _check("moe_nvfp4_dispatch", _lib.moe_nvfp4_dispatch(
        _p(x), _p(topk_idx), _p(token_row), _p(offsets), T, d, n_routed, top_k, _p(xq), _p(xsf), _p(token_row_pad),
        _p(offsets_pad), _stream(stream)))


def moe_nvfp4_grouped_gemm(aq, asf, offsets_pad, n_groups: int, rows_cap: int, wq, wsf, gscale, N: int, K: int,
                           epilogue: int, out_q, out_sf, out, offsets_out, out_rows: int, stream=None):
    _check("moe_nvfp4_grouped_gemm", _lib.moe_nvfp4_grouped_gemm(
        _p(aq), _p(asf), _p(offsets_pad), n_groups, rows_cap, _p(wq), _p(wsf), _p(gscale), N, K, epilogue,
        _p(out_q), _p(out_sf), _p(out), _p(offsets_out), out_rows, _stream(stream)))


# ---------------------------------------------------------------------------
# expert parallelism over peer memory (moe_ep_*) and the peer mappings (moe_ipc_*)
# ---------------------------------------------------------------------------
def moe_ep_plan(counts_all, rank: int, world: int, n_routed: int, send_base, recv_offsets, stream=None):
    _check("moe_ep_plan", _lib.moe_ep_plan(_p(counts_all), rank, world, n_routed, _p(send_base), _p(recv_offsets),
                                           _stream(stream)))


def moe_ep_dispatch(x, topk_idx, token_row, offsets, send_base, T: int, d: int, n_routed: int, top_k: int,
                    world: int, recv_x, recv_rows: int, stream=None):
    """recv_x: a device tensor of ``world`` int64 device addresses (rank q's receive buffer)."""
    _check("moe_ep_dispatch", _lib.moe_ep_dispatch(
        _p(x), _p(topk_idx), _p(token_row), _p(offsets), _p(send_base), T, d, n_routed, top_k, world, _p(recv_x),
        int(recv_rows), _stream(stream)))


def moe_ep_combine(recv_y, topk_idx, token_row, offsets, send_base, gates, y_shared, T: int, d: int, n_routed: int,
                   top_k: int, n_shared: int, world: int, recv_rows: int, out, stream=None):
    """recv_y: a device tensor of ``world`` int64 device addresses (rank q's output buffer)."""
    _check("moe_ep_combine", _lib.moe_ep_combine(
        _p(recv_y), _p(topk_idx), _p(token_row), _p(offsets), _p(send_base), _p(gates), _p(y_shared), T, d, n_routed,
        top_k, n_shared, world, int(recv_rows), _p(out), _stream(stream)))


def moe_ipc_get_handle(t):
    """(handle bytes, byte offset) of the device allocation holding tensor t's data."""
    n = int(_lib.moe_ipc_handle_bytes())
    buf = ctypes.create_string_buffer(n)
    off = ctypes.c_ulonglong(0)
    _check("moe_ipc_get_handle", _lib.moe_ipc_get_handle(_p(t), buf, ctypes.byref(off)))
    return buf.raw, int(off.value)


def moe_ipc_open(handle: bytes, offset: int) -> int:
    """Map a peer process's allocation; returns the device address of its data in this process."""
    ptr = _vp()
    buf = ctypes.create_string_buffer(bytes(handle), len(handle))
    _check("moe_ipc_open", _lib.moe_ipc_open(buf, int(offset), ctypes.byref(ptr)))
    return int(ptr.value)


def moe_ipc_close(ptr: int):
    _check("moe_ipc_close", _lib.moe_ipc_close(int(ptr)))


def capacity_for(factor: float, T: int, k: int, n_routed: int) -> int:
    """Expert capacity in tokens (moe_capacity_for), the Python float factor passed
    as the exact fraction of the decimal it prints as (1.25 -> 5/4)."""
    from fractions import Fraction
    q = Fraction(repr(float(factor)))
    return moe_capacity_for(q.numerator, q.denominator, T, k, n_routed)


def moe_get_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status bits."""
    v = _i32(0)
    rc = _lib.moe_get_status(_stream(stream), ctypes.byref(v))
    if rc not in (MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE):
        raise MoEError("moe_get_status", rc)
    return v.value


def moe_set_wait_timeout_ns(ns: int):
    _check("moe_set_wait_timeout_ns", _lib.moe_set_wait_timeout_ns(int(ns)))


def moe_debug_bounded_wait(timeout_ns: int, stream=None):
    _check("moe_debug_bounded_wait", _lib.moe_debug_bounded_wait(int(timeout_ns), _stream(stream)))


# ---------------------------------------------------------------------------
# host orchestration of one layer forward: the calls above, in the pages'
# order, on two streams (shared experts beside the routed path)
# ---------------------------------------------------------------------------
@dataclass
class LayerShape:
    T: int
    d: int
    d_ff: int
    n_routed: int = 256
    n_shared: int = 2
    top_k: int = 6


class MoELayer:
    """Device buffers for one layer shape and the call sequence of a forward.

    Weights are caller-owned torch tensors: w_router [n_routed + n_shared, d],
    w1 [n_routed + n_shared, d_ff, d] (``activation="swiglu"``: [n_routed + n_shared,
    2*d_ff, d], gate rows then up rows), w2 [n_routed + n_shared, d, d_ff] (bf16),
    bias [n_routed] fp32 (updated in place by ``bias_update``).  ``route_scale``
    multiplies the joint routing weights (route_scale x global_scale of the released
    configuration; 1 keeps them summing to 1).
    """

    def __init__(self, shape: LayerShape, device="cuda", fused_experts: bool = True, gather_rows: bool = False,
                 capacity_factor: Optional[float] = None, activation: str = "gelu_tanh", route_scale: float = 1.0,
                 precision: str = "bf16"):
        import torch

        self.shape = s = shape
        # "nvfp4": the routed experts in NVFP4 (W4A4, quantized weights set by set_nvfp4_weights);
        # the router and the shared experts stay bf16
        if precision not in ("bf16", "nvfp4"):
            raise ValueError(precision)
        self.nvfp4 = precision == "nvfp4"
        # expert type: GELU MLP (w1 [E, d_ff, d]) or SwiGLU (w1 [E, 2*d_ff, d]: gate rows, then up rows)
        self.activation = {"gelu_tanh": MOE_ACT_GELU_TANH, "swiglu": MOE_ACT_SWIGLU}[activation]
        # multiplier of the joint routing weights (route_scale x global_scale of the released config)
        self.route_scale = float(route_scale)
        # hard expert capacity (tokens per expert per batch); None: every assignment is served
        self.capacity = None if capacity_factor is None else capacity_for(capacity_factor, s.T, s.top_k, s.n_routed)
        self.fused_experts = fused_experts
        # with the fused experts, GEMM1 can gather the routed rows from x itself (TMA tile::gather4
        # loads, no x_perm copy); measured slower on B200 (at prefill size GEMM1 took 1.65x as long:
        # 32 four-row gathers per stage bound the TMA unit), so the default copies the rows in
        # moe_permute and loads whole tiles
        self.gather_rows = gather_rows and fused_experts
        dev = torch.device(device)
        R = s.T * s.top_k
        bf = torch.bfloat16
        self.topk_idx = torch.empty((s.T, s.top_k), dtype=torch.int32, device=dev)
        self.gates = torch.empty((s.T, s.top_k + s.n_shared), dtype=torch.float32, device=dev)
        self.counts = torch.empty((s.n_routed,), dtype=torch.int32, device=dev)
        self.offsets = torch.empty((s.n_routed + 1,), dtype=torch.int32, device=dev)
        # the bf16 path's copied rows and hidden rows (the NVFP4 path keeps its own FP4 buffers)
        R_bf16 = 1 if self.nvfp4 else max(R, 1)
        self.x_perm = torch.empty((R_bf16, s.d), dtype=bf, device=dev)
        self.row_token = torch.empty((max(R, 1),), dtype=torch.int32, device=dev)
        self.token_row = torch.empty((s.T, s.top_k), dtype=torch.int32, device=dev)
        self.scratch_bytes = moe_permute_scratch_bytes(s.T, s.n_routed)
        self.scratch = torch.empty((self.scratch_bytes,), dtype=torch.uint8, device=dev)
        # hidden rows: routed rows, then (fused path) the shared experts' rows
        self.h = torch.empty((1 if self.nvfp4 else max(R + s.n_shared * s.T, 1), s.d_ff), dtype=bf, device=dev)
        self.y_perm = torch.empty((max(R, 1), s.d), dtype=bf, device=dev)
        self.h_shared = torch.empty((max(s.n_shared, 1), s.T, s.d_ff), dtype=bf, device=dev)
        self.y_shared = torch.empty((max(s.n_shared, 1), s.T, s.d), dtype=bf, device=dev)
        self.out = torch.empty((s.T, s.d), dtype=bf, device=dev)
        # moe_load_stats output: max load and dropped assignments (int32), then MaxVio and the drop rate (fp32 bits)
        self.stats = torch.zeros((4,), dtype=torch.int32, device=dev)
        if self.nvfp4:
            self.rows_cap = moe_nvfp4_rows_capacity(s.T, s.n_routed, s.top_k)
            u8 = torch.uint8
            self.xq = torch.empty((self.rows_cap, s.d // 2), dtype=u8, device=dev)
            self.xsf = torch.empty((self.rows_cap * s.d // 16,), dtype=u8, device=dev)
            self.hq = torch.empty((self.rows_cap, s.d_ff // 2), dtype=u8, device=dev)
            self.hsf = torch.empty((self.rows_cap * s.d_ff // 16,), dtype=u8, device=dev)
            self.token_row_pad = torch.empty((s.T, s.top_k), dtype=torch.int32, device=dev)
            self.offsets_pad = torch.empty((s.n_routed + 1,), dtype=torch.int32, device=dev)
            self.w1q = self.w1sf = self.g1 = self.w2q = self.w2sf = self.g2 = None
        self.side = torch.cuda.Stream(device=dev)
        self.ev_start = torch.cuda.Event()
        self.ev_shared = torch.cuda.Event()

    def set_nvfp4_weights(self, w1, w2, stream=None):
        """Quantize the routed experts' weights (the first n_routed of w1 [E, d_ff, d] -- [E, 2*d_ff, d]
        for SwiGLU, one quantized matrix per expert -- and w2 [E, d, d_ff]) to NVFP4 on the device; the
        shared experts keep using w1, w2."""
        import torch

        s = self.shape
        dev = w1.device
        E, f, d = s.n_routed, s.d_ff, s.d
        f1 = 2 * f if self.activation == MOE_ACT_SWIGLU else f  # rows of each W1
        self.w1q = torch.empty((E, f1, d // 2), dtype=torch.uint8, device=dev)
        self.w1sf = torch.empty((E, f1 * d // 16), dtype=torch.uint8, device=dev)
        self.g1 = torch.empty((E,), dtype=torch.float32, device=dev)
        self.w2q = torch.empty((E, d, f // 2), dtype=torch.uint8, device=dev)
        self.w2sf = torch.empty((E, d * f // 16), dtype=torch.uint8, device=dev)
        self.g2 = torch.empty((E,), dtype=torch.float32, device=dev)
        moe_nvfp4_quantize_weights(w1, E, f1, d, self.w1q, self.w1sf, self.g1, stream=stream)
        moe_nvfp4_quantize_weights(w2, E, d, f, self.w2q, self.w2sf, self.g2, stream=stream)

    def _forward_nvfp4(self, x, w1, w2, main, ffn_events=None):
        s = self.shape
        T, d, f, k = s.T, s.d, s.d_ff, s.top_k
        if self.w1q is None:
            raise RuntimeError("set_nvfp4_weights() first")
        moe_nvfp4_dispatch(x, self.topk_idx, self.token_row, self.offsets, T, d, s.n_routed, k, self.xq, self.xsf,
                           self.token_row_pad, self.offsets_pad, stream=main)
        if ffn_events is not None:
            ffn_events[0].record(main)
        epi1 = MOE_NVFP4_EPI_SWIGLU_FP4 if self.activation == MOE_ACT_SWIGLU else MOE_NVFP4_EPI_GELU_FP4
        moe_nvfp4_grouped_gemm(self.xq, self.xsf, self.offsets_pad, s.n_routed, self.rows_cap, self.w1q, self.w1sf,
                               self.g1, f, d, epi1, self.hq, self.hsf, None, self.offsets, T * k, stream=main)
        moe_nvfp4_grouped_gemm(self.hq, self.hsf, self.offsets_pad, s.n_routed, self.rows_cap, self.w2q, self.w2sf,
                               self.g2, d, f, MOE_NVFP4_EPI_BF16, None, None, self.y_perm, self.offsets, T * k,
                               stream=main)
        if ffn_events is not None:
            ffn_events[1].record(main)
        if s.n_shared > 0:
            moe_grouped_ffn(x, None, s.n_shared, T, s.n_routed, w1, w2, d, f, self.activation, self.h_shared,
                            self.y_shared, stream=main)

    def forward(self, x, w_router, w1, w2, bias, logit_offset=None, stream=None, scores_out=None,
                ffn_events=None, out=None):
        """Router -> dispatch -> experts -> combine, on the given (default: current) stream.

        With ``fused_experts`` (default) the routed and shared experts run in one
        pair of grouped-GEMM launches (moe_experts_ffn).  Otherwise the shared
        experts run beside dispatch and the routed experts on a second stream
        (moe_grouped_ffn twice).  ``ffn_events`` = (start, end) torch events
        recorded around the expert launches on the main stream.  ``out``: a [T, d]
        bf16 tensor to write the result into (default: this layer's own buffer)."""
        import torch

        s = self.shape
        main = stream if stream is not None else torch.cuda.current_stream()
        T, d, f, k = s.T, s.d, s.d_ff, s.top_k
        side = s.n_shared > 0 and not self.fused_experts and not self.nvfp4
        if side:
            # the shared experts need only x: their stream starts with the router, and the
            # dispatch kernels (small, memory-bound) run beside their GEMM tiles
            self.ev_start.record(main)
            self.side.wait_event(self.ev_start)
        moe_router_topk(x, w_router, bias, logit_offset, T, d, s.n_routed, s.n_shared, k, self.route_scale,
                        self.topk_idx, self.gates, self.counts, scores_out, stream=main)
        if side:
            moe_grouped_ffn(x, None, s.n_shared, T, s.n_routed, w1, w2, d, f, self.activation, self.h_shared,
                            self.y_shared, stream=self.side)
            self.ev_shared.record(self.side)
        x_perm = None if (self.gather_rows or self.nvfp4) else self.x_perm
        if self.capacity is None:
            moe_permute(x, self.topk_idx, self.counts, T, d, s.n_routed, k, self.offsets, x_perm, self.row_token,
                        self.token_row, self.scratch, self.scratch_bytes, stream=main)
        else:
            moe_permute_capped(x, self.topk_idx, self.counts, T, d, s.n_routed, k, self.capacity, self.offsets,
                               x_perm, self.row_token, self.token_row, self.scratch, self.scratch_bytes, stream=main)
        if ffn_events is not None and not self.nvfp4:
            ffn_events[0].record(main)
        if self.nvfp4:  # its events bracket the two FP4 GEMMs alone
            self._forward_nvfp4(x, w1, w2, main, ffn_events)
        elif self.fused_experts:
            moe_experts_ffn(x, x_perm, self.row_token, self.offsets, T, s.n_routed, s.n_shared, k, w1, w2, d, f,
                            self.activation, self.h, self.y_perm, self.y_shared, stream=main)
        else:
            moe_grouped_ffn(self.x_perm, self.offsets, s.n_routed, T * k, 0, w1, w2, d, f, self.activation,
                            self.h, self.y_perm, stream=main)
        if ffn_events is not None and not self.nvfp4:
            ffn_events[1].record(main)
        if side:
            main.wait_event(self.ev_shared)
        dst = self.out if out is None else out
        moe_combine(self.y_perm, self.token_row, self.gates, self.y_shared if s.n_shared > 0 else None, T, d, k,
                    s.n_shared, dst, stream=main)
        return dst

    # kernels of libmoe launched by one forward + bias update
    def launches_per_step(self) -> int:
        """libmoe kernels one forward + bias update launches."""
        one_chunk = self.shape.T <= 256 and os.environ.get("MOE_PERMUTE_ONE_CHUNK") != "0"
        indices = 1 if one_chunk else 3  # the dispatch's index launches (one CTA when one chunk holds every token)
        if self.nvfp4:  # permute (indices), FP4 dispatch 1, FP4 GEMMs 2, shared bf16 GEMMs 2
            return 1 + indices + 1 + 2 + 2 + 1 + 1
        experts = 2 if self.fused_experts else 4
        permute = indices + (0 if self.gather_rows else 1)
        return 1 + permute + experts + 1 + 1

    def balance(self, stream=None) -> dict:
        """MaxVio and drop rate of the last forward's loads (synchronises the stream).  With
        data-parallel replicas call it before ``dp.bias_step``, which sums the counts over the
        ranks in place: it describes this rank's batch."""
        import torch

        s = self.shape
        cap = self.capacity if self.capacity is not None else 2 ** 31 - 1
        st = stream if stream is not None else torch.cuda.current_stream()
        moe_load_stats(self.counts, s.n_routed, s.T, s.top_k, cap, self.stats[:2], self.stats[2:].view(torch.float32),
                       stream=st)
        host = self.stats.cpu()
        max_load, dropped = (int(v) for v in host[:2].tolist())
        max_vio, drop_rate = (float(v) for v in host[2:].view(torch.float32).tolist())
        return {"max_load": max_load, "dropped": dropped, "max_vio": max_vio, "drop_rate": drop_rate}

    def bias_update(self, bias, gamma: float, stream=None, T_total: Optional[int] = None):
        """b += gamma * sign(Lbar - L) from this layer's counts; T_total: the batch's token
        count when the counts were summed over data-parallel ranks (default: this layer's T)."""
        s = self.shape
        moe_bias_update(self.counts, s.n_routed, s.T if T_total is None else T_total, s.top_k, gamma, bias,
                        stream=stream)


# MOE_NVTX=1: every moe_* call above is bracketed by an NVTX range named after it (for timelines
# in a profiler; off by default, when the functions are left untouched).
def _nvtx_wrap(fn):
    import functools

    import torch

    @functools.wraps(fn)
    def wrapped(*args, **kwargs):
        torch.cuda.nvtx.range_push(fn.__name__)
        try:
            return fn(*args, **kwargs)
        finally:
            torch.cuda.nvtx.range_pop()

    return wrapped


if os.environ.get("MOE_NVTX") == "1":
    for _name in [n for n in list(globals()) if n.startswith("moe_") and callable(globals()[n])]:
        globals()[_name] = _nvtx_wrap(globals()[_name])
