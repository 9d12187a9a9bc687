"""The C ABI without a GPU: the library loads, exports every function
include/moe.h declares, and rejects bad arguments on the host (nothing is
launched for a call that fails validation, so these run on a CPU-only box)."""
import ctypes

import pytest

import oracle
import sparse_moe_layer_joint_b200 as moe

NULL = None
A16 = 0x10000      # a 16-byte aligned, never dereferenced fake device address
MIS = 0x10004      # misaligned by 4


def test_every_declared_function_is_exported():
    names = moe.header_functions()
    assert {"moe_router_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_bias_update"} <= set(names)
    for n in names:
        assert hasattr(moe.lib(), n), n


def test_status_strings():
    for code in (moe.MOE_OK, moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_UNSUPPORTED, moe.MOE_ERR_CUDA,
                 moe.MOE_ERR_TIMEOUT, moe.MOE_ERR_DEVICE, moe.MOE_ERR_SCRATCH):
        assert moe.status_string(code) and moe.status_string(code) != "unknown status"
    assert moe.status_string(12345) == "unknown status"


def test_permute_scratch_size():
    assert moe.moe_permute_scratch_bytes(0, 256) >= 0
    a = moe.moe_permute_scratch_bytes(65536, 256)
    assert a >= 2 * 256 * 256 * 4
    assert moe.moe_permute_scratch_bytes(257, 256) > moe.moe_permute_scratch_bytes(256, 256)


L = moe.lib()


def router(**kw):
    a = dict(x=A16, w=A16, b=A16, off=NULL, T=4, d=64, nr=256, ns=2, k=6, rs=1.0, idx=A16, g=A16, c=A16, sc=NULL,
             s=NULL)
    a.update(kw)
    return L.moe_router_topk(a["x"], a["w"], a["b"], a["off"], a["T"], a["d"], a["nr"], a["ns"], a["k"], a["rs"],
                             a["idx"], a["g"], a["c"], a["sc"], a["s"])


@pytest.mark.parametrize("kw,code", [
    (dict(x=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(x=MIS), moe.MOE_ERR_INVALID_ARG),
    (dict(w=MIS), moe.MOE_ERR_INVALID_ARG),
    (dict(c=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(off=0x10002), moe.MOE_ERR_INVALID_ARG),
    (dict(k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(k=9), moe.MOE_ERR_INVALID_ARG),
    (dict(nr=4, k=5), moe.MOE_ERR_INVALID_ARG),
    (dict(T=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(d=100), moe.MOE_ERR_UNSUPPORTED),
    (dict(nr=300), moe.MOE_ERR_UNSUPPORTED),
    (dict(ns=9), moe.MOE_ERR_UNSUPPORTED),
    (dict(d=36), moe.MOE_ERR_UNSUPPORTED),
    (dict(rs=0.0), moe.MOE_ERR_INVALID_ARG),
    (dict(rs=-8.0), moe.MOE_ERR_INVALID_ARG),
    (dict(rs=float("nan")), moe.MOE_ERR_INVALID_ARG),
    (dict(rs=float("inf")), moe.MOE_ERR_INVALID_ARG),
])
def test_router_rejects(kw, code):
    assert router(**kw) == code


def test_permute_rejects():
    ok = dict(x=A16, idx=A16, cnt=NULL, T=8, d=64, nr=256, k=6, off=A16, xp=A16, rt=A16, tr=A16, scr=A16,
              sb=1 << 20, s=NULL)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.moe_permute(a["x"], a["idx"], a["cnt"], a["T"], a["d"], a["nr"], a["k"], a["off"], a["xp"],
                             a["rt"], a["tr"], a["scr"], a["sb"], a["s"])

    assert call(x=NULL) == moe.MOE_ERR_INVALID_ARG
    assert call(xp=MIS) == moe.MOE_ERR_INVALID_ARG
    assert call(tr=NULL) == moe.MOE_ERR_INVALID_ARG
    assert call(k=9) == moe.MOE_ERR_INVALID_ARG
    assert call(d=12) == moe.MOE_ERR_UNSUPPORTED
    assert call(sb=16) == moe.MOE_ERR_SCRATCH
    assert call(scr=NULL) == moe.MOE_ERR_INVALID_ARG


def test_grouped_ffn_rejects_and_empty_is_noop():
    def call(rows=A16, off=A16, G=256, n=100, base=0, w1=A16, w2=A16, d=64, f=64, act=0, h=A16, y=A16):
        return L.moe_grouped_ffn(rows, off, G, n, base, w1, w2, d, f, act, h, y, NULL)

    assert call(rows=NULL) == moe.MOE_ERR_INVALID_ARG
    assert call(w1=MIS) == moe.MOE_ERR_INVALID_ARG
    assert call(act=3) == moe.MOE_ERR_INVALID_ARG
    assert call(d=96) == moe.MOE_ERR_UNSUPPORTED
    assert call(f=100) == moe.MOE_ERR_UNSUPPORTED
    assert call(G=5000) == moe.MOE_ERR_UNSUPPORTED
    assert call(n=-1) == moe.MOE_ERR_INVALID_ARG
    # no rows or no groups: nothing to do, nothing launched
    assert call(n=0) == moe.MOE_OK
    assert call(G=0) == moe.MOE_OK


def test_experts_ffn_rejects():
    def call(x=A16, xp=A16, rt=A16, off=A16, T=64, nr=256, ns=2, k=6, w1=A16, w2=A16, d=64, f=64, act=0, h=A16,
             yp=A16, ys=A16):
        return L.moe_experts_ffn(x, xp, rt, off, T, nr, ns, k, w1, w2, d, f, act, h, yp, ys, NULL)

    assert call(xp=NULL, rt=NULL) == moe.MOE_ERR_INVALID_ARG   # gathering needs row_token
    assert call(xp=0x10008) == moe.MOE_ERR_INVALID_ARG
    assert call(ys=NULL) == moe.MOE_ERR_INVALID_ARG
    assert call(off=0x10002) == moe.MOE_ERR_INVALID_ARG
    assert call(d=96) == moe.MOE_ERR_UNSUPPORTED
    assert call(nr=1024, ns=8) == moe.MOE_ERR_UNSUPPORTED
    assert call(k=0) == moe.MOE_ERR_INVALID_ARG
    assert call(T=0) == moe.MOE_OK
    assert call(nr=0, ns=0) == moe.MOE_OK


def test_combine_and_bias_update_reject():
    assert L.moe_combine(A16, A16, A16, NULL, 4, 64, 6, 2, A16, NULL) == moe.MOE_ERR_INVALID_ARG  # y_shared missing
    assert L.moe_combine(A16, A16, A16, A16, 4, 60, 6, 2, A16, NULL) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_combine(MIS, A16, A16, A16, 4, 64, 6, 2, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(A16, A16, A16, A16, 0, 64, 6, 2, A16, NULL) == moe.MOE_OK   # T = 0
    assert L.moe_bias_update(NULL, 256, 4, 6, 1e-3, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_bias_update(A16, 0, 4, 6, 1e-3, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_bias_update(A16, 256, 4, 6, float("nan"), A16, NULL) == moe.MOE_ERR_INVALID_ARG


def test_wait_timeout_setting():
    assert L.moe_set_wait_timeout_ns(0) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_set_wait_timeout_ns(2_000_000_000) == moe.MOE_OK
    assert L.moe_debug_bounded_wait(0, NULL) == moe.MOE_ERR_INVALID_ARG


def test_ffn_rejects_unknown_activation():
    for act in (2, -1, 99):
        assert L.moe_grouped_ffn(A16, NULL, 2, 8, 0, A16, A16, 64, 64, act, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
        assert L.moe_experts_ffn(A16, A16, A16, A16, 8, 4, 2, 2, A16, A16, 64, 64, act, A16, A16, A16,
                                 NULL) == moe.MOE_ERR_INVALID_ARG


def test_capacity_and_stats_reject():
    assert L.moe_permute_capped(A16, A16, NULL, 8, 64, 256, 6, -1, A16, A16, A16, A16, A16, 1 << 20,
                                NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_permute_capped(A16, A16, NULL, 8, 64, 256, 6, 5, A16, A16, A16, A16, A16, 16,
                                NULL) == moe.MOE_ERR_SCRATCH
    assert L.moe_load_stats(A16, 256, 64, 6, -3, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_load_stats(A16, 257, 64, 6, 3, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_load_stats(NULL, 256, 64, 6, 3, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_load_stats(0x10002, 256, 64, 6, 3, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_load_stats(A16, 256, -1, 6, 3, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_load_stats(A16, 256, 64, 0, 3, A16, A16, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_load_stats(A16, 256, 64, 6, 3, A16, 0x10002, NULL) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("factor,T,k,E", [(1.25, 2048, 6, 64), (1.25, 65536, 6, 256), (1.25, 100, 6, 64),
                                          (1.0, 256, 6, 256), (1.1, 1000, 1, 10), (0.0, 500, 6, 256),
                                          (2.5, 1, 6, 256), (1.3333, 4096, 8, 7)])
def test_capacity_for_matches_the_oracle(factor, T, k, E):
    """moe_capacity_for (exact integer floor of factor * k*T / n_routed) against the oracle's
    definition, with the Python float factor passed as the fraction of its decimal form."""
    assert moe.capacity_for(factor, T, k, E) == oracle.capacity_for(factor, T, k, E)


def test_capacity_for_rejects_and_clamps():
    assert L.moe_capacity_for(5, 0, 10, 6, 64) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_capacity_for(-1, 4, 10, 6, 64) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_capacity_for(5, 4, -1, 6, 64) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_capacity_for(5, 4, 10, 0, 64) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_capacity_for(5, 4, 10, 6, 0) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_capacity_for(10 ** 12, 1, 2 ** 31 - 1, 8, 1) == 2 ** 31 - 1      # clamped, no overflow
    assert L.moe_capacity_for(5, 4, 0, 6, 64) == 0


def test_nvfp4_entry_points_reject():
    E = moe.MOE_ERR_INVALID_ARG
    U = moe.MOE_ERR_UNSUPPORTED
    qw = L.moe_nvfp4_quantize_weights
    assert qw(A16, 2, 100, 256, A16, A16, A16, NULL) == U            # N not a multiple of 128
    assert qw(A16, 2, 128, 200, A16, A16, A16, NULL) == U            # K not a multiple of 256
    assert qw(NULL, 2, 128, 256, A16, A16, A16, NULL) == E
    assert qw(MIS, 2, 128, 256, A16, A16, A16, NULL) == E
    assert qw(A16, 0, 128, 256, A16, A16, A16, NULL) == moe.MOE_OK  # nothing to do
    dsp = L.moe_nvfp4_dispatch
    assert dsp(A16, A16, A16, A16, 8, 128, 16, 2, A16, A16, A16, A16, NULL) == U      # d % 256
    assert dsp(A16, A16, A16, A16, 8, 256, 300, 2, A16, A16, A16, A16, NULL) == E     # n_routed > 256
    assert dsp(A16, A16, A16, A16, 8, 256, 16, 9, A16, A16, A16, A16, NULL) == E      # top_k > 8
    assert dsp(A16, A16, A16, 0x10002, 8, 256, 16, 2, A16, A16, A16, A16, NULL) == E  # misaligned offsets
    gm = L.moe_nvfp4_grouped_gemm
    args = [A16, A16, A16, 4, 1024, A16, A16, A16, 256, 512, 1, NULL, NULL, A16, NULL, 0, NULL]

    def call(**kw):
        a = list(args)
        names = ["aq", "asf", "offp", "G", "rows", "wq", "wsf", "g", "N", "K", "epi", "oq", "osf", "out", "offo",
                 "orows", "s"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return gm(*a)

    assert call(N=200) == U
    assert call(K=300) == U
    assert call(rows=1000) == U                                      # rows_cap % 128
    assert call(G=300) == U
    assert call(epi=5) == E
    assert call(epi=0) == E                                          # FP4 out needs out_q / out_sf
    assert call(out=NULL) == E                                       # bf16 out needs out
    assert call(offo=0x10002) == E
    assert call(G=0) == moe.MOE_OK


def test_binding_arity_matches_the_header():
    """Every function the header declares has a ctypes signature with as many arguments."""
    arity = moe.header_arity()
    assert set(arity) == set(moe.header_functions())
    for name, n in arity.items():
        fn = getattr(L, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_expert_parallel_entry_points_reject():
    E, U = moe.MOE_ERR_INVALID_ARG, moe.MOE_ERR_UNSUPPORTED
    plan = L.moe_ep_plan
    assert plan(A16, 0, 3, 256, A16, A16, NULL) == E          # 3 ranks do not split 256 experts
    assert plan(A16, 0, 0, 256, A16, A16, NULL) == E          # no ranks
    assert plan(A16, 2, 2, 256, A16, A16, NULL) == E          # rank outside [0, world)
    assert plan(A16, 0, 128, 256, A16, A16, NULL) == E        # more ranks than MOE_EP_MAX_WORLD
    assert plan(NULL, 0, 2, 256, A16, A16, NULL) == E
    assert plan(A16, 0, 2, 256, 0x10002, A16, NULL) == E      # misaligned
    disp = L.moe_ep_dispatch
    assert disp(A16, A16, A16, A16, A16, 8, 64, 256, 9, 2, A16, 100, NULL) == E      # top_k > 8
    assert disp(A16, A16, A16, A16, A16, 8, 60, 256, 6, 2, A16, 100, NULL) == U      # d % 8 != 0
    assert disp(A16, A16, A16, A16, A16, 8, 64, 256, 6, 2, 0x10004, 100, NULL) == E  # pointer array misaligned
    assert disp(A16, A16, A16, A16, NULL, 8, 64, 256, 6, 2, A16, 100, NULL) == E
    assert disp(A16, A16, A16, A16, A16, 8, 64, 256, 6, 2, A16, -1, NULL) == E
    assert disp(A16, A16, A16, A16, A16, 0, 64, 256, 6, 2, A16, 100, NULL) == moe.MOE_OK  # T = 0: nothing to do
    comb = L.moe_ep_combine
    assert comb(A16, A16, A16, A16, A16, A16, NULL, 8, 64, 256, 6, 2, 2, 100, A16, NULL) == E   # shared rows missing
    assert comb(A16, A16, A16, A16, A16, A16, A16, 8, 64, 256, 6, 9, 2, 100, A16, NULL) == E    # n_shared > 8
    assert comb(A16, A16, A16, A16, A16, A16, A16, 8, 64, 255, 6, 2, 2, 100, A16, NULL) == E    # 2 ranks, 255 experts
    assert comb(A16, A16, A16, A16, A16, A16, A16, 8, 68, 256, 6, 2, 2, 100, A16, NULL) == U    # d % 8 != 0
    assert comb(A16, A16, A16, A16, A16, A16, A16, 0, 64, 256, 6, 2, 2, 100, A16, NULL) == moe.MOE_OK


def test_ipc_calls_reject_null():
    assert L.moe_ipc_handle_bytes() == 64
    off = ctypes.c_ulonglong(0)
    buf = ctypes.create_string_buffer(64)
    assert L.moe_ipc_get_handle(NULL, buf, ctypes.byref(off)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ipc_get_handle(A16, NULL, ctypes.byref(off)) == moe.MOE_ERR_INVALID_ARG
    ptr = ctypes.c_void_p()
    assert L.moe_ipc_open(NULL, 0, ctypes.byref(ptr)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ipc_open(buf, 0, NULL) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ipc_close(NULL) == moe.MOE_ERR_INVALID_ARG
