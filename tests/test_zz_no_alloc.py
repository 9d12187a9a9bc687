"""moe_permute_noalloc: the permute entry point for callers that cannot
allocate device memory (a plugin whose host application owns every device
allocation, a process that reserved all of HBM up front, a loop that must not
call cudaMalloc/cudaFree).  Its scratch is a fixed device array inside the
library; this checks, through the C ABI, that it gives the oracle's dispatch
and the same outputs as moe_permute with a caller scratch buffer, on calls in a
row, and that it refuses sizes beyond its limit.  Kept in its own file,
collected last."""
import ctypes

import numpy as np
import pytest

import moe_inputs as mi
import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if torch.cuda.is_available():
    import sparse_moe_layer_joint_b200 as moe


def _inputs(T, k, n_routed, d, seed):
    w = mi.words(T * n_routed, seed, mi.STREAM_TEST_TOPK).reshape(T, n_routed)
    topk = np.argsort(w, axis=1, kind="stable")[:, :k].astype(np.int32)
    x = mi.normal_bf16(T * d, seed, mi.STREAM_X).reshape(T, d)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return xd, torch.from_numpy(topk).cuda()


def _outputs(T, k, n_routed, d):
    return (torch.full((n_routed + 1,), -9, dtype=torch.int32, device="cuda"),
            torch.full((T * k, d), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((T * k,), -9, dtype=torch.int32, device="cuda"),
            torch.full((T, k), -9, dtype=torch.int32, device="cuda"))


def _noalloc(x, topk, T, d, n_routed, k, outs):
    off, xp, rt, tr = outs
    s = torch.cuda.current_stream().cuda_stream
    return moe.lib().moe_permute_noalloc(x.data_ptr(), topk.data_ptr(), None, T, d, n_routed, k, off.data_ptr(),
                                         xp.data_ptr(), rt.data_ptr(), tr.data_ptr(), s)


def _with_scratch(x, topk, T, d, n_routed, k, outs):
    off, xp, rt, tr = outs
    nb = moe.moe_permute_scratch_bytes(T, n_routed)
    scratch = torch.empty(nb, dtype=torch.uint8, device="cuda")
    moe.moe_permute(x, topk, None, T, d, n_routed, k, off, xp, rt, tr, scratch, nb)


def test_noalloc_permute_matches_permute_on_two_calls_in_a_row():
    # different problems back to back: a later one must not see an earlier one's scratch (the third fits one
    # 256-token chunk and takes the single-CTA index kernel)
    for (T, k, n_routed, d, seed) in [(4096, 6, 256, 512, 1), (1000, 8, 64, 136, 2), (200, 6, 256, 64, 3)]:
        x, topk = _inputs(T, k, n_routed, d, seed)
        ref = _outputs(T, k, n_routed, d)
        got = _outputs(T, k, n_routed, d)
        _with_scratch(x, topk, T, d, n_routed, k, ref)
        assert _noalloc(x, topk, T, d, n_routed, k, got) == moe.MOE_OK
        torch.cuda.synchronize()
        assert moe.moe_get_status() == 0
        for a, b in zip(ref, got):   # integer and byte outputs: bit-exact
            if a.dtype == torch.bfloat16:
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b)
        # and directly against the oracle's dispatch
        want = oracle.dispatch(topk.cpu().numpy(), n_routed)
        off, xp, rt, tr = got
        np.testing.assert_array_equal(off.cpu().numpy(), want["offsets"])
        np.testing.assert_array_equal(rt.cpu().numpy(), want["row_token"])
        np.testing.assert_array_equal(tr.cpu().numpy(), want["token_row"])
        x_bits = x.view(torch.int16).cpu().numpy()
        np.testing.assert_array_equal(xp.view(torch.int16).cpu().numpy(), x_bits[want["row_token"]])


def test_noalloc_permute_rejects_sizes_beyond_its_limit():
    T, k, n_routed, d = 130816 + 256, 6, 256, 8   # one chunk past the 1 MiB limit
    assert moe.moe_permute_scratch_bytes(T, n_routed) > (1 << 20)
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    rc = moe.lib().moe_permute_noalloc(p, p, None, T, d, n_routed, k, p, p, p, p,
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == moe.MOE_ERR_SCRATCH
    # the largest size it takes
    assert moe.moe_permute_scratch_bytes(130816, n_routed) <= (1 << 20)
