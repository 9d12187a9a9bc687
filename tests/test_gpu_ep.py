"""Expert parallelism on the GPU ("Inkling, Dissected" §02d: the experts sit on
different GPUs and every token's rows travel to its experts' GPUs and back):
ExpertParallelLayer's step -- router, dispatch, row exchange, the owned experts
per source chunk, the way back, combine -- and its bias step over summed loads.

* one rank over NCCL: the step equals the one-GPU layer on the same batch;
* two ranks sharing one GPU over gloo (the exchange goes through host memory,
  so no kernel of one rank waits on the other): each rank's output matches the
  oracle on its own tokens and both ranks end with the bias the whole batch
  gives.
Both for the all-to-all step (ExpertParallelLayer) and for the step whose
exchange is fused into the dispatch and combine kernels through peer pointers
(PeerExpertParallelLayer: at two ranks the peer buffers are CUDA IPC mappings
between the two processes).  Each rank is a spawned process."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, backend, out_dir, peer=False):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import moe_inputs as mi
    import sparse_moe_layer_joint_b200 as moe
    from sparse_moe_layer_joint_b200 import ep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    kw = {"device_id": torch.device("cuda", 0)} if backend == "nccl" else {}
    dist.init_process_group(backend, rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60), **kw)
    try:
        w = mi.WORKLOADS["tiny"]
        t = mi.torch_workload(w)
        T_loc = w.T // world
        x_loc = t["x"][rank * T_loc:(rank + 1) * T_loc].contiguous()
        lo, hi = ep.expert_range(w.n_routed, world, rank)
        w1_loc = torch.cat([t["w1"][lo:hi], t["w1"][w.n_routed:]]).contiguous()
        w2_loc = torch.cat([t["w2"][lo:hi], t["w2"][w.n_routed:]]).contiguous()
        shape = moe.LayerShape(T_loc, w.d, w.f)
        if peer:
            layer = ep.PeerExpertParallelLayer(shape, rank, world, recv_rows=w.T * w.k)
        else:
            layer = ep.ExpertParallelLayer(shape, rank, world)
        b0 = t["bias"].clone()
        out = layer.forward(x_loc, t["w_r"], w1_loc, w2_loc, t["bias"]).clone()
        layer.bias_update(t["bias"], w.gamma)
        torch.cuda.synchronize()
        res = {"status": moe.moe_get_status(), "out": out.view(torch.int16).cpu().numpy(),
               "topk": layer.local.topk_idx.cpu().numpy(), "counts_global": layer.local.counts.cpu().numpy(),
               "bias": t["bias"].cpu().numpy(), "bias0": b0.cpu().numpy()}
        if peer:
            # a second step from the same bias gives the same bits: the buffers the ranks share
            # carry nothing from one step into the next
            b2 = b0.clone()
            out2 = layer.forward(x_loc, t["w_r"], w1_loc, w2_loc, b2).clone()
            torch.cuda.synchronize()
            res["repeat_equal"] = bool(torch.equal(out2.view(torch.int16), out.view(torch.int16)))
            res["status"] |= moe.moe_get_status()
            dist.barrier()
            layer.close()
        if world == 1:
            # the one-GPU layer on the same batch, from the same starting bias
            t["bias"].copy_(b0)
            single = moe.MoELayer(moe.LayerShape(w.T, w.d, w.f))
            o1 = single.forward(t["x"], t["w_r"], t["w1"], t["w2"], t["bias"])
            single.bias_update(t["bias"], w.gamma)
            torch.cuda.synchronize()
            res["out_single"] = o1.view(torch.int16).cpu().numpy()
            res["bias_single"] = t["bias"].cpu().numpy()
            res["topk_single"] = single.topk_idx.cpu().numpy()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **res)
    finally:
        dist.destroy_process_group()


def _run(world, backend, tmp_path, peer=False):
    mp.start_processes(_worker, args=(world, _free_port(), backend, str(tmp_path), peer), nprocs=world,
                       start_method="spawn")
    return [dict(np.load(os.path.join(tmp_path, f"rank{r}.npz"))) for r in range(world)]


def _bf16(bits):
    import moe_inputs as mi

    return mi.bf16_to_f64(np.asarray(bits).view(np.uint16))


@pytest.mark.parametrize("peer", [False, True], ids=["all_to_all", "peer"])
def test_one_rank_nccl_equals_the_one_gpu_layer(tmp_path, peer):
    from parity import check_output

    (r,) = _run(1, "nccl", tmp_path, peer)
    assert r["status"] == 0
    assert r.get("repeat_equal", True)
    np.testing.assert_array_equal(r["topk"], r["topk_single"])
    check_output(_bf16(r["out"]), _bf16(r["out_single"]), "EP world 1 vs one-GPU layer")
    np.testing.assert_array_equal(r["bias"].view(np.uint32), r["bias_single"].view(np.uint32))


@pytest.mark.parametrize("peer", [False, True], ids=["all_to_all", "peer"])
def test_two_ranks_gloo_match_the_oracle(tmp_path, peer):
    import moe_inputs as mi
    import oracle
    from parity import check_output

    world = 2
    res = _run(world, "gloo", tmp_path, peer)
    w = mi.WORKLOADS["tiny"]
    b0 = res[0]["bias0"]
    T_loc = w.T // world
    full = oracle.route_workload(w, b0)
    for rank, r in enumerate(res):
        assert r["status"] == 0
        assert r.get("repeat_equal", True)
        tokens = np.arange(rank * T_loc, (rank + 1) * T_loc)
        ref = oracle.forward_tokens(w, tokens, b0)
        same = (np.sort(r["topk"], 1) == np.sort(ref["topk_idx"], 1)).all(1)
        assert (same | (ref["margin"] < 1e-3)).all()
        check_output(_bf16(r["out"])[same], ref["out"][same], f"EP rank {rank}")
    # every rank holds the loads of the whole batch and the same bias afterwards
    np.testing.assert_array_equal(res[0]["counts_global"], res[1]["counts_global"])
    np.testing.assert_array_equal(res[0]["bias"].view(np.uint32), res[1]["bias"].view(np.uint32))
    counts = oracle.load_counts(full["topk_idx"], w.n_routed)
    if (res[0]["counts_global"] == counts).all():
        nb = oracle.bias_update(counts, b0, w.T, w.k, w.gamma)
        np.testing.assert_array_equal(res[0]["bias"].view(np.uint32), nb.view(np.uint32))


# ---------------------------------------------------------------------------
# the peer-memory kernels in one process: W ranks emulated as W buffer sets on
# the one GPU, their kernels launched one after another (none waits on another)
# ---------------------------------------------------------------------------
def _plan_reference(cnt, rank):
    """send_base and recv_offsets written out from their definition."""
    W, E = cnt.shape
    E_loc = E // W
    send_base = np.zeros(E, dtype=np.int64)
    for e in range(E):
        q = e // E_loc
        send_base[e] = sum(int(cnt[:, e2].sum()) for e2 in range(q * E_loc, e)) + int(cnt[:rank, e].sum())
    recv = np.zeros(E_loc + 1, dtype=np.int64)
    for el in range(E_loc):
        recv[el + 1] = recv[el] + int(cnt[:, rank * E_loc + el].sum())
    return send_base, recv


@pytest.mark.parametrize("W,E", [(1, 256), (2, 256), (4, 64), (8, 256), (3, 9)])
def test_ep_plan_matches_its_definition(W, E):
    import moe_inputs as mi
    import sparse_moe_layer_joint_b200 as moe

    cnt = (mi.words(W * E, W + E, mi.STREAM_TEST_TOPK) % 50).reshape(W, E).astype(np.int32)
    cnt[0, 0] = 0
    c = torch.from_numpy(cnt).cuda()
    for rank in range(W):
        sb = torch.full((E,), -7, dtype=torch.int32, device="cuda")
        ro = torch.full((E // W + 1,), -7, dtype=torch.int32, device="cuda")
        moe.moe_ep_plan(c, rank, W, E, sb, ro)
        ref_sb, ref_ro = _plan_reference(cnt, rank)
        np.testing.assert_array_equal(sb.cpu().numpy(), ref_sb)
        np.testing.assert_array_equal(ro.cpu().numpy(), ref_ro)


@pytest.mark.parametrize("W,E,k,ns,d", [(4, 64, 6, 2, 256), (2, 256, 8, 1, 136), (1, 16, 3, 0, 64)])
def test_ep_dispatch_combine_emulated_ranks(W, E, k, ns, d):
    """With the identity as every expert (the owner copies recv_x to recv_y), each emulated rank's
    moe_ep_combine equals moe_combine on its own rows in dispatch order, bit for bit: every row
    went to its owner's buffer and came back to the right (token, slot).  The owners' buffers
    are filled exactly (no row lost or written twice)."""
    import moe_inputs as mi
    import oracle
    import sparse_moe_layer_joint_b200 as moe

    Ts = [37 + 50 * r for r in range(W)]
    ranks = []
    for r, T in enumerate(Ts):
        x = mi.normal_bf16(T * d, 30 + r, mi.STREAM_X).reshape(T, d)
        u = mi.words(T * E, 40 + r, mi.STREAM_TEST_TOPK).reshape(T, E)
        topk = np.argsort(u, axis=1, kind="stable")[:, :k].astype(np.int32)
        g = (mi.words(T * (k + ns), 50 + r, mi.STREAM_TEST_GATES) % 1000).reshape(T, k + ns).astype(np.float32) / 997
        ysh = mi.normal_bf16(max(ns, 1) * T * d, 60 + r, mi.STREAM_TEST_SHARED).reshape(max(ns, 1), T, d)
        dp = oracle.dispatch(topk, E)
        ranks.append({"T": T, "x": torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda(),
                      "topk": torch.from_numpy(topk).cuda(), "gates": torch.from_numpy(g).cuda(),
                      "ysh": torch.from_numpy(ysh.view(np.int16)).view(torch.bfloat16).cuda(),
                      "offsets": torch.from_numpy(dp["offsets"]).cuda(),
                      "token_row": torch.from_numpy(dp["token_row"]).cuda(),
                      "row_token": dp["row_token"],
                      "counts": np.diff(dp["offsets"]).astype(np.int32)})
    cnt = torch.from_numpy(np.stack([rk["counts"] for rk in ranks])).cuda()
    recv_rows = sum(Ts) * k
    recv_x = [torch.full((recv_rows, d), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    recv_y = [torch.empty((recv_rows, d), dtype=torch.bfloat16, device="cuda") for _ in range(W)]
    px = torch.tensor([b.data_ptr() for b in recv_x], dtype=torch.int64, device="cuda")
    py = torch.tensor([b.data_ptr() for b in recv_y], dtype=torch.int64, device="cuda")
    for r, rk in enumerate(ranks):
        rk["send_base"] = torch.empty(E, dtype=torch.int32, device="cuda")
        rk["recv_off"] = torch.empty(E // W + 1, dtype=torch.int32, device="cuda")
        moe.moe_ep_plan(cnt, r, W, E, rk["send_base"], rk["recv_off"])
        moe.moe_ep_dispatch(rk["x"], rk["topk"], rk["token_row"], rk["offsets"], rk["send_base"], rk["T"], d, E, k, W,
                            px, recv_rows)
    torch.cuda.synchronize()
    for q in range(W):   # the identity expert on each owner; every received row is filled
        n = int(ranks[q]["recv_off"][-1].item())
        assert not torch.isnan(recv_x[q][:n].float()).any()
        recv_y[q][:n].copy_(recv_x[q][:n])
    for r, rk in enumerate(ranks):
        T = rk["T"]
        out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        moe.moe_ep_combine(py, rk["topk"], rk["token_row"], rk["offsets"], rk["send_base"], rk["gates"],
                           rk["ysh"] if ns else None, T, d, E, k, ns, W, recv_rows, out)
        xp = rk["x"][torch.from_numpy(rk["row_token"].astype(np.int64)).cuda()]
        ref = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        moe.moe_combine(xp, rk["token_row"], rk["gates"], rk["ysh"] if ns else None, T, d, k, ns, ref)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"rank {r}"
    assert moe.moe_get_status() == 0
