"""Expert parallelism on the GPU ("Inkling, Dissected" §02d: the experts sit on
different GPUs and every token's rows travel to its experts' GPUs and back):
ExpertParallelLayer's step -- router, dispatch, row exchange, the owned experts
per source chunk, the way back, combine -- and its bias step over summed loads.

* one rank over NCCL: the step equals the one-GPU layer on the same batch;
* two ranks sharing one GPU over gloo (the exchange goes through host memory,
  so no kernel of one rank waits on the other): each rank's output matches the
  oracle on its own tokens and both ranks end with the bias the whole batch
  gives.
Each rank is a spawned process."""
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


def _worker(rank, world, port, backend, out_dir):
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
        layer = ep.ExpertParallelLayer(moe.LayerShape(T_loc, w.d, w.f), rank, world)
        b0 = t["bias"].clone()
        out = layer.forward(x_loc, t["w_r"], w1_loc, w2_loc, t["bias"])
        layer.bias_update(t["bias"], w.gamma)
        torch.cuda.synchronize()
        res = {"status": moe.moe_get_status(), "out": out.view(torch.int16).cpu().numpy(),
               "topk": layer.local.topk_idx.cpu().numpy(), "counts_global": layer.local.counts.cpu().numpy(),
               "bias": t["bias"].cpu().numpy(), "bias0": b0.cpu().numpy()}
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


def _run(world, backend, tmp_path):
    mp.start_processes(_worker, args=(world, _free_port(), backend, str(tmp_path)), nprocs=world,
                       start_method="spawn")
    return [dict(np.load(os.path.join(tmp_path, f"rank{r}.npz"))) for r in range(world)]


def _bf16(bits):
    import moe_inputs as mi

    return mi.bf16_to_f64(np.asarray(bits).view(np.uint16))


def test_one_rank_nccl_equals_the_one_gpu_layer(tmp_path):
    from parity import check_output

    (r,) = _run(1, "nccl", tmp_path)
    assert r["status"] == 0
    np.testing.assert_array_equal(r["topk"], r["topk_single"])
    check_output(_bf16(r["out"]), _bf16(r["out_single"]), "EP world 1 vs one-GPU layer")
    np.testing.assert_array_equal(r["bias"].view(np.uint32), r["bias_single"].view(np.uint32))


def test_two_ranks_gloo_match_the_oracle(tmp_path):
    import moe_inputs as mi
    import oracle
    from parity import check_output

    world = 2
    res = _run(world, "gloo", tmp_path)
    w = mi.WORKLOADS["tiny"]
    b0 = res[0]["bias0"]
    T_loc = w.T // world
    full = oracle.route_workload(w, b0)
    for rank, r in enumerate(res):
        assert r["status"] == 0
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
