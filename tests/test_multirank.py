"""The data-parallel exchange on CPU (gloo, world size 2): each rank routes its
half of the batch with the oracle, the per-expert loads are summed with
sparse_moe_layer_joint_b200.dp, and the bias update on every rank equals the
single-process update on the whole batch (the rule of §02e counts the batch's
loads)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist

    import moe_inputs as mi
    import oracle
    from sparse_moe_layer_joint_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = mi.WORKLOADS["tiny"]
        T_local = w.T // world
        tokens = np.arange(rank * T_local, (rank + 1) * T_local)
        b = mi.host_bias(w)
        r = oracle.route_workload(w, b, tokens=tokens)
        counts = torch.from_numpy(oracle.load_counts(r["topk_idx"], w.n_routed).astype(np.int32))
        dp.global_counts(counts)
        T_total = dp.total_tokens(T_local)
        nb = oracle.bias_update(counts.numpy(), b, T_total, w.k, w.gamma)
        np.save(os.path.join(out_dir, f"bias_{rank}.npy"), nb)
        np.save(os.path.join(out_dir, f"counts_{rank}.npy"), counts.numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_with_the_whole_batch(tmp_path):
    import moe_inputs as mi
    import oracle

    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    w = mi.WORKLOADS["tiny"]
    b = mi.host_bias(w)
    full = oracle.route_workload(w, b)
    counts = oracle.load_counts(full["topk_idx"], w.n_routed)
    expect = oracle.bias_update(counts, b, w.T, w.k, w.gamma)
    for rank in range(world):
        np.testing.assert_array_equal(np.load(tmp_path / f"counts_{rank}.npy"), counts)
        np.testing.assert_array_equal(np.load(tmp_path / f"bias_{rank}.npy").view(np.uint32), expect.view(np.uint32))


def test_single_process_is_a_no_op():
    from sparse_moe_layer_joint_b200 import dp

    c = torch.arange(4, dtype=torch.int32)
    assert dp.world_size() == 1
    assert dp.global_counts(c) is c and c.tolist() == [0, 1, 2, 3]
    assert dp.total_tokens(100) == 100


def _lab_worker(rank, world, port, out_dir, steps, gamma):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist

    import moe_inputs as mi
    import oracle
    from sparse_moe_layer_joint_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = mi.LAB
        half = w.T // world
        wr = mi.lab_wr(w)
        b = np.zeros(w.n_routed, np.float32)
        for s in range(steps):
            x = mi.lab_x(w, s)[rank * half:(rank + 1) * half]      # this rank's share of the step's batch
            r = oracle.route(oracle.logits(x, wr), b, w.k, w.n_routed, 0)
            counts = torch.from_numpy(oracle.load_counts(r["topk_idx"], w.n_routed).astype(np.int32))
            dp.global_counts(counts)
            b = oracle.bias_update(counts.numpy(), b, dp.total_tokens(half), w.k, gamma)
        np.save(os.path.join(out_dir, f"lab_bias_{rank}.npy"), b)
    finally:
        dist.destroy_process_group()


def test_two_ranks_run_the_lab_like_one(tmp_path):
    """The Router Balance Lab split over two data-parallel ranks (each routes half of every
    step's batch; the loads are summed before each update) ends with the bias of the
    single-process run on whole batches, bit for bit."""
    import moe_inputs as mi
    import oracle

    steps, gamma = 12, 0.01
    mp.start_processes(_lab_worker, args=(2, _free_port(), str(tmp_path), steps, gamma), nprocs=2,
                       start_method="spawn")
    ref = oracle.lab_run(mi.LAB, gamma, steps=steps)["bias"][-1]
    for rank in range(2):
        np.testing.assert_array_equal(np.load(tmp_path / f"lab_bias_{rank}.npy").view(np.uint32), ref.view(np.uint32))


def _ep_worker(rank, world, port, out_dir):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist

    import moe_inputs as mi
    import oracle
    from sparse_moe_layer_joint_b200 import ep

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = mi.WORKLOADS["tiny"]
        T_local = w.T // world
        tokens = np.arange(rank * T_local, (rank + 1) * T_local)
        b = mi.host_bias(w)
        x = mi.host_x(w, tokens)
        r = oracle.route_workload(w, b, tokens, x=x)
        dp = oracle.dispatch(r["topk_idx"], w.n_routed)
        x_perm = torch.from_numpy(mi.bf16_to_f64(x)[dp["row_token"]])
        send = ep.send_counts(dp["offsets"], w.n_routed, world)
        by_expert = torch.from_numpy(np.diff(dp["offsets"]).astype(np.int32))
        recv_by_expert = ep.exchange_counts(by_expert, world).numpy()
        recv = recv_by_expert.sum(axis=1)
        x_recv = ep.exchange_rows(x_perm, send, recv)
        lo, hi = ep.expert_range(w.n_routed, world, rank)
        # this rank's experts on the rows from every source (the oracle stands in for the GPU kernels)
        y_recv = np.zeros_like(x_recv.numpy())
        start = 0
        for off in ep.chunk_offsets(recv_by_expert):
            for j in range(hi - lo):
                a0, a1 = start + off[j], start + off[j + 1]
                if a1 > a0:
                    rows = mi.f32_to_bf16_bits(x_recv.numpy()[a0:a1].astype(np.float32))
                    y_recv[a0:a1] = oracle.expert(rows, mi.host_w1(w, lo + j), mi.host_w2(w, lo + j))
            start += int(off[-1])
        y_perm = ep.exchange_rows(torch.from_numpy(y_recv), recv, send).numpy()
        y_sh = np.stack([oracle.expert(x, mi.host_w1(w, e), mi.host_w2(w, e))
                         for e in range(w.n_routed, w.n_experts)])
        out = oracle.combine(y_perm, dp["token_row"], r["gates"], y_sh)
        np.save(os.path.join(out_dir, f"ep_out_{rank}.npy"), out)
        np.save(os.path.join(out_dir, f"ep_recv_{rank}.npy"), recv_by_expert)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_matches_one_process(tmp_path, world):
    """Experts split over ranks (rank r holds 256/W routed experts): the rows each token sends
    to its experts' ranks come back in dispatch order, and the combined output equals the
    single-process layer on the same tokens (every expert row computed the same way in fp64;
    only the order of the gate-weighted sum differs, so to fp64 rounding)."""
    import moe_inputs as mi
    import oracle

    mp.start_processes(_ep_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    w = mi.WORKLOADS["tiny"]
    b = mi.host_bias(w)
    full = oracle.forward_tokens(w, np.arange(w.T), b)
    T_local = w.T // world
    counts = np.zeros(w.n_routed, np.int64)
    for rank in range(world):
        got = np.load(tmp_path / f"ep_out_{rank}.npy")
        np.testing.assert_allclose(got, full["out"][rank * T_local:(rank + 1) * T_local], rtol=1e-12, atol=1e-14)
        counts[rank * (w.n_routed // world):(rank + 1) * (w.n_routed // world)] = \
            np.load(tmp_path / f"ep_recv_{rank}.npy").sum(axis=0)
    # every (token, slot) pair reached the rank of its expert exactly once
    np.testing.assert_array_equal(counts, oracle.load_counts(full["topk_idx"], w.n_routed))
