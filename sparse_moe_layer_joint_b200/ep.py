"""Expert parallelism across ranks (one process per GPU).

"Inkling, Dissected" §02d: each expert can serve only so many tokens per batch,
"set by memory and the all-to-all communication schedule" -- the experts live on
different GPUs and every token's rows travel to the GPUs of its experts and back.
Here rank r holds the routed experts [r*E/W, (r+1)*E/W) (E = n_routed, W ranks,
W dividing E) and a replica of the shared experts.  One step on rank r:

1. route its own tokens (router kernel) and group the (token, slot) pairs by
   expert (moe_permute): the experts of each destination rank are then one
   contiguous block of rows;
2. exchange the per-expert row counts, then the rows (two all-to-alls); the
   shared experts run on a second stream meanwhile;
3. run the owned experts on the rows received from every source rank
   (moe_grouped_ffn once per source chunk, whose rows are grouped by expert);
4. send the results back (all-to-all): they land in the sender's dispatch order,
   so the combine is the one-GPU combine (moe_combine through token_row);
5. ``bias_update``: the loads summed over ranks (one all-reduce, as in ``dp``),
   then the update with the whole batch's token count on every rank.

No capacity is applied in this mode: every (token, slot) pair is served.

The plan and exchange functions below are device-agnostic (torch tensors, any
backend that implements all_to_all_single; with gloo, CUDA tensors are staged
through host memory).  ``ExpertParallelLayer`` runs the GPU step with the
library's kernels and NCCL (or gloo).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def expert_range(n_routed: int, world: int, rank: int) -> Tuple[int, int]:
    """Routed experts [lo, hi) held by ``rank``."""
    if n_routed % world != 0:
        raise ValueError(f"{n_routed} routed experts do not split over {world} ranks")
    per = n_routed // world
    return rank * per, (rank + 1) * per


def send_counts(offsets: Sequence[int], n_routed: int, world: int) -> List[int]:
    """Rows this rank sends to each rank: the dispatch offsets at the experts blocks' bounds."""
    off = np.asarray(offsets, dtype=np.int64)
    per = n_routed // world
    return [int(off[(q + 1) * per] - off[q * per]) for q in range(world)]


def _all_to_all(out, inp, out_splits=None, in_splits=None, group=None):
    """all_to_all_single; gloo has no CUDA all-to-all, so there CUDA tensors go through host copies."""
    import torch.distributed as dist

    if inp.is_cuda and dist.get_backend(group) == "gloo":
        host_out = out.new_empty(out.shape, device="cpu")
        dist.all_to_all_single(host_out, inp.cpu(), output_split_sizes=out_splits, input_split_sizes=in_splits,
                               group=group)
        out.copy_(host_out)
        return out
    dist.all_to_all_single(out, inp, output_split_sizes=out_splits, input_split_sizes=in_splits, group=group)
    return out


def exchange_counts(counts_by_expert, world: int, group=None):
    """All-to-all of per-expert row counts: ``counts_by_expert`` [n_routed] int32 (this rank's
    dispatch); returns [world, n_routed/world]: row s = the rows source s sends for each of
    this rank's experts."""
    import torch

    per = counts_by_expert.numel() // world
    out = torch.empty((world * per,), dtype=counts_by_expert.dtype, device=counts_by_expert.device)
    _all_to_all(out, counts_by_expert.contiguous(), group=group)
    return out.view(world, per)


def exchange_rows(rows, send: Sequence[int], recv: Sequence[int], group=None, out=None):
    """All-to-all of row blocks: ``rows`` [sum(send), ...] ordered by destination rank; returns
    [sum(recv), ...] ordered by source rank (in ``out`` when given)."""
    import torch

    n = int(sum(recv))
    if out is None:
        out = torch.empty((n,) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    else:
        out = out[:n]
    return _all_to_all(out, rows.contiguous(), [int(v) for v in recv], [int(v) for v in send], group)


def chunk_offsets(recv_by_expert: np.ndarray) -> List[np.ndarray]:
    """Per source rank, the group offsets of its received chunk (rows grouped by this rank's
    experts, in expert order), relative to the chunk's first row."""
    return [np.concatenate([[0], np.cumsum(row)]).astype(np.int32) for row in np.asarray(recv_by_expert)]


class ExpertParallelLayer:
    """One layer step with the routed experts split over ranks (bf16, GELU or SwiGLU experts).

    Its compute is the library's kernels (router, permute, grouped FFN, combine, bias update);
    its exchange is an all-to-all of the dispatched rows and of the expert outputs (NCCL, or
    gloo through host copies).  Weights: ``w_router`` and the shared experts' matrices as on one
    GPU; ``w1_local`` / ``w2_local`` hold only this rank's routed experts, followed by the
    shared experts.  The tests run it at one rank (NCCL) and at two ranks sharing one GPU (gloo:
    the ranks' kernels never wait on each other, the exchange is on the host); across several
    GPUs it is not measured here.
    """

    def __init__(self, shape, rank: int, world: int, device="cuda", group=None, activation: str = "gelu_tanh",
                 route_scale: float = 1.0):
        import torch

        from sparse_moe_layer_joint_b200 import MoELayer

        self.rank, self.world, self.group = rank, world, group
        self.lo, self.hi = expert_range(shape.n_routed, world, rank)
        self.local = MoELayer(shape, device=device, activation=activation, route_scale=route_scale)
        self.dev = torch.device(device)
        self.offsets_host = torch.empty((shape.n_routed + 1,), dtype=torch.int32).pin_memory()
        self.ev_offsets = torch.cuda.Event()
        self.ev_routed = torch.cuda.Event()
        self.ev_shared = torch.cuda.Event()

    def forward(self, x, w_router, w1_local, w2_local, bias, logit_offset=None):
        import torch

        import sparse_moe_layer_joint_b200 as moe

        L, s = self.local, self.local.shape
        T, d, f, k = s.T, s.d, s.d_ff, s.top_k
        E_loc = self.hi - self.lo
        main = torch.cuda.current_stream(self.dev)
        moe.moe_router_topk(x, w_router, bias, logit_offset, T, d, s.n_routed, s.n_shared, k, L.route_scale,
                            L.topk_idx, L.gates, L.counts, None, stream=main)
        # shared experts on this rank's tokens, on the side stream while the exchange runs
        if s.n_shared > 0:
            self.ev_routed.record(main)
            L.side.wait_event(self.ev_routed)
            moe.moe_grouped_ffn(x, None, s.n_shared, T, E_loc, w1_local, w2_local, d, f, L.activation,
                                L.h_shared, L.y_shared, stream=L.side)
            self.ev_shared.record(L.side)
        moe.moe_permute(x, L.topk_idx, L.counts, T, d, s.n_routed, k, L.offsets, L.x_perm, L.row_token,
                        L.token_row, L.scratch, L.scratch_bytes, stream=main)
        # the split sizes of the exchange are host values: copy the 257 offsets (1 KB) and wait for
        # that copy alone (the event is on the main stream; the side stream keeps running)
        self.offsets_host.copy_(L.offsets, non_blocking=True)
        self.ev_offsets.record(main)
        self.ev_offsets.synchronize()
        offsets = self.offsets_host.numpy().astype(np.int64)
        send = send_counts(offsets, s.n_routed, self.world)
        # rows per expert = the router's counts (no capacity in this mode)
        recv_by_expert = exchange_counts(L.counts, self.world, self.group).cpu().numpy()
        recv = recv_by_expert.sum(axis=1)
        x_recv = exchange_rows(L.x_perm[:int(offsets[-1])], send, recv, self.group)
        y_recv = torch.empty_like(x_recv)
        h = torch.empty((max(x_recv.shape[0], 1), f), dtype=x_recv.dtype, device=self.dev)
        start = 0
        for src, off in enumerate(chunk_offsets(recv_by_expert)):
            n = int(off[-1])
            if n:
                off_dev = torch.from_numpy(off).to(self.dev)
                moe.moe_grouped_ffn(x_recv[start:start + n], off_dev, E_loc, n, 0, w1_local, w2_local, d, f,
                                    L.activation, h[:n], y_recv[start:start + n], stream=main)
            start += n
        exchange_rows(y_recv, recv, send, self.group, out=L.y_perm)   # back in this rank's dispatch order
        if s.n_shared > 0:
            main.wait_event(self.ev_shared)
        moe.moe_combine(L.y_perm, L.token_row, L.gates, L.y_shared if s.n_shared > 0 else None, T, d, k,
                        s.n_shared, L.out, stream=main)
        return L.out

    def bias_update(self, bias, gamma: float):
        """§02e after the step: this rank's loads summed over all ranks (in place, one all-reduce of
        n_routed int32), then b += gamma * sign(Lbar - L) with the whole batch's token count."""
        from sparse_moe_layer_joint_b200 import dp

        dp.bias_step(self.local, bias, gamma, group=self.group)


class PeerExpertParallelLayer:
    """The expert-parallel step with the exchange fused into the library's kernels: rows go
    straight from the source rank's x into the owner's receive buffer (moe_ep_dispatch, stores
    through peer pointers), the owner runs one grouped GEMM over all rows it received, and each
    source gathers its tokens' outputs back from the owners' buffers (moe_ep_combine, peer loads).
    The only collectives are an all-gather of the per-expert counts (W x n_routed int32), two
    barriers between the phases, and the bias step's all-reduce of the counts.

    Every rank allocates ``recv_rows`` rows for its receive and output buffers (sized by the
    caller: the rows its experts can receive in a step; more raise MOE_STATUS_RECV_OVERFLOW).
    The buffers of the other ranks are mapped with CUDA IPC handles exchanged over the process
    group; at one rank nothing is mapped.  With NCCL the barriers are stream-ordered collectives
    (no host wait); with gloo the host synchronises the device and meets the other ranks, which
    also lets several ranks share one GPU (no kernel of one rank ever waits on another's).
    Weights: ``w1_local`` / ``w2_local`` hold this rank's routed experts followed by the shared
    experts, as for ``ExpertParallelLayer``.
    """

    def __init__(self, shape, rank: int, world: int, recv_rows: int, device="cuda", group=None,
                 activation: str = "gelu_tanh", route_scale: float = 1.0):
        import torch
        import torch.distributed as dist

        from sparse_moe_layer_joint_b200 import MoELayer

        import sparse_moe_layer_joint_b200 as moe

        self.rank, self.world, self.group = rank, world, group
        self.lo, self.hi = expert_range(shape.n_routed, world, rank)
        self.local = MoELayer(shape, device=device, activation=activation, route_scale=route_scale)
        self.dev = torch.device(device)
        s = shape
        self.recv_rows = int(recv_rows)
        bf = torch.bfloat16
        self.recv_x = torch.empty((max(self.recv_rows, 1), s.d), dtype=bf, device=self.dev)
        self.recv_y = torch.empty((max(self.recv_rows, 1), s.d), dtype=bf, device=self.dev)
        self.recv_h = torch.empty((max(self.recv_rows, 1), s.d_ff), dtype=bf, device=self.dev)
        self.counts_all = torch.empty((world, s.n_routed), dtype=torch.int32, device=self.dev)
        self.send_base = torch.empty((s.n_routed,), dtype=torch.int32, device=self.dev)
        self.recv_offsets = torch.empty((self.hi - self.lo + 1,), dtype=torch.int32, device=self.dev)
        self.nccl = world > 1 and dist.get_backend(group) == "nccl"
        self.opened = []
        ptr_x, ptr_y = [0] * world, [0] * world
        ptr_x[rank], ptr_y[rank] = self.recv_x.data_ptr(), self.recv_y.data_ptr()
        if world > 1:
            mine = (moe.moe_ipc_get_handle(self.recv_x), moe.moe_ipc_get_handle(self.recv_y))
            every = [None] * world
            dist.all_gather_object(every, mine, group=group)
            for q in range(world):
                if q != rank:
                    ptr_x[q] = moe.moe_ipc_open(*every[q][0])
                    ptr_y[q] = moe.moe_ipc_open(*every[q][1])
                    self.opened += [ptr_x[q], ptr_y[q]]
        self.ptr_x = torch.tensor(ptr_x, dtype=torch.int64, device=self.dev)
        self.ptr_y = torch.tensor(ptr_y, dtype=torch.int64, device=self.dev)
        self.ev_routed = torch.cuda.Event()
        self.ev_shared = torch.cuda.Event()
        self.token = torch.zeros(1, dtype=torch.int32, device=self.dev)

    def _gather_counts(self):
        import torch.distributed as dist

        L = self.local
        if self.world == 1:
            self.counts_all[0].copy_(L.counts)
        elif self.nccl:
            dist.all_gather_into_tensor(self.counts_all.view(-1), L.counts, group=self.group)
        else:  # gloo: host tensors
            import torch

            parts = [torch.empty((L.counts.numel(),), dtype=torch.int32) for _ in range(self.world)]
            dist.all_gather(parts, L.counts.cpu(), group=self.group)
            self.counts_all.copy_(torch.stack(parts))

    def _barrier(self):
        """Every rank's work so far is complete before any rank goes on."""
        import torch
        import torch.distributed as dist

        if self.world == 1:
            return
        if self.nccl:
            dist.all_reduce(self.token, group=self.group)   # stream-ordered: no host wait
        else:
            torch.cuda.synchronize(self.dev)
            dist.barrier(group=self.group)

    def forward(self, x, w_router, w1_local, w2_local, bias, logit_offset=None):
        import torch

        import sparse_moe_layer_joint_b200 as moe

        L, s = self.local, self.local.shape
        T, d, f, k = s.T, s.d, s.d_ff, s.top_k
        E_loc = self.hi - self.lo
        main = torch.cuda.current_stream(self.dev)
        moe.moe_router_topk(x, w_router, bias, logit_offset, T, d, s.n_routed, s.n_shared, k, L.route_scale,
                            L.topk_idx, L.gates, L.counts, None, stream=main)
        if s.n_shared > 0:
            self.ev_routed.record(main)
            L.side.wait_event(self.ev_routed)
            moe.moe_grouped_ffn(x, None, s.n_shared, T, E_loc, w1_local, w2_local, d, f, L.activation,
                                L.h_shared, L.y_shared, stream=L.side)
            self.ev_shared.record(L.side)
        moe.moe_permute(x, L.topk_idx, L.counts, T, d, s.n_routed, k, L.offsets, None, L.row_token, L.token_row,
                        L.scratch, L.scratch_bytes, stream=main)
        self._gather_counts()
        moe.moe_ep_plan(self.counts_all, self.rank, self.world, s.n_routed, self.send_base, self.recv_offsets,
                        stream=main)
        moe.moe_ep_dispatch(x, L.topk_idx, L.token_row, L.offsets, self.send_base, T, d, s.n_routed, k, self.world,
                            self.ptr_x, self.recv_rows, stream=main)
        self._barrier()        # every rank's rows are in its owners' buffers
        if E_loc > 0 and self.recv_rows > 0:
            moe.moe_grouped_ffn(self.recv_x, self.recv_offsets, E_loc, self.recv_rows, 0, w1_local, w2_local, d, f,
                                L.activation, self.recv_h, self.recv_y, stream=main)
        self._barrier()        # every owner's outputs are written
        if s.n_shared > 0:
            main.wait_event(self.ev_shared)
        moe.moe_ep_combine(self.ptr_y, L.topk_idx, L.token_row, L.offsets, self.send_base, L.gates,
                           L.y_shared if s.n_shared > 0 else None, T, d, s.n_routed, k, s.n_shared, self.world,
                           self.recv_rows, L.out, stream=main)
        return L.out

    def bias_update(self, bias, gamma: float):
        """§02e after the step: the loads summed over all ranks, then the update with the whole
        batch's token count (as ``ExpertParallelLayer.bias_update``)."""
        from sparse_moe_layer_joint_b200 import dp

        dp.bias_step(self.local, bias, gamma, group=self.group)

    def close(self):
        """Unmap the peers' buffers (call on every rank before the process group goes away)."""
        import sparse_moe_layer_joint_b200 as moe

        for p in self.opened:
            moe.moe_ipc_close(p)
        self.opened = []
