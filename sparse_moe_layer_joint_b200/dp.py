"""Data-parallel replicas of the layer (one process per GPU).

Every rank holds the same weights and routes its own T tokens; the balancing
bias must stay identical on all ranks, and the bias rule of "Inkling,
Dissected" §02e counts the loads of the whole batch (L_i = tokens that picked
expert i, Lbar = total selections / n_routed).  So before the update the
per-expert loads are summed over the ranks (one all-reduce of n_routed int32)
and the update uses the batch's total token count.  Ranks are assumed to hold
the same number of tokens.
"""
from __future__ import annotations


def _all_reduce_sum(t, group=None):
    """All-reduce (sum); gloo has no CUDA all-reduce path here, so CUDA tensors go through a host copy."""
    import torch.distributed as dist

    if t.is_cuda and dist.get_backend(group) == "gloo":
        h = t.cpu()
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
        t.copy_(h)
        return t
    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def world_size(group=None) -> int:
    import torch.distributed as dist

    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def global_counts(counts, group=None):
    """Sum the per-expert load counts over all ranks, in place (no-op on one rank)."""
    if world_size(group) > 1:
        _all_reduce_sum(counts, group)
    return counts


def total_tokens(T_local: int, group=None) -> int:
    """Tokens of the whole batch when every rank holds T_local of them."""
    return T_local * world_size(group)


def bias_step(layer, bias, gamma: float, group=None, stream=None):
    """The bias update of one data-parallel step: global loads, then the update on every rank."""
    global_counts(layer.counts, group)
    layer.bias_update(bias, gamma, stream=stream, T_total=total_tokens(layer.shape.T, group))
