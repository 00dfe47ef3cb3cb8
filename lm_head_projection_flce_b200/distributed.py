"""Data-parallel use of the fused loss: the pages' ``materialize_lm_weight``.

"nemo_automodel.components.loss.linear_ce" (FusedLinearCrossEntropy
.materialize_lm_weight) and "nemo_automodel.components.loss.linear_ce_base"
(LinearCrossEntropy.materialize_lm_weight): the fused loss consumes the head
outside the module that owns its FSDP shards, so every data/context-parallel
rank computes a rank-local gradient of the *full* head.  Materialising the
head must therefore (1) gather the shards into a regular ``[vocab, hidden]``
tensor on every rank and (2) in backward *sum* the ranks' full gradients and
hand each rank its own shard - not merely slice the local gradient, which is
what marking the gathered tensor "replicated" would do.  A regular tensor is
returned unchanged; a trainable sharded head without a matching reduction
group is refused (``ValueError``) instead of silently producing rank-local
shards.

Here (1) is one all-gather and (2) one reduce-scatter over the given process
group (NCCL on GPUs: over NVLink / NVSwitch; any backend without a
reduce-scatter, such as gloo, uses all-reduce + slice).  The head may be a
``torch.distributed.tensor.DTensor`` sharded on dim 0 over a 1-D mesh (the
FSDP layout), including uneven shards.  The loss itself is the single-GPU
fused path: each rank passes its own tokens and the *global*
``num_label_tokens``, so the ranks' losses add up to the global loss.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["materialize_lm_weight", "data_parallel_fused_linear_cross_entropy"]


def _is_dtensor(t) -> bool:
    try:
        from torch.distributed.tensor import DTensor
    except ImportError:  # pragma: no cover - torch without DTensor
        return False
    return isinstance(t, DTensor)


def _has_reduce_scatter(group) -> bool:
    return dist.get_backend(group) == "nccl"


class _GatherRows(torch.autograd.Function):
    """Forward: all-gather equal row shards; backward: sum-reduce-scatter."""

    @staticmethod
    def forward(ctx, shard: torch.Tensor, group, world: int, rank: int, rows: int):
        shard = shard.contiguous()
        per = shard.shape[0]
        full = torch.empty((per * world,) + tuple(shard.shape[1:]), dtype=shard.dtype,
                           device=shard.device)
        dist.all_gather_into_tensor(full, shard, group=group)
        ctx.group, ctx.world, ctx.rank, ctx.per, ctx.rows = group, world, rank, per, rows
        return full[:rows]

    @staticmethod
    def backward(ctx, grad_rows: torch.Tensor):
        per, world = ctx.per, ctx.world
        grad = torch.zeros((per * world,) + tuple(grad_rows.shape[1:]), dtype=grad_rows.dtype,
                           device=grad_rows.device)
        grad[: ctx.rows] = grad_rows
        if _has_reduce_scatter(ctx.group):
            out = torch.empty((per,) + tuple(grad.shape[1:]), dtype=grad.dtype, device=grad.device)
            dist.reduce_scatter_tensor(out, grad, op=dist.ReduceOp.SUM, group=ctx.group)
        else:
            dist.all_reduce(grad, op=dist.ReduceOp.SUM, group=ctx.group)
            out = grad[ctx.rank * per:(ctx.rank + 1) * per].clone()
        return out, None, None, None, None


def materialize_lm_weight(lm_weight: torch.Tensor, grad_reduce_group=None) -> torch.Tensor:
    """Regular ``[vocab, hidden]`` head with gradient-correct reduction semantics.

    ``lm_weight``: a regular tensor (returned unchanged) or a DTensor sharded on
    dim 0 over a 1-D device mesh.  ``grad_reduce_group``: the ranks that
    contribute independent token losses; its size must match the mesh.
    """
    if not _is_dtensor(lm_weight):
        return lm_weight
    from torch.distributed.tensor import Replicate, Shard

    mesh = lm_weight.device_mesh
    placements = tuple(lm_weight.placements)
    if mesh.ndim != 1:
        raise ValueError("materialize_lm_weight supports a 1-D device mesh")
    if all(isinstance(p, Replicate) for p in placements):
        return lm_weight.to_local()
    if not (len(placements) == 1 and isinstance(placements[0], Shard) and placements[0].dim == 0):
        raise ValueError(f"unsupported head placement {placements}: expected Shard(0)")
    if grad_reduce_group is None:
        if lm_weight.requires_grad:
            raise ValueError("a trainable sharded head needs grad_reduce_group: without it each "
                             "rank would keep only its own slice of a rank-local gradient")
        grad_reduce_group = mesh.get_group()
    world = dist.get_world_size(grad_reduce_group)
    if world != mesh.size():
        raise ValueError(f"grad_reduce_group has {world} ranks but the head is sharded over "
                         f"{mesh.size()}")
    rank = dist.get_rank(grad_reduce_group)
    rows = lm_weight.shape[0]
    per = -(-rows // world)
    local = lm_weight.to_local()
    if local.shape[0] < per:  # uneven last shards: pad to equal rows for the collective
        pad = torch.zeros((per - local.shape[0],) + tuple(local.shape[1:]), dtype=local.dtype,
                          device=local.device)
        local = torch.cat([local, pad], dim=0)
    return _GatherRows.apply(local, grad_reduce_group, world, rank, rows)


def data_parallel_fused_linear_cross_entropy(hidden, lm_weight, labels, *, num_label_tokens,
                                             grad_reduce_group=None, ignore_index: int = -100,
                                             softcap: float = 0.0,
                                             unpadded_vocab: int | None = None,
                                             fused_head_cast: bool = False):
    """Rank-local fused loss over this rank's tokens, normalised by the global
    label count; the ranks' losses sum to the global loss and the head's
    gradient reaches its shards summed over ranks.

    With FP32 master weights the gathered head is FP32; ``fused_head_cast=True``
    rounds it to BF16 inside the loss's GEMMs instead of into a BF16 copy
    (the same results, V x H x 2 bytes less memory, slower GEMMs)."""
    from .flce import fused_linear_cross_entropy

    head = materialize_lm_weight(lm_weight, grad_reduce_group)
    return fused_linear_cross_entropy(hidden, head, labels, ignore_index=ignore_index,
                                      softcap=softcap, unpadded_vocab=unpadded_vocab,
                                      reduction="sum", num_label_tokens=num_label_tokens,
                                      fused_head_cast=fused_head_cast)
