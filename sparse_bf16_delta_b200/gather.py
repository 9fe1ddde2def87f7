"""Gathering the ranks' shard deltas to one rank over ``torch.distributed``.

The protocol of the verl PR's ``gather_v_batched_to_rank0`` (review of verl PR
#6974, key source snippets, sparse_gather.py): one all_gather of the ranks'
per-parameter counts, each rank's concatenated positions and values padded to
the largest total, gathered to the destination, which splits them by the
counts and concatenates, per parameter, the ranks' pieces in rank order.

Here a rank's delta is the dws layout of ``dws_encode_global`` (offsets
int64[T+1], int64 global positions, bf16 bits), so the all_gather carries the
offsets (the counts are their differences) and the split-and-concatenate on
the destination is ``dws_merge_shards``, a libdws kernel.  This module is host
plumbing only: it moves buffers with collectives and calls the merge.
"""
from __future__ import annotations


def gather_to_rank0(delta, plan=None, group=None, dst: int = 0, merge=None):
    """Collective over ``group``: every rank calls it with its own delta (same
    number of tensors T everywhere), in the same order as its other
    collectives.

    delta: this rank's ``Delta`` with int64 global positions
      (``DeltaPlan.encode_global``).
    plan: on ``dst``, the ``DeltaPlan`` of the T tensors that runs the libdws
      merge (ignored elsewhere, and when ``merge`` is given).
    merge: optional callable ``merge(rank_offsets [R, T+1], rank_indices
      [R, stride], rank_values [R, stride]) -> Delta`` replacing the libdws
      merge (the buffers are the gathered ones, row r = rank r, padded).

    Steps, identical on every rank: (1) all_gather of the offsets; (2) pad
    the positions and values to the largest total (at least one entry, so no
    collective moves an empty tensor); (3) gather the padded positions, then
    the padded values (as bytes), to ``dst``; (4) on ``dst``, merge.
    Returns the merged ``Delta`` on ``dst`` and None on the other ranks."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    offsets = delta.offsets.contiguous()
    dev = offsets.device

    # (1) every rank learns every rank's layout
    all_offs = [torch.empty_like(offsets) for _ in range(world)]
    dist.all_gather(all_offs, offsets, group=group)
    totals = [int(o[-1].item()) for o in all_offs]
    stride = max(1, max(totals))

    # (2) pad to the largest total
    n = totals[rank]
    pidx = torch.zeros(stride, dtype=torch.int64, device=dev)
    pval = torch.zeros(stride, dtype=torch.int16, device=dev)
    if n:
        pidx[:n] = delta.indices[:n]
        pval[:n] = delta.values[:n].view(torch.int16)

    # (3) gather to dst; values travel as bytes (every backend moves uint8)
    pbytes = pval.view(torch.uint8)
    if rank == dst:
        gi = [torch.empty_like(pidx) for _ in range(world)]
        gv = [torch.empty_like(pbytes) for _ in range(world)]
    else:
        gi = gv = None
    dist.gather(pidx, gi, dst=dst, group=group)
    dist.gather(pbytes, gv, dst=dst, group=group)
    if rank != dst:
        return None

    # (4) split and concatenate
    rank_offsets = torch.stack(all_offs)
    rank_indices = torch.stack(gi)
    rank_values = torch.stack([g.view(torch.int16) for g in gv])
    if merge is not None:
        return merge(rank_offsets, rank_indices, rank_values)
    if plan is None:
        raise ValueError("gather_to_rank0: the destination needs the plan (or a merge)")
    if rank_indices.device.type != "cuda":
        raise ValueError("gather_to_rank0: the libdws merge needs CUDA tensors")
    return plan.merge_shards(rank_offsets, rank_indices, rank_values)
