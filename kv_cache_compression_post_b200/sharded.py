"""Head-parallel DensityKV admission across processes (one per GPU).

A layer's banks are independent per head (DensityKV App. B.1), so the heads of a
layer can live on different GPUs.  Under synchronised admission (App. E
cross-head synchronisation) they still share one admitted count P = min over
every head of the layer: that single int32 is the only data the ranks exchange,
an all-reduce (MIN) between the two halves of the admit step
(kvb_admit_begin / kvb_admit_finish).  Attention needs no exchange.

Plumbing only: the arithmetic runs in the library's kernels; the MIN goes
through torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations


def shard_heads(heads: int, world: int, rank: int) -> tuple:
    """[h0, h1): the contiguous heads rank `rank` holds; the first heads % world
    ranks take one head more.  Every rank holds at least one head."""
    if not (1 <= world <= heads) or not (0 <= rank < world):
        raise ValueError(f"cannot split {heads} heads over {world} ranks (rank {rank})")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def admit_sharded(bank, layer: int, candK, candV, cand_ids, prefix, group=None, stream=None) -> None:
    """One synchronised admit step of this rank's heads of `layer`.

    ``bank`` holds this rank's heads (a ``kvb.Bank`` or anything with
    ``admit_begin`` / ``admit_finish``); candK/candV are this rank's head slices
    [H_rank][N][d]; cand_ids [N] is the same on every rank; ``prefix`` is a
    one-element int32 tensor on this rank's device, reused across calls.  Every
    rank of ``group`` must call this for the same layer and block.

    ``stream`` (a torch.cuda.Stream or None for the current stream) carries the
    whole step: the collective is issued with it as torch's current stream, so
    torch orders the all-reduce after the prefix is written and the second half
    after the reduced value has landed."""
    import contextlib

    import torch
    import torch.distributed as dist
    ctx = torch.cuda.stream(stream) if (stream is not None and prefix.is_cuda) else contextlib.nullcontext()
    with ctx:
        bank.admit_begin(layer, candK, candV, cand_ids, prefix, stream)
        dist.all_reduce(prefix, op=dist.ReduceOp.MIN, group=group)
        bank.admit_finish(layer, prefix, stream)
