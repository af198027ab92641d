"""Host side of head-parallel admission (kv_cache_compression_post_b200.sharded)
on CPU: the head split, and the MIN exchange of the synchronised prefix between
two gloo ranks, with a stand-in bank whose begin reports a per-rank prefix."""
import os
import socket

import pytest

from kv_cache_compression_post_b200.sharded import shard_heads


def test_shard_heads_covers_every_head_once():
    for H in (1, 2, 12, 13, 64):
        for world in range(1, min(H, 8) + 1):
            spans = [shard_heads(H, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    assert shard_heads(12, 8, 0) == (0, 2) and shard_heads(12, 8, 7) == (11, 12)
    with pytest.raises(ValueError):
        shard_heads(4, 5, 0)
    with pytest.raises(ValueError):
        shard_heads(4, 2, 2)


class _StandInBank:
    """Records the calls; begin writes this rank's own prefix."""

    def __init__(self, own_prefix):
        self.own = own_prefix
        self.calls = []

    def admit_begin(self, layer, candK, candV, cand_ids, prefix, stream=None):
        prefix.fill_(self.own)
        self.calls.append(("begin", layer))

    def admit_finish(self, layer, prefix_bound, stream=None):
        self.calls.append(("finish", layer, int(prefix_bound.item())))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, own, out):
    import torch
    import torch.distributed as dist
    from kv_cache_compression_post_b200.sharded import admit_sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    bank = _StandInBank(own[rank])
    prefix = torch.zeros(1, dtype=torch.int32)
    for layer in (0, 3):
        admit_sharded(bank, layer, None, None, None, prefix)
    dist.destroy_process_group()
    out.put((rank, bank.calls))


def test_two_ranks_exchange_the_min_prefix():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    own = [4093, 517]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, own, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert res[r] == [("begin", 0), ("finish", 0, 517), ("begin", 3), ("finish", 3, 517)]
