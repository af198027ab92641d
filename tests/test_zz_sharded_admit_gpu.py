"""Head-parallel admission (kvb_admit_begin / kvb_admit_finish) on one GPU.

The four heads of the mid workload are split over two banks (heads 0-1 and
2-3), as two ranks would hold them.  Each bank's kvb_admit_begin reports its
prefix, the host takes the MIN (what the ranks' all-reduce computes), and
kvb_admit_finish completes both halves.  Stepwise against the oracle's
synchronised admit over all four heads, with the parity bar of the other
DensityKV tests (tests.gpu_util.check_admit_step: decisions equal to the
oracle's or a near-tie outcome it replays, then ids, K, rho and rho0 on every
step).  No kernel
waits on another: the two banks run one after the other on one stream."""
import pytest

import kvgen
from oracle import densitykv as dkv
from tests.gpu_util import check_admit_step, dev_ids, dev_tensor, import_oracle_banks

pytestmark = pytest.mark.gpu

SPLIT = [(0, 2), (2, 4)]


def _cfg(w, H, tau, sync=1):
    import kv_cache_compression_post_b200 as kvb
    return kvb.make_config(method=kvb.KVB_DENSITYKV, dtype=kvb.KVB_BF16, layers=1, heads=H, head_dim=w.head_dim,
                           capacity=w.capacity, max_candidates=w.chunk_tokens, tau=tau, eps=w.eps, s=w.s,
                           sync_heads=sync, max_queries=w.chunk_tokens)


def test_two_bank_head_split_matches_oracle():
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["mid"]
    tau = 1.0   # prefixes below N that differ between the two halves
    L = kvgen.LayerInputs(w, 0, tagged=True)
    p = dkv.Params(capacity=w.capacity, tau=tau, eps=w.eps, s=w.s)
    banks = [dkv.HeadBank.empty(w.head_dim) for _ in range(w.heads)]
    gb = [kvb.Bank(_cfg(w, h1 - h0, tau)) for h0, h1 in SPLIT]
    prefix = [torch.full((1,), -1, dtype=torch.int32, device="cuda") for _ in SPLIT]
    counts = []
    for i in range(1, w.n_chunks):
        x = L.step(i)
        r = dkv.admit(banks, x["cand_ids"], x["candK"], x["candV"], p)
        ids = dev_ids(x["cand_ids"])
        # each half's candidate buffers stay alive until its kvb_admit_finish has run
        cand = [(dev_tensor(x["candK"][h0:h1]), dev_tensor(x["candV"][h0:h1])) for h0, h1 in SPLIT]
        for (h0, h1), bank, pre, (cK, cV) in zip(SPLIT, gb, prefix, cand):
            import_oracle_banks(bank, banks[h0:h1], p, w)
            bank.admit_begin(0, cK, cV, ids, pre)
        bound = torch.minimum(prefix[0], prefix[1])
        for bank in gb:
            bank.admit_finish(0, bound)
        torch.cuda.synchronize()
        assert all(bank.status() == 0 for bank in gb)
        # each half's prefix: min(its heads' feasible counts, M, N), within the
        # ranges the near-tie margin allows
        N = len(x["cand_ids"])
        for (h0, h1), pre in zip(SPLIT, prefix):
            lo = min(min(dkv.feasible_bounds(p, r.score[hh], x["cand_ids"], 1e-4)[0] for hh in range(h0, h1)),
                     w.capacity, N)
            hi = min(min(dkv.feasible_bounds(p, r.score[hh], x["cand_ids"], 1e-4)[1] for hh in range(h0, h1)),
                     w.capacity, N)
            assert lo <= int(pre.item()) <= hi, (i, h0, int(pre.item()), lo, hi)
        # the layer as a whole against the oracle's synchronised step over all four
        # heads: one shared P, decisions equal or a near-tie outcome it replays
        parts = [(bank, h0, h1) for bank, (h0, h1) in zip(gb, SPLIT)]
        counts.append(check_admit_step(parts, w, p, banks, x, r, label=f"head split step {i}"))
        banks = r.banks
    print(f"\nhead split: per step (flips, oracle near ties): {counts}")
    for bank in gb:
        bank.close()


def test_begin_finish_state_errors():
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["mid"]
    x = kvgen.LayerInputs(w, 0, tagged=True).step(1)
    K, V, ids = dev_tensor(x["candK"]), dev_tensor(x["candV"]), dev_ids(x["cand_ids"])
    pre = torch.zeros(1, dtype=torch.int32, device="cuda")
    bank = kvb.Bank(_cfg(w, w.heads, 2.0))
    with pytest.raises(kvb.KvbError) as e:           # nothing begun
        bank.admit_finish(0, pre)
    assert e.value.status == 6
    bank.admit_begin(0, K, V, ids, pre)
    bank.admit(0, K, V, ids)                          # a plain admit cancels the begun step
    with pytest.raises(kvb.KvbError) as e:
        bank.admit_finish(0, pre)
    assert e.value.status == 6
    with pytest.raises(kvb.KvbError) as e:           # prefix_out is required
        kvb.kvb_admit_begin(bank.handle, 0, K, V, ids, ids.shape[0], None)
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert bank.status() == 0
    bank.close()
    indep = kvb.Bank(_cfg(w, w.heads, 2.0, sync=0))
    indep.admit_begin(0, K, V, ids, pre)
    with pytest.raises(kvb.KvbError) as e:           # a bound needs synchronised heads
        indep.admit_finish(0, pre)
    assert e.value.status == 1
    indep.admit_finish(0, None)                       # the step still completes unbounded
    torch.cuda.synchronize()
    assert indep.status() == 0
    indep.close()


def test_admit_sharded_on_a_side_stream():
    """admit_sharded with a stream that is not torch's current one (a one-rank
    NCCL group): the all-reduce must see the prefix written on that stream and the
    second half the reduced value, so the bank equals a plain kvb_admit's."""
    import os
    import socket

    import numpy as np
    import torch
    import torch.distributed as dist
    import kv_cache_compression_post_b200 as kvb
    from kv_cache_compression_post_b200.sharded import admit_sharded
    from tests.gpu_util import export_banks
    w = kvgen.WORKLOADS["mid"]
    L = kvgen.LayerInputs(w, 0, tagged=True)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1)
    try:
        side = torch.cuda.Stream()
        a, b = kvb.Bank(_cfg(w, w.heads, 1.0)), kvb.Bank(_cfg(w, w.heads, 1.0))
        prefix = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        for i in range(1, 4):
            x = L.step(i)
            K, V, ids = dev_tensor(x["candK"]), dev_tensor(x["candV"]), dev_ids(x["cand_ids"])
            torch.cuda.synchronize()
            with torch.cuda.stream(side):
                # a long kernel on the side stream first, so that a collective not
                # ordered after it would read the prefix early
                busy = torch.randn(4096, 4096, device="cuda")
                for _ in range(8):
                    busy = busy @ busy * 1e-3
            admit_sharded(a, 0, K, V, ids, prefix, stream=side)
            b.admit(0, K, V, ids)
            torch.cuda.synchronize()
            assert a.status() == 0 and b.status() == 0
            for ga, gb_ in zip(export_banks(a, 0, w.heads), export_banks(b, 0, w.heads)):
                np.testing.assert_array_equal(np.sort(ga["ids"]), np.sort(gb_["ids"]))
        a.close()
        b.close()
    finally:
        dist.destroy_process_group()
