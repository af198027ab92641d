"""The long streaming rollout (30 layers x 80 chunks at 480P, background-correlated
keys) at reduced depth: 2 layers of one bank, 6 chunks, all 12 heads at full
per-head size, inputs from the GPU generator (kvgen.gpu).  Every step of both
layers must keep the device status clean; the last two steps of each layer are
checked on sampled outputs and invariants against the oracle (the same checks as
the full-size step test)."""
import numpy as np
import pytest

import kvgen
from tests.gpu_util import check_admit_sampled, export_banks, host

pytestmark = pytest.mark.gpu


def test_rollout_layers_sampled():
    import torch
    import kv_cache_compression_post_b200 as kvb
    from kvgen.gpu import GpuLayerStream
    w = kvgen.WORKLOADS["rollout"]
    n_layers, steps = 2, 6
    cfg = kvb.make_config(method=kvb.KVB_DENSITYKV, dtype=kvb.KVB_BF16, layers=n_layers, heads=w.heads,
                          head_dim=w.head_dim, capacity=w.capacity, max_candidates=w.chunk_tokens, tau=w.tau,
                          eps=w.eps, s=w.s, sync_heads=1, max_queries=w.chunk_tokens)
    bank = kvb.Bank(cfg)
    streams = [GpuLayerStream(w, l, tagged=True) for l in range(n_layers)]
    rng = np.random.default_rng(3)
    O = torch.empty(w.heads, w.chunk_tokens, w.head_dim, dtype=torch.bfloat16, device="cuda")
    for i in range(1, steps + 1):
        for l in range(n_layers):
            x = streams[l].step(i)
            check = i >= steps - 1
            pre = export_banks(bank, l, w.heads) if check else None
            bank.admit(l, x["candK"], x["candV"], x["cand_ids"])
            bank.attend(l, x["Q"], x["sinkK"], x["sinkV"], x["winK"], x["winV"], O)
            torch.cuda.synchronize()
            assert bank.status() == 0, (i, l)
            if check:
                post = export_banks(bank, l, w.heads)
                check_admit_sampled(w, pre, post, bank.stats(l), host(x["cand_ids"]), host(x["candK"]), rng, n=6)
    assert np.isfinite(host(O)).all()
    bank.close()
