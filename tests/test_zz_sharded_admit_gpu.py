"""Head-parallel admission (kvb_admit_begin / kvb_admit_finish) on one GPU.

The four heads of the mid workload are split over two banks (heads 0-1 and
2-3), as two ranks would hold them.  Each bank's kvb_admit_begin reports its
prefix, the host takes the MIN (what the ranks' all-reduce computes), and
kvb_admit_finish completes both halves.  Stepwise against the oracle's
synchronised admit over all four heads, with the parity bar of the other
DensityKV tests (ids exact except near ties, densities within 1e-4).  No kernel
waits on another: the two banks run one after the other on one stream."""
import dataclasses

import numpy as np
import pytest

import kvgen
from oracle import densitykv as dkv
from tests.gpu_util import dev_ids, dev_tensor, export_banks, import_oracle_banks

pytestmark = pytest.mark.gpu

RTOL = 1e-4
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
    exact_steps = 0
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
        banks = r.banks   # the next step starts from the oracle's banks whatever happens here
        # one shared P on both halves; it can differ from the oracle's only through
        # a feasibility decision within the near-tie margin (one flip in the head
        # that sets the minimum moves every head's cut), and then the step is not compared
        P_gpu = {st["admitted"] for bank in gb for st in bank.stats(0)}
        assert len(P_gpu) == 1
        P_gpu = P_gpu.pop()
        if P_gpu != r.P:
            assert abs(P_gpu - r.P) <= sum(len(t) for t in r.tie_cand_ids), (P_gpu, r.P)
            continue
        all_exact = True
        for (h0, h1), bank, pre in zip(SPLIT, gb, prefix):
            if not any(r.tie_cand_ids[h0:h1]):
                N = len(x["cand_ids"])
                assert int(pre.item()) == min(int(r.P_h[h0:h1].min()), w.capacity, N)
            g = export_banks(bank, 0, h1 - h0)
            st = bank.stats(0)
            for j, hh in enumerate(range(h0, h1)):
                ob = r.banks[hh]
                diff = set(g[j]["ids"].tolist()) ^ set(ob.ids.tolist())
                ties = r.tie_cand_ids[hh] | r.tie_bank_ids[hh]
                assert diff <= ties, f"head {hh}: ids differ outside near ties: {sorted(diff - ties)[:10]}"
                np.testing.assert_array_equal(kvgen.untag_ids(g[j]["V"]), g[j]["ids"])
                if diff:
                    all_exact = False
                    continue
                go, oo = np.argsort(g[j]["ids"]), np.argsort(ob.ids)
                np.testing.assert_array_equal(g[j]["K"][go], ob.K[oo].astype(np.float32))
                np.testing.assert_allclose(g[j]["rho"][go], r.rho_new[hh][oo], rtol=RTOL)
                np.testing.assert_allclose(g[j]["rho0"][go], ob.rho0[oo], rtol=RTOL)
                assert st[j]["admitted"] == len(r.admitted[hh]) == r.P
        exact_steps += int(all_exact)
    assert exact_steps >= (w.n_chunks - 1) // 2
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
