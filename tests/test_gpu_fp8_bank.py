"""DensityKV with the bank's K and V stored in FP8 E4M3 (kvb_config.storage =
KVB_STORE_FP8_E4M3), against the fp64 oracle with its inputs rounded by
oracle.fp8.e4m3 (to nearest, ties to even, saturating at 448):

* import + export: the stored values are the E4M3 roundings of what was imported,
  bit for bit, including ties, subnormals and saturation;
* the mid workload stepwise (tests.gpu_util.check_admit_step, every step): the
  library rounds the candidates itself; the oracle admits the rounded candidates,
  so densities, decisions and bank contents compare as with bf16 storage, K rows
  bit for bit;
* attention over the stored (rounded) bank with bf16 sink, window and queries,
  within 2e-2 of the oracle."""
import numpy as np
import pytest

import kvgen
from oracle import densitykv as dkv
from oracle import fp8
from oracle.attention import attention
from tests.gpu_util import check_admit_step, dev_ids, dev_tensor, export_banks, host, import_step_state

pytestmark = pytest.mark.gpu


def _cfg(w, **kw):
    import kv_cache_compression_post_b200 as kvb
    return kvb.make_config(method=kvb.KVB_DENSITYKV, dtype=kvb.KVB_BF16, layers=kw.pop("layers", 1), heads=w.heads,
                           head_dim=w.head_dim, capacity=w.capacity, max_candidates=w.chunk_tokens, tau=w.tau,
                           eps=w.eps, s=w.s, sync_heads=1, max_queries=w.chunk_tokens,
                           storage=kvb.KVB_STORE_FP8_E4M3, **kw)


def test_import_export_rounds_to_e4m3():
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["mid"]
    bank = kvb.Bank(_cfg(w, layers=2))
    rng = np.random.default_rng(1)
    n = 300
    K = rng.standard_normal((n, w.head_dim)).astype(np.float32) * np.float32(2.0)
    V = rng.standard_normal((n, w.head_dim)).astype(np.float32)
    # exact ties, subnormals and values past the largest finite code
    K[0, :8] = [1.0625, 1.1875, -1.0625, 2.0 ** -10, 3 * 2.0 ** -10, 460.0, -1000.0, 17.5]
    K, V = kvgen.round_bf16(K), kvgen.round_bf16(V)
    ids = np.arange(5000, 5000 + n)
    rho = np.ones(n)
    for layer in (1, 0):
        bank.import_(layer, 2, dev_ids(ids), dev_tensor(rho, "f32"), dev_tensor(rho, "f32"), dev_tensor(K, "bf16"),
                     dev_tensor(V, "bf16"))
    torch.cuda.synchronize()
    for layer in (0, 1):
        g = export_banks(bank, layer, w.heads)[2]
        np.testing.assert_array_equal(g["K"], fp8.e4m3(K).astype(np.float32))
        np.testing.assert_array_equal(g["V"], fp8.e4m3(V).astype(np.float32))
        np.testing.assert_array_equal(g["ids"], ids)
    assert bank.status() == 0
    bank.close()


def test_mid_stepwise_fp8_storage():
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["mid"]
    L = kvgen.LayerInputs(w, 0)   # untagged: E4M3 cannot hold id tags; V rows are compared by id instead
    p = dkv.Params(capacity=w.capacity, tau=w.tau, eps=w.eps, s=w.s)
    bank = kvb.Bank(_cfg(w))
    banks = [dkv.HeadBank.empty(w.head_dim) for _ in range(w.heads)]
    counts = []
    rng = np.random.default_rng(4)
    for i in range(1, w.n_chunks):
        x = L.step(i)
        # the oracle's step takes the candidates as the bank will store them
        xq = dict(x, candK=fp8.e4m3(x["candK"]), candV=fp8.e4m3(x["candV"]))
        r = dkv.admit(banks, xq["cand_ids"], xq["candK"], xq["candV"], p)
        import_step_state(bank, banks, p, w)
        bank.admit(0, dev_tensor(x["candK"]), dev_tensor(x["candV"]), dev_ids(x["cand_ids"]))
        Q = dev_tensor(x["Q"])
        O = torch.empty_like(Q)
        bank.attend(0, Q, dev_tensor(x["sinkK"]), dev_tensor(x["sinkV"]), dev_tensor(x["winK"]),
                    dev_tensor(x["winV"]), O)
        torch.cuda.synchronize()
        assert bank.status() == 0
        counts.append(check_admit_step(bank, w, p, banks, xq, r, label=f"fp8 step {i}", tagged=False))
        # attention over the stored bank (the oracle's step or its replay hold the same ids)
        g = export_banks(bank, 0, w.heads)
        Oh = host(O)
        for hh in range(w.heads):
            gb = dkv.HeadBank(g[hh]["ids"], g[hh]["K"].astype(np.float64), g[hh]["V"].astype(np.float64),
                              g[hh]["rho0"])
            Kall, Vall = dkv.attention_set(gb, x["sinkK"][hh], x["sinkV"][hh], x["winK"][hh], x["winV"][hh])
            rows = np.sort(rng.choice(w.chunk_tokens, 32, replace=False))
            ref, _ = attention(x["Q"][hh][rows], Kall, Vall)
            np.testing.assert_allclose(Oh[hh][rows], ref, atol=2e-2, rtol=0)
        banks = r.banks
    print(f"\nfp8 storage mid: per step (flips, oracle near ties): {counts}")
    bank.close()
