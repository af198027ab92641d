"""GPU parity of kvb_attend (tcgen05 flash attention over ragged [sink | bank |
window] segments) against the fp64 oracle: bf16 within 2e-2 absolute, fp32
within 1e-4.  The bank contents come from the oracle (imported), so every
step is compared on identical inputs."""
import numpy as np
import pytest

import kvgen
from oracle import densitykv as dkv
from oracle.attention import attention
from tests.gpu_util import dev_ids, dev_tensor, host, import_oracle_banks

pytestmark = pytest.mark.gpu

ATOL_BF16 = 2e-2


def _cfg(w, layers=1, max_queries=None):
    import kv_cache_compression_post_b200 as kvb
    return kvb.make_config(method=kvb.KVB_DENSITYKV, dtype=kvb.KVB_BF16 if w.dtype == "bf16" else kvb.KVB_F32,
                           layers=layers, heads=w.heads, head_dim=w.head_dim, capacity=w.capacity,
                           max_candidates=w.chunk_tokens, tau=w.tau, eps=w.eps, s=w.s,
                           max_queries=max_queries or w.chunk_tokens)


def _attend(bank, w, x, with_sink=True):
    import torch
    dt = w.dtype
    Q = dev_tensor(x["Q"], dt)
    O = torch.empty_like(Q)
    lse = torch.empty(Q.shape[0], Q.shape[1], device="cuda")
    if with_sink:
        sK, sV = dev_tensor(x["sinkK"], dt), dev_tensor(x["sinkV"], dt)
    else:
        sK = sV = torch.empty(w.heads, 0, w.head_dim, device="cuda",
                              dtype=torch.bfloat16 if dt == "bf16" else torch.float32)
    bank.attend(0, Q, sK, sV, dev_tensor(x["winK"], dt), dev_tensor(x["winV"], dt), O, lse)
    torch.cuda.synchronize()
    assert bank.status() == 0
    return host(O), host(lse)


@pytest.mark.parametrize("name", ["mid", "tiny"])
def test_attend_rollout_matches_oracle(name):
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS[name]
    L = kvgen.LayerInputs(w, 0)
    p = dkv.Params(capacity=w.capacity, tau=w.tau, eps=w.eps, s=w.s)
    res = dkv.rollout(L, p, w.n_chunks - 1, attend=True)
    bank = kvb.Bank(_cfg(w))
    atol = ATOL_BF16 if w.dtype == "bf16" else 1e-4
    for rec in res:
        import_oracle_banks(bank, rec["admit"].banks, p, w)
        O, lse = _attend(bank, w, rec["inputs"])
        for hh in range(w.heads):
            O_ref, lse_ref = rec["attn"][hh]
            np.testing.assert_allclose(O[hh], O_ref, atol=atol, rtol=0)
            np.testing.assert_allclose(lse[hh], lse_ref, atol=2e-3 if w.dtype == "bf16" else 1e-4, rtol=0)
    bank.close()


@pytest.mark.parametrize("bank_size", [0, 1, 127, 129, 300])
def test_attend_ragged_bank_sizes_and_no_sink(bank_size):
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["mid"]
    L = kvgen.LayerInputs(w, 0)
    x = L.step(3)
    rng = np.random.default_rng(bank_size)
    banks = []
    for hh in range(w.heads):
        n = max(0, bank_size - hh)          # per-head sizes differ
        ids = np.arange(n) + 10 ** 6
        K = kvgen.round_bf16(rng.standard_normal((n, w.head_dim)).astype(np.float32))
        V = kvgen.round_bf16(rng.standard_normal((n, w.head_dim)).astype(np.float32))
        banks.append(dkv.HeadBank(ids, K.astype(np.float64), V.astype(np.float64), np.ones(n)))
    p = dkv.Params(capacity=w.capacity)
    bank = kvb.Bank(_cfg(w))
    import_oracle_banks(bank, banks, p, w)
    for with_sink in (True, False):
        O, lse = _attend(bank, w, x, with_sink)
        for hh in range(w.heads):
            sK = x["sinkK"][hh] if with_sink else np.zeros((0, w.head_dim))
            sV = x["sinkV"][hh] if with_sink else np.zeros((0, w.head_dim))
            K, V = dkv.attention_set(banks[hh], sK, sV, x["winK"][hh], x["winV"][hh])
            O_ref, lse_ref = attention(x["Q"][hh], K, V)
            np.testing.assert_allclose(O[hh], O_ref, atol=ATOL_BF16, rtol=0)
            np.testing.assert_allclose(lse[hh], lse_ref, atol=2e-3, rtol=0)
    bank.close()


@pytest.mark.parametrize("name,H", [("wan480", 4), ("wan1080", 1)])
def test_attend_full_size_sampled_rows(name, H):
    """480P shapes: 4680 queries over 1560 sink + 9360 bank + 4680 window keys;
    1080P: 24480 queries over 8160 + 32640 + 24480 keys.  Fewer heads keep the
    host-side generation short; the shapes per head are full size."""
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS[name]
    L = kvgen.LayerInputs(w, 0, n_chunks=5, heads=range(H))
    x = L.step(4)
    rng = np.random.default_rng(1)
    banks = []
    for hh in range(H):
        n = w.capacity - 37 * hh
        K = kvgen.round_bf16((0.9 * x["winK"][hh][rng.integers(0, w.chunk_tokens, n)] +
                              0.44 * rng.standard_normal((n, w.head_dim))).astype(np.float32))
        V = kvgen.round_bf16(rng.standard_normal((n, w.head_dim)).astype(np.float32))
        banks.append(dkv.HeadBank(np.arange(n), K.astype(np.float64), V.astype(np.float64), np.ones(n)))
    cfg = kvb.make_config(method=kvb.KVB_DENSITYKV, dtype=kvb.KVB_BF16, heads=H, head_dim=w.head_dim,
                          capacity=w.capacity, max_candidates=w.chunk_tokens, max_queries=w.chunk_tokens)
    bank = kvb.Bank(cfg)
    import_oracle_banks(bank, banks, dkv.Params(capacity=w.capacity), w, densities=False)  # attention reads K, V only
    kvb.kvb_trace_enable(True)
    O, lse = _attend(bank, w, x)
    trace = kvb.kvb_trace_read()
    kvb.kvb_trace_enable(False)
    # the launch trace saw exactly the one attention launch, with a device time
    assert [n for n, _ in trace] == ["attend_bf16_kernel"] and trace[0][1] > 0
    for hh in range(H):
        idx = np.sort(rng.choice(w.chunk_tokens, 16, replace=False))
        K, V = dkv.attention_set(banks[hh], x["sinkK"][hh], x["sinkV"][hh], x["winK"][hh], x["winV"][hh])
        O_ref, lse_ref = attention(x["Q"][hh][idx], K, V)
        np.testing.assert_allclose(O[hh][idx], O_ref, atol=ATOL_BF16, rtol=0)
        np.testing.assert_allclose(lse[hh][idx], lse_ref, atol=2e-3, rtol=0)
    bank.close()


@pytest.mark.parametrize("nq", [1, 129, 300])
def test_attend_fewer_queries_than_max(nq):
    """Nq below max_queries (one query; a ragged second tile; three tiles, so one
    unit holds a lone tile) with the full window and a bank of ragged sizes."""
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["mid"]
    L = kvgen.LayerInputs(w, 0)
    x = dict(L.step(3))
    x["Q"] = x["Q"][:, :nq]
    rng = np.random.default_rng(nq)
    banks = []
    for hh in range(w.heads):
        n = 200 + 37 * hh
        K = kvgen.round_bf16(rng.standard_normal((n, w.head_dim)).astype(np.float32))
        V = kvgen.round_bf16(rng.standard_normal((n, w.head_dim)).astype(np.float32))
        banks.append(dkv.HeadBank(np.arange(n) + 10 ** 6, K.astype(np.float64), V.astype(np.float64), np.ones(n)))
    p = dkv.Params(capacity=w.capacity)
    bank = kvb.Bank(_cfg(w))
    import_oracle_banks(bank, banks, p, w)
    O, lse = _attend(bank, w, x)
    for hh in range(w.heads):
        K, V = dkv.attention_set(banks[hh], x["sinkK"][hh], x["sinkV"][hh], x["winK"][hh], x["winV"][hh])
        O_ref, lse_ref = attention(x["Q"][hh], K, V)
        np.testing.assert_allclose(O[hh], O_ref, atol=ATOL_BF16, rtol=0)
        np.testing.assert_allclose(lse[hh], lse_ref, atol=2e-3, rtol=0)
    bank.close()
