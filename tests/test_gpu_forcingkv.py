"""GPU parity of the Forcing-KV path against the fp64 oracle (Forcing-KV reading
notes §3.3-§3.5): segment-wise cosine, per-frame BottomK into the dynamic heads'
FIFO, the static heads' transition frame, and hybrid attention."""
import numpy as np
import pytest

import kvgen
from oracle import forcingkv as fkv
from oracle.attention import attention
from tests.gpu_util import dev_ids, dev_tensor, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,dtype,H,nf", [("forcing_mid", "bf16", 4, 3), ("forcing480", "bf16", 2, 3),
                                             ("forcing_mid", "f32", 2, 2), ("wan1080", "bf16", 1, 2)])
def test_segment_cosine_matches_oracle(name, dtype, H, nf):
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS[name]
    L = kvgen.LayerInputs(w, 0, n_chunks=2, heads=range(H))
    frames = list(range(1, 1 + nf))
    K = L.keys(frames, memory=False)
    if dtype == "f32":
        K = K + np.float32(1e-3) * np.random.default_rng(0).standard_normal(K.shape).astype(np.float32)
    nxt = L.keys([1 + nf], memory=False)
    segs = fkv.segments(w.frame_h, w.frame_w, w.seg_h, w.seg_w)
    sim = torch.full((H, nf, len(segs)), float("nan"), device="cuda")
    kvb.kvb_segment_cosine(dev_tensor(K, dtype), dev_tensor(nxt, dtype), H, nf, w.frame_h, w.frame_w, w.seg_h,
                           w.seg_w, w.head_dim, kvb.KVB_BF16 if dtype == "bf16" else kvb.KVB_F32, sim)
    torch.cuda.synchronize()
    got = host(sim)
    for hh in range(H):
        Kf = K[hh].reshape(nf, w.F, -1)
        for t in range(nf):
            succ = Kf[t + 1] if t + 1 < nf else nxt[hh]
            ref = fkv.segment_similarity(Kf[t], succ, segs)
            np.testing.assert_allclose(got[hh, t], ref, atol=2e-6, rtol=0)


def _cfg(w, layers=1, **kw):
    import kv_cache_compression_post_b200 as kvb
    return kvb.make_config(method=kvb.KVB_FORCINGKV, dtype=kvb.KVB_BF16, layers=layers, heads=w.heads,
                           head_dim=w.head_dim, frame_h=w.frame_h, frame_w=w.frame_w, seg_h=w.seg_h,
                           seg_w=w.seg_w, hist_frames=w.hist_frames, max_new_frames=w.chunk_frames,
                           retention=w.retention, max_queries=w.chunk_tokens, **kw)


def _kept_near_tie(sim, k, margin=1e-4):
    order = np.lexsort((np.arange(sim.size), sim))
    if k == 0 or k >= sim.size:
        return False
    a, b = sim[order[k - 1]], sim[order[k]]
    return abs(b - a) <= margin * max(abs(a), 1e-3)


def _rollout(name, steps, labels, sample_rows=None, scope="frame", **geometry):
    """``geometry`` overrides the segmentation (frame_h, frame_w, seg_h, seg_w,
    retention) of both the library and the oracle; the inputs keep the workload's
    own frames.  ``scope``: the BottomK scope ("frame", or "global": one ranking
    over a call's frames)."""
    import dataclasses
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS[name]
    H = len(labels)
    L = kvgen.LayerInputs(w, 0, n_chunks=steps + 2, heads=range(H))
    ws = dataclasses.replace(w, heads=H, **geometry)
    p = fkv.Params(ws.frame_h, ws.frame_w, ws.seg_h, ws.seg_w, ws.retention, ws.hist_frames, bottomk_scope=scope)
    states = [fkv.HeadState(bool(s)) for s in labels]
    bank = kvb.Bank(_cfg(ws, bottomk_scope=kvb.KVB_BOTTOMK_CALL if scope == "global" else kvb.KVB_BOTTOMK_FRAME))
    rng = np.random.default_rng(0)
    tie_frames = [set() for _ in range(H)]   # frames pushed with a near-tie BottomK decision
    for i in range(1, steps + 1):
        x = L.step(i, forcing=True)
        nf = len(x["new_ids"]) // w.F
        fkv.prune_hybrid(states, p, x["newK"], x["newV"], x["new_ids"], x["nextK"])
        new_frames = [int(f) for f in x["new_ids"][::w.F] // w.F]
        for hh in range(H):
            if states[hh].static:
                continue
            if scope == "global":   # one cut over the call's frames: a near tie there touches all of them
                allsim = np.concatenate(states[hh].sims)
                if _kept_near_tie(allsim, fkv.keep_count(allsim.size, ws.retention)):
                    tie_frames[hh].update(new_frames)
                continue
            for f, s in zip(new_frames, states[hh].sims):
                if _kept_near_tie(s, fkv.keep_count(s.size, ws.retention)):
                    tie_frames[hh].add(f)
        bank.prune_hybrid(0, np.array(labels, np.uint8), dev_tensor(x["newK"], "bf16"), dev_tensor(x["newV"], "bf16"),
                          dev_tensor(x["nextK"], "bf16"), dev_ids(x["new_ids"]), nf)
        Q = dev_tensor(x["Q"], "bf16")
        O = torch.empty_like(Q)
        lse = torch.empty(H, Q.shape[1], device="cuda")
        bank.attend(0, Q, dev_tensor(x["sinkK"], "bf16"), dev_tensor(x["sinkV"], "bf16"),
                    dev_tensor(x["winK"], "bf16"), dev_tensor(x["winV"], "bf16"), O, lse)
        torch.cuda.synchronize()
        assert bank.status() == 0
        O = host(O)
        st = bank.stats(0)
        for hh in range(H):
            ids, _, _, K, V = bank.export(0, hh)
            gid, gK, gV = host(ids).astype(np.int64), host(K), host(V)
            oid, oK, oV = fkv.history(states[hh], w.head_dim)
            gf, of = gid // w.F, oid // w.F
            assert sorted(set(gf.tolist())) == sorted(set(of.tolist()))   # same frames held
            clean = True
            for f in sorted(set(of.tolist())):
                if f in tie_frames[hh]:
                    clean = False
                    continue
                np.testing.assert_array_equal(gid[gf == f], oid[of == f])
                np.testing.assert_array_equal(gK[gf == f], oK[of == f].astype(np.float32))
                np.testing.assert_array_equal(gV[gf == f], oV[of == f].astype(np.float32))
            if clean:
                assert st[hh]["size"] == len(oid)
                Kall, Vall = fkv.attention_set(states[hh], x["sinkK"][hh], x["sinkV"][hh], x["winK"][hh],
                                               x["winV"][hh])
                rows = np.arange(Q.shape[1]) if sample_rows is None else \
                    np.sort(rng.choice(Q.shape[1], sample_rows, replace=False))
                O_ref, _ = attention(x["Q"][hh][rows], Kall, Vall)
                np.testing.assert_allclose(O[hh][rows], O_ref, atol=2e-2, rtol=0)
    bank.close()


def test_forcing_mid_rollout_matches_oracle():
    # hist_frames 7 < frames pushed: the FIFO wraps and drops old frames
    _rollout("forcing_mid", 4, [1, 0, 1, 0])


def test_forcing_mid_contiguous_segments():
    # the pages' own segmentation: n = 6 contiguous runs of the row-major frame,
    # r = 0.3 (one run kept per frame)
    F = kvgen.WORKLOADS["forcing_mid"].F
    _rollout("forcing_mid", 4, [0, 1, 0, 0], frame_h=1, frame_w=F, seg_h=1, seg_w=F // 6, retention=0.3)


def test_forcing480_full_size_sampled():
    # 480P, 4 heads (2 static, 2 dynamic), 8 chunks: the 21-frame FIFO fills up
    _rollout("forcing480", 8, [0, 1, 0, 1], sample_rows=16)


def test_forcing_mid_global_bottomk():
    """The call scope of BottomK (the reading notes' §3.5 listing): the kept
    (frame, segment) pairs of each call, ranked together, against the oracle."""
    _rollout("forcing_mid", 4, [0, 1, 0, 0], scope="global")


def test_forcing_mid_first_block_proxy():
    """The first-block similarity proxy (reading notes §3.4 implementation notes):
    two layers with different keys and labels; layer 0 computes every head's
    similarities, layer 1 keeps the segments they select, filled with its own K
    and V.  Head 1 is static in layer 0 and dynamic in layer 1, so layer 1 uses a
    selection layer 0 computed for a head it did not prune by similarity."""
    import dataclasses
    import torch
    import kv_cache_compression_post_b200 as kvb
    w = kvgen.WORKLOADS["forcing_mid"]
    H, steps = 3, 4
    labels = [[0, 1, 0], [0, 0, 1]]
    Ls = [kvgen.LayerInputs(w, l, n_chunks=steps + 2, heads=range(H)) for l in range(2)]
    p = fkv.Params(w.frame_h, w.frame_w, w.seg_h, w.seg_w, w.retention, w.hist_frames)
    states = [[fkv.HeadState(bool(s)) for s in lab] for lab in labels]
    bank = kvb.Bank(_cfg(dataclasses.replace(w, heads=H), layers=2, sim_source=kvb.KVB_SIM_FIRST_LAYER))
    x1 = Ls[1].step(1, forcing=True)
    with pytest.raises(kvb.KvbError) as e:   # a later layer before layer 0 has been pruned
        bank.prune_hybrid(1, np.array(labels[1], np.uint8), dev_tensor(x1["newK"]), dev_tensor(x1["newV"]),
                          dev_tensor(x1["nextK"]), dev_ids(x1["new_ids"]), len(x1["new_ids"]) // w.F)
    assert e.value.status == 6
    ties = [set() for _ in range(H)]   # frames whose selection had a near tie (they stay in the FIFO)
    for i in range(1, steps + 1):
        xs = [L.step(i, forcing=True) for L in Ls]
        nf = len(xs[0]["new_ids"]) // w.F
        for l in range(2):
            x = xs[l]
            fkv.prune_hybrid(states[l], p, x["newK"], x["newV"], x["new_ids"], x["nextK"],
                             sim_keys=(xs[0]["newK"], xs[0]["nextK"]))
            bank.prune_hybrid(l, np.array(labels[l], np.uint8), dev_tensor(x["newK"]), dev_tensor(x["newV"]),
                              dev_tensor(x["nextK"]), dev_ids(x["new_ids"]), nf)
        # the selection is layer 0's: a near tie in its similarities touches every layer
        sims0 = [fkv.segment_similarity(xs[0]["newK"][hh].reshape(nf, w.F, -1)[t],
                                        xs[0]["newK"][hh].reshape(nf, w.F, -1)[t + 1] if t + 1 < nf
                                        else xs[0]["nextK"][hh], fkv.segments(w.frame_h, w.frame_w, w.seg_h, w.seg_w))
                 for hh in range(H) for t in range(nf)]
        new_frames = [int(f) for f in xs[0]["new_ids"][::w.F] // w.F]
        for hh in range(H):
            for t in range(nf):
                sm = sims0[hh * nf + t]
                if _kept_near_tie(sm, fkv.keep_count(sm.size, w.retention)):
                    ties[hh].add(new_frames[t])
        torch.cuda.synchronize()
        assert bank.status() == 0
        for l in range(2):
            for hh in range(H):
                ids, _, _, K, V = bank.export(l, hh)
                gid, gK, gV = host(ids).astype(np.int64), host(K), host(V)
                oid, oK, oV = fkv.history(states[l][hh], w.head_dim)
                gf, of = gid // w.F, oid // w.F
                assert sorted(set(gf.tolist())) == sorted(set(of.tolist()))
                for f in sorted(set(of.tolist())):
                    if f in ties[hh]:
                        continue
                    np.testing.assert_array_equal(gid[gf == f], oid[of == f])
                    np.testing.assert_array_equal(gK[gf == f], oK[of == f].astype(np.float32))
                    np.testing.assert_array_equal(gV[gf == f], oV[of == f].astype(np.float32))
    bank.close()


@pytest.mark.parametrize("dtype,d", [("bf16", 48), ("f32", 20), ("bf16", 80), ("f32", 72), ("bf16", 256),
                                     ("bf16", 32), ("bf16", 64), ("f32", 64), ("f32", 128)])
def test_segment_cosine_row_widths(dtype, d):
    """Every row form of the kernel: 4, 8, 16 and 32 words of 16 bytes (a lane
    holds 1, 2, 4 or 8 words of each row), word counts that are not a power of
    two (a lane group narrower than the row, looping), and wide rows; a 7 x 9
    frame in 2 x 3 segments, partial at both edges."""
    import torch
    import kv_cache_compression_post_b200 as kvb
    H, nf, fh, fw, sh, sw = 3, 2, 7, 9, 2, 3
    rng = np.random.default_rng(d)
    K = rng.standard_normal((H, nf * fh * fw, d)).astype(np.float32)
    nxt = rng.standard_normal((H, fh * fw, d)).astype(np.float32)
    if dtype == "bf16":  # the stored values, rounded on the host
        K, nxt = (torch.from_numpy(a).to(torch.bfloat16).float().numpy() for a in (K, nxt))
    segs = fkv.segments(fh, fw, sh, sw)
    sim = torch.full((H, nf, len(segs)), float("nan"), device="cuda")
    kvb.kvb_segment_cosine(dev_tensor(K, dtype), dev_tensor(nxt, dtype), H, nf, fh, fw, sh, sw, d,
                           kvb.KVB_BF16 if dtype == "bf16" else kvb.KVB_F32, sim)
    torch.cuda.synchronize()
    got = host(sim)
    for hh in range(H):
        Kf = K[hh].reshape(nf, fh * fw, d)
        for t in range(nf):
            succ = Kf[t + 1] if t + 1 < nf else nxt[hh]
            np.testing.assert_allclose(got[hh, t], fkv.segment_similarity(Kf[t], succ, segs), atol=2e-6, rtol=0)
