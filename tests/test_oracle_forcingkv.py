"""Pins of the oracle's Forcing-KV hybrid prune (reading notes §3.3, §3.4, §3.5).

Hand-built frames with known cosines, partition counts of the 4x4 segmentation of
a 30x52 frame, the r = 1 and identical-frame special cases, the static-head set
[sink, transition, current chunk] and the FIFO length of the dynamic history."""
import math

import numpy as np
import pytest

import kvgen
from oracle import forcingkv as fkv


def test_segment_partition_480p():
    segs = fkv.segments(30, 52, 4, 4)
    assert len(segs) == 8 * 13 == 104
    sizes = np.array([s.size for s in segs])
    assert (sizes == 16).sum() == 91 and (sizes == 8).sum() == 13
    allt = np.sort(np.concatenate(segs))
    np.testing.assert_array_equal(allt, np.arange(1560))
    # segment 0 = rows 0..3, cols 0..3 in row-major order
    np.testing.assert_array_equal(segs[0], [0, 1, 2, 3, 52, 53, 54, 55, 104, 105, 106, 107, 156, 157, 158, 159])
    assert fkv.keep_count(104, 0.7) == 72      # floor(72.8)
    assert fkv.keep_count(6, 0.3) == 1         # the pages' default n=6, r=0.3
    assert fkv.keep_count(104, 1.0) == 104


def test_contiguous_segments_as_a_one_row_frame():
    """The pages' n = 6 contiguous segments of a frame (Forcing-KV §3.4 and its
    implementation notes: the frame's tokens reshaped into n runs) are the 1 x F
    view of the row-major frame cut into 1 x F/n tiles."""
    F = 30 * 52
    segs = fkv.segments(1, F, 1, F // 6)
    assert len(segs) == 6
    for j, sg in enumerate(segs):
        np.testing.assert_array_equal(sg, np.arange(j * 260, (j + 1) * 260))
    # a length that does not divide: the last run is partial
    segs = fkv.segments(1, 10, 1, 4)
    assert [sg.tolist() for sg in segs] == [[0, 1, 2, 3], [4, 5, 6, 7], [8, 9]]
    assert fkv.keep_count(6, 0.33) == 1


def test_hand_built_cosines_and_bottom_k():
    # frame 2 x 4 tokens, 2 x 2 segments -> segment 0 = tokens {0,1,4,5}, segment 1 = {2,3,6,7}
    Kt = np.array([[1, 0]] * 8, dtype=np.float64)
    Kn = Kt.copy()
    Kn[[2, 3, 6, 7]] = [0, 1]                     # segment 1 turns 90 degrees: cos 0
    Kn[[0]] = [1, 1]                              # one token of segment 0 at 45 degrees
    segs = fkv.segments(2, 4, 2, 2)
    np.testing.assert_array_equal(segs[1], [2, 3, 6, 7])
    sim = fkv.segment_similarity(Kt, Kn, segs)
    assert sim[0] == pytest.approx((3 + 1 / math.sqrt(2)) / 4, rel=1e-14)
    assert sim[1] == pytest.approx(0.0, abs=1e-15)
    # the least similar segment is kept
    np.testing.assert_array_equal(fkv.bottom_k(sim, 1), [1])
    # opposite direction counts as least similar (cos -1)
    Kn2 = Kt.copy()
    Kn2[[0, 1, 4, 5]] = [-2, 0]
    sim2 = fkv.segment_similarity(Kt, Kn2, segs)
    np.testing.assert_allclose(sim2, [-1.0, 1.0], rtol=1e-15)
    np.testing.assert_array_equal(fkv.bottom_k(sim2, 1), [0])
    # zero-norm tokens give cos 0 (norm product clamped), not NaN
    assert fkv.token_cosine(np.zeros((1, 2)), np.ones((1, 2)))[0] == 0.0


def _two_frame_chunk(d=2):
    """Frames 1 and 2 (2 x 4 tokens, 2 x 2 segments) and the next chunk's first
    frame, built so that both of frame 1's segments change more than either of
    frame 2's: cos(frame1 seg0 -> frame2) = 0, seg1 = 0.5; frame 2 -> next:
    seg0 = 0.8, seg1 = 0.9 (every token of a segment turns by the same angle)."""
    F = 8
    segs = fkv.segments(2, 4, 2, 2)
    base = np.zeros((F, d))
    base[:, 0] = 1.0

    def turned(cos_by_seg, ref):
        out = ref.copy()
        for j, c in enumerate(cos_by_seg):
            for k in segs[j]:
                a = np.arctan2(ref[k, 1], ref[k, 0]) + np.arccos(c)
                out[k] = [np.cos(a), np.sin(a)]
        return out
    f1 = base
    f2 = turned([0.0, 0.5], f1)
    nxt = turned([0.8, 0.9], f2)
    K = np.concatenate([f1, f2])[None]
    return K, nxt[None], np.arange(8, 24)


def test_global_bottom_k_ranks_all_frames_of_the_call_together():
    """The listing's variant: 2 frames x 2 segments at r = 0.5 keep floor(0.5*4) = 2
    (frame, segment) pairs overall -- both of frame 1's, none of frame 2's --
    where the per-frame formula keeps one segment of each frame."""
    K, nxt, ids = _two_frame_chunk()
    V = K.copy()
    per = fkv.Params(2, 4, 2, 2, 0.5, 8)
    glob = fkv.Params(2, 4, 2, 2, 0.5, 8, bottomk_scope="global")
    a, b = [fkv.HeadState(False)], [fkv.HeadState(False)]
    fkv.prune_hybrid(a, per, K, V, ids, nxt)
    fkv.prune_hybrid(b, glob, K, V, ids, nxt)
    np.testing.assert_allclose(a[0].sims[0], [0.0, 0.5], atol=1e-12)
    np.testing.assert_allclose(a[0].sims[1], [0.8, 0.9], atol=1e-12)
    assert [k.tolist() for k in a[0].kept] == [[0], [0]]
    assert [k.tolist() for k in b[0].kept] == [[0, 1], []]
    gid, _, _ = fkv.history(b[0], 2)
    np.testing.assert_array_equal(gid, ids[:8][np.concatenate(fkv.segments(2, 4, 2, 2))])
    # one frame per call: both scopes agree
    c, e = [fkv.HeadState(False)], [fkv.HeadState(False)]
    fkv.prune_hybrid(c, per, K[:, :8], V[:, :8], ids[:8], K[:, 8:])
    fkv.prune_hybrid(e, glob, K[:, :8], V[:, :8], ids[:8], K[:, 8:])
    assert [k.tolist() for k in c[0].kept] == [k.tolist() for k in e[0].kept] == [[0]]


def test_bottom_k_ties_take_lower_index_and_sorted_output():
    sim = np.array([0.5, 0.2, 0.5, 0.2, 0.9])
    np.testing.assert_array_equal(fkv.bottom_k(sim, 3), [0, 1, 3])
    np.testing.assert_array_equal(fkv.bottom_k(np.ones(6), 4), [0, 1, 2, 3])


def _run(w, steps, labels, retention=None):
    L = kvgen.LayerInputs(w, 0)
    p = fkv.Params(w.frame_h, w.frame_w, w.seg_h, w.seg_w,
                   w.retention if retention is None else retention, w.hist_frames)
    states = [fkv.HeadState(bool(s)) for s in labels]
    out = []
    for i in range(1, steps + 1):
        x = L.step(i, forcing=True)
        fkv.prune_hybrid(states, p, x["newK"], x["newV"], x["new_ids"], x["nextK"])
        out.append((i, x, [fkv.history(st, w.head_dim) for st in states]))
    return L, p, states, out


def test_static_heads_keep_sink_transition_chunk():
    w = kvgen.WORKLOADS["forcing_mid"]
    L, p, states, out = _run(w, 4, [1, 0, 1, 0])
    for i, x, hist in out:
        last = (i - 1) * w.chunk_frames + w.chunk_frames - 1
        for hh in (0, 2):
            ids, K, V = hist[hh]
            np.testing.assert_array_equal(ids, kvgen.token_ids(w, [last]))
            Kall, _ = fkv.attention_set(states[hh], x["sinkK"][hh], x["sinkV"][hh], x["winK"][hh], x["winV"][hh])
        assert Kall.shape[0] == 5 * w.F                      # sink + transition + 3-frame chunk


def test_retention_one_keeps_everything_and_ring_is_fifo():
    w = kvgen.WORKLOADS["forcing_mid"]
    L, p, states, out = _run(w, 5, [0, 0, 0, 0], retention=1.0)
    for i, x, hist in out:
        frames = list(range(1, i * w.chunk_frames))[-w.hist_frames:]
        for hh in range(4):
            np.testing.assert_array_equal(np.sort(hist[hh][0]), kvgen.token_ids(w, frames))
            # inside a frame, tokens come segment by segment (segments ascending)
            segs = fkv.segments(w.frame_h, w.frame_w, w.seg_h, w.seg_w)
            first = hist[hh][0][:w.F] - frames[0] * w.F
            np.testing.assert_array_equal(first, np.concatenate(segs))


def test_identical_frames_tie_to_lowest_segments():
    p = fkv.Params(4, 8, 2, 2, 0.5, 3)
    st = [fkv.HeadState(False)]
    # one-hot keys: every cosine is exactly 1 in floating point, so all segments tie
    K = np.tile(np.eye(16)[np.arange(32) % 16][None], (1, 2, 1))
    fkv.prune_hybrid(st, p, K, K, np.arange(64), K[:, :32])
    for sim, keep in zip(st[0].sims, st[0].kept):
        np.testing.assert_allclose(sim, 1.0, rtol=1e-14)
        np.testing.assert_array_equal(keep, [0, 1, 2, 3])


def test_dynamic_direction_uses_successor_frame():
    """The last new frame is compared with the next chunk's first frame (successor t+1)."""
    p = fkv.Params(2, 2, 1, 1, 0.5, 4)   # 4 one-token segments, keep 2
    st = [fkv.HeadState(False)]
    f0 = np.array([[1, 0], [1, 0], [1, 0], [1, 0]], float)
    nxt = np.array([[1, 0], [0, 1], [-1, 0], [1, 1]], float)     # cos 1, 0, -1, 1/sqrt2
    fkv.prune_hybrid(st, p, f0[None], f0[None], np.arange(4), nxt[None])
    np.testing.assert_allclose(st[0].sims[0], [1, 0, -1, 1 / math.sqrt(2)], atol=1e-15)
    np.testing.assert_array_equal(st[0].kept[0], [1, 2])
    np.testing.assert_array_equal(st[0].ring[0].ids, [1, 2])


def _two_layer_chunk():
    """One head, one new frame of 2 x 4 tokens in 2 x 2 segments (segment 0 =
    tokens {0, 1, 4, 5}, segment 1 = {2, 3, 6, 7}), r = 0.5 (one segment kept).
    Layer 0: segment 0 turns 90 degrees towards the next frame (cos 0), segment 1
    stays (cos 1).  Layer 1: the opposite.  Values carry (layer, token)."""
    base = np.array([[1.0, 0.0]] * 8)
    turned = lambda toks: np.array([[0.0, 1.0] if i in toks else [1.0, 0.0] for i in range(8)])
    K = [base[None], 2.0 * base[None]]
    nxt = [turned({0, 1, 4, 5})[None], 2.0 * turned({2, 3, 6, 7})[None]]
    V = [np.array([[10 * l + i, 0.0] for i in range(8)])[None] for l in (0, 1)]
    return K, V, nxt, np.arange(100, 108)


def test_first_block_proxy_selects_by_the_first_layers_keys():
    K, V, nxt, ids = _two_layer_chunk()
    p = fkv.Params(2, 4, 2, 2, 0.5, hist_frames=4)
    own = [fkv.HeadState(False)]
    fkv.prune_hybrid(own, p, K[1], V[1], ids, nxt[1])
    np.testing.assert_array_equal(own[0].kept[0], [1])            # layer 1 on its own keys: segment 1
    proxy = [fkv.HeadState(False)]
    fkv.prune_hybrid(proxy, p, K[1], V[1], ids, nxt[1], sim_keys=(K[0], nxt[0]))
    np.testing.assert_array_equal(proxy[0].kept[0], [0])          # the first layer's choice: segment 0
    hid, hK, hV = fkv.history(proxy[0], 2)
    np.testing.assert_array_equal(hid, ids[[0, 1, 4, 5]])
    np.testing.assert_array_equal(hK, K[1][0][[0, 1, 4, 5]])      # this layer's own keys and values
    np.testing.assert_array_equal(hV[:, 0], [10, 11, 14, 15])
    np.testing.assert_allclose(proxy[0].sims[0], [0.0, 1.0], atol=1e-15)


def test_first_block_proxy_with_its_own_keys_is_the_plain_prune():
    w = kvgen.WORKLOADS["forcing_mid"]
    L = kvgen.LayerInputs(w, 0, n_chunks=4, heads=range(2))
    p = fkv.Params(w.frame_h, w.frame_w, w.seg_h, w.seg_w, w.retention, w.hist_frames)
    a, b = [fkv.HeadState(False) for _ in range(2)], [fkv.HeadState(False) for _ in range(2)]
    for i in range(1, 3):
        x = L.step(i, forcing=True)
        fkv.prune_hybrid(a, p, x["newK"], x["newV"], x["new_ids"], x["nextK"])
        fkv.prune_hybrid(b, p, x["newK"], x["newV"], x["new_ids"], x["nextK"], sim_keys=(x["newK"], x["nextK"]))
    for sa, sb in zip(a, b):
        for fa, fb in zip(sa.ring, sb.ring):
            np.testing.assert_array_equal(fa.ids, fb.ids)
            np.testing.assert_array_equal(fa.K, fb.K)
