"""The synthetic input recipe (kvgen): AR(1) keys with the stated coefficients,
token layout, chunk bookkeeping, memory RoPE with the frame index zeroed, exact
value tags and reproducible, independent seeds.  CPU only."""
import dataclasses

import numpy as np
import pytest

import kvgen


def _lag1(K):
    """Per-(token, dim) lag-1 correlation over frames, averaged."""
    a, b = K[:-1].reshape(K.shape[0] - 1, -1), K[1:].reshape(K.shape[0] - 1, -1)
    return float((a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum()))


def test_ar1_keys_have_the_stated_correlation_and_unit_variance():
    w = dataclasses.replace(kvgen.WORKLOADS["mid"], frame_h=10, frame_w=17)
    K = kvgen.HeadStream(w, 0, 0, 60).K.astype(np.float64)
    assert _lag1(K) == pytest.approx(w.ar_a, abs=0.01)
    assert K[20:].var() == pytest.approx(w.ar_a ** 2 + w.ar_b ** 2, rel=0.03)   # 0.9^2 + 0.44^2 = 0.9936


def test_background_band_uses_its_own_coefficient():
    w = dataclasses.replace(kvgen.WORKLOADS["mid"], background_rows=6)
    K = kvgen.HeadStream(w, 0, 0, 80).K.astype(np.float64).reshape(80, w.frame_h, w.frame_w, -1)
    assert _lag1(K[:, :6]) == pytest.approx(w.ar_a_bg, abs=0.01)
    assert _lag1(K[:, 6:]) == pytest.approx(w.ar_a_fg, abs=0.03)
    assert K[20:].var() == pytest.approx(1.0, rel=0.05)                          # b = sqrt(1 - a^2)


def test_token_ids_and_chunk_bookkeeping():
    w = kvgen.WORKLOADS["mid"]
    ids = kvgen.token_ids(w, [2, 5])
    assert ids[0] == 2 * w.F and ids[w.F] == 5 * w.F
    # row-major inside a frame: id = frame*F + row*W + col
    assert ids[3 * w.frame_w + 4] == 2 * w.F + 3 * w.frame_w + 4
    L = kvgen.LayerInputs(w, 0, n_chunks=4)
    x1, x2 = L.step(1), L.step(2)
    # chunk 0 minus the sink frame, then the whole of chunk 1
    np.testing.assert_array_equal(x1["cand_ids"], kvgen.token_ids(w, [1, 2]))
    np.testing.assert_array_equal(x2["cand_ids"], kvgen.token_ids(w, [3, 4, 5]))
    assert x2["winK"].shape == (w.heads, w.chunk_tokens, w.head_dim) == x2["Q"].shape
    assert x2["sinkK"].shape == (w.heads, w.F, w.head_dim)
    # the window of step 1 is the candidate block of step 2 (same raw keys, other rotation)
    np.testing.assert_array_equal(x1["winV"], x2["candV"])
    # Forcing-KV: the frames entering the history are the previous window, keys and
    # values alike (true frame index), and the successor frame opens the window
    f1, f2 = L.step(1, forcing=True), L.step(2, forcing=True)
    np.testing.assert_array_equal(f1["winK"], f2["newK"])
    np.testing.assert_array_equal(f1["winV"], f2["newV"])
    np.testing.assert_array_equal(f2["nextK"], f2["winK"][:, :w.F])


def test_memory_keys_are_rotated_with_frame_zero():
    w = kvgen.WORKLOADS["tiny"]          # fp32 storage: exact comparisons
    L = kvgen.LayerInputs(w, 0, n_chunks=3)
    x = L.step(2)
    raw = L.streams[1].K
    cand = x["candK"][1].reshape(3, w.F, w.head_dim)
    for i, t in enumerate([3, 4, 5]):
        np.testing.assert_array_equal(cand[i], kvgen.apply_rope(raw[t], kvgen.frame_rotation(w, 0)))
    win = x["winK"][1].reshape(3, w.F, w.head_dim)
    np.testing.assert_array_equal(win[0], kvgen.apply_rope(raw[6], kvgen.frame_rotation(w, 6)))
    # the window key differs from its memory form only by the temporal rotation
    assert not np.array_equal(win[0], kvgen.apply_rope(raw[6], kvgen.frame_rotation(w, 0)))


def test_value_tags_survive_bf16_storage():
    ids = np.array([0, 1, 255, 256, 65535, 65536, 9360 * 30, 2 ** 24 - 1])
    V = kvgen.tag_values(np.zeros((ids.size, 8), np.float32), ids)
    np.testing.assert_array_equal(kvgen.untag_ids(kvgen.round_bf16(V)), ids)


def test_seeds_are_reproducible_and_independent():
    w = kvgen.WORKLOADS["mid"]
    a = kvgen.HeadStream(w, 0, 0, 3).K
    np.testing.assert_array_equal(a, kvgen.HeadStream(w, 0, 0, 3).K)
    for other in (kvgen.HeadStream(w, 0, 1, 3).K, kvgen.HeadStream(w, 1, 0, 3).K,
                  kvgen.HeadStream(w, 0, 0, 3, seed_offset=1).K):
        assert abs(np.corrcoef(a.ravel(), other.ravel())[0, 1]) < 0.02
    # per-frame value draws do not depend on which frames were drawn before
    s = kvgen.HeadStream(w, 0, 0, 1)
    np.testing.assert_array_equal(s.V[5], kvgen.HeadStream(w, 0, 0, 1).V[[2, 5]][1])
