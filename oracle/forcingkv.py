"""Forcing-KV hybrid pruning (static structural + dynamic similarity), fp64.

Forcing-KV reading notes, §3.3 "Static Structural Pruning": a static head attends
[sink frame, transition frame (the last frame before the current chunk), current
chunk].  §3.4 "Dynamic Similarity Pruning": each history frame t is split into n
segments; s_t^(j) = Cosine(K_{t,j}, K_{t+1,j}); the frame keeps
BottomK({s_t^(j)}_j, floor(r n)) -- its least similar segments.  §3.5: the
similarity is a token-wise cosine averaged over the segment, the last compressed
frame is compared with the first frame of the new chunk, kept segment indices are
sorted, and a dynamic head attends [sink, retained history, current chunk].

Readings taken:

* segments are seg_h x seg_w spatial tiles of the frame_h x frame_w token grid,
  numbered row-major; edge tiles are partial (ceil division), and a segment's
  similarity is the mean over the tokens it has (30 x 52 with 4 x 4 -> 104
  segments, the 13 of the last row have 2 x 4 tokens);
* cosine(a, b) = a.b / max(||a|| ||b||, 1e-8);
* the successor of frame t is frame t+1 (the pages' direction);
* BottomK per frame (the pages' formula); ties go to the lower segment index;
  kept segments are emitted in ascending index, tokens row-major inside each;
* the dynamic history is a FIFO of the last ``hist_frames`` pruned frames; the
  sink frame (frame 0) is kept whole and separately and never enters it;
* head labels are inputs (the offline profiling step needs a trained model).

Variant (off by default): ``bottomk_scope="global"`` follows the reading notes'
§3.5 listing instead of the §3.4 formula: the similarities of all frames pushed
by one call are ranked together and floor(r * n_frames * n) (frame, segment)
pairs are kept, so a frame can keep more or fewer than floor(r n) segments; ties
go to the lower (frame, segment) position.

Variant (off by default): the first-block similarity proxy of the reading notes'
implementation notes (§3.4, and the §3.5 listing's comment): the segment
similarities are computed on the first DiT block's keys only, and the indices
they select are reused by the later blocks.  ``prune_hybrid(..., sim_keys=...)``
takes those first-block keys; a layer then keeps, in each of its frames, the
segments the first block's similarities select, and stores its own K and V at
those positions.  Reading: the sharing is per head (head h of every layer reuses
head h's selection of the first layer), and the first layer computes the
similarities of every head, whatever its own static/dynamic label, so that a
head that is dynamic only in a later layer has a selection to reuse.
"""
from __future__ import annotations

import dataclasses
import math
from collections import deque
from typing import List

import numpy as np


@dataclasses.dataclass
class Params:
    frame_h: int
    frame_w: int
    seg_h: int
    seg_w: int
    retention: float
    hist_frames: int
    bottomk_scope: str = "frame"     # "frame" (per-frame BottomK) | "global" (over the call's frames)

    @property
    def F(self) -> int:
        return self.frame_h * self.frame_w


def segments(frame_h: int, frame_w: int, seg_h: int, seg_w: int) -> List[np.ndarray]:
    """Token indices (row-major inside each) of every segment, segments row-major."""
    out = []
    for r0 in range(0, frame_h, seg_h):
        for c0 in range(0, frame_w, seg_w):
            rows = np.arange(r0, min(r0 + seg_h, frame_h))
            cols = np.arange(c0, min(c0 + seg_w, frame_w))
            out.append((rows[:, None] * frame_w + cols[None, :]).reshape(-1))
    return out


def keep_count(n_segments: int, retention: float) -> int:
    """floor(r * n) -- the number of segments a frame keeps."""
    return int(math.floor(retention * n_segments + 1e-9))


def token_cosine(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    num = np.einsum("ij,ij->i", A, B)
    den = np.sqrt(np.einsum("ij,ij->i", A, A)) * np.sqrt(np.einsum("ij,ij->i", B, B))
    return num / np.maximum(den, 1e-8)


def segment_similarity(Kt: np.ndarray, Knext: np.ndarray, segs: List[np.ndarray]) -> np.ndarray:
    """s^(j) = mean over tokens p of segment j of cos(K_t[p], K_{t+1}[p])."""
    c = token_cosine(Kt, Knext)
    return np.array([c[s].mean() for s in segs])


def bottom_k(sim: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k smallest similarities (ties: lower index), ascending."""
    order = np.lexsort((np.arange(sim.shape[0]), sim))
    return np.sort(order[:k])


@dataclasses.dataclass
class Frame:
    ids: np.ndarray
    K: np.ndarray
    V: np.ndarray


class HeadState:
    def __init__(self, static: bool):
        self.static = static
        self.transition: Frame | None = None   # static heads
        self.ring: deque = deque()             # dynamic heads: pruned frames, oldest first
        self.sims: list = []                   # last prune's similarities (dynamic heads)
        self.kept: list = []                   # last prune's kept segment lists


def prune_hybrid(states: List[HeadState], p: Params, newK, newV, new_ids, nextK, sim_keys=None):
    """Push the frames of a finalised chunk into each head's history.

    newK/newV [H][n_frames*F][d], new_ids [n_frames*F], nextK [H][F][d] (the first
    frame of the next chunk: the successor of the last new frame).  ``sim_keys``
    = (newK0, nextK0): the first block's keys of the same frames, from which the
    similarities are computed instead of this layer's own (first-block proxy)."""
    F = p.F
    segs = segments(p.frame_h, p.frame_w, p.seg_h, p.seg_w)
    kkeep = keep_count(len(segs), p.retention)
    n_frames = np.asarray(new_ids).shape[0] // F
    for hh, st in enumerate(states):
        K = np.asarray(newK[hh], np.float64).reshape(n_frames, F, -1)
        V = np.asarray(newV[hh], np.float64).reshape(n_frames, F, -1)
        ids = np.asarray(new_ids, np.int64).reshape(n_frames, F)
        if st.static:
            st.transition = Frame(ids[-1], K[-1], V[-1])
            continue
        st.sims, st.kept = [], []
        if sim_keys is None:
            Ks, nxt = K, np.asarray(nextK[hh], np.float64)
        else:
            Ks = np.asarray(sim_keys[0][hh], np.float64).reshape(n_frames, F, -1)
            nxt = np.asarray(sim_keys[1][hh], np.float64)
        sims = [segment_similarity(Ks[t], Ks[t + 1] if t + 1 < n_frames else nxt, segs) for t in range(n_frames)]
        keeps = _keep_sets(p, sims, kkeep)
        for t in range(n_frames):
            sim, keep = sims[t], keeps[t]
            tok = np.concatenate([segs[j] for j in keep]) if keep.size else np.zeros(0, np.int64)
            st.ring.append(Frame(ids[t][tok], K[t][tok], V[t][tok]))
            st.sims.append(sim)
            st.kept.append(keep)
            while len(st.ring) > p.hist_frames:
                st.ring.popleft()


def _keep_sets(p: Params, sims: List[np.ndarray], kkeep: int) -> List[np.ndarray]:
    """Kept segment indices (ascending) of each frame: BottomK per frame, or one
    BottomK over every (frame, segment) pair of the call (global scope)."""
    if p.bottomk_scope != "global":
        return [bottom_k(sim, kkeep) for sim in sims]
    n = sims[0].size
    flat = bottom_k(np.concatenate(sims), keep_count(n * len(sims), p.retention))
    return [flat[flat // n == t] - t * n for t in range(len(sims))]


def history(st: HeadState, d: int):
    """(ids, K, V) of a head's retained history between the sink and the chunk."""
    frames = [st.transition] if st.static else list(st.ring)
    frames = [f for f in frames if f is not None]
    if not frames:
        return np.zeros(0, np.int64), np.zeros((0, d)), np.zeros((0, d))
    return (np.concatenate([f.ids for f in frames]), np.concatenate([f.K for f in frames]),
            np.concatenate([f.V for f in frames]))


def attention_set(st: HeadState, sinkK, sinkV, winK, winV):
    d = np.shape(sinkK)[-1]
    _, K, V = history(st, d)
    Kall = np.concatenate([np.asarray(sinkK, np.float64), K, np.asarray(winK, np.float64)])
    Vall = np.concatenate([np.asarray(sinkV, np.float64), V, np.asarray(winV, np.float64)])
    return Kall, Vall
