"""Seeded synthetic inputs shaped like a Wan2.1-1.3B autoregressive video rollout.

This module feeds BOTH the CUDA library's tests/bench and the fp64 oracle with the
same numbers.  It contains none of the cache-management arithmetic (no density,
no selection, no similarity, no attention): only random draws, the backbone's 3D
rotary position embedding (applied before keys ever reach a KV cache) and the
bookkeeping of which tokens form which chunk.

Recipe (the workloads of the DensityKV and Forcing-KV pages, with synthetic data
standing in for the generator's activations):

* A latent frame is a ``frame_h x frame_w`` grid of tokens (480P: 30 x 52 = 1560,
  1080P: 68 x 120 = 8160), a chunk is 3 frames.  Token id = frame*F + row*W + col.
* Raw keys, per (layer, head, spatial position), follow an AR(1) process over
  frames: k_0 ~ N(0, I), k_t = a*k_{t-1} + b*n_t.  The tiny/480P/1080P/Forcing-KV
  workloads use a = 0.9, b = 0.44; the long-rollout workload uses a = 0.95 on the
  top 60 % of rows (static background) and a = 0.5 elsewhere, b = sqrt(1 - a^2).
* Values and queries are i.i.d. N(0, 1).
* 3D RoPE (base 10000) on interleaved pairs: of the d/2 pairs, floor(d/6) rotate
  with the row index, floor(d/6) with the column index and the rest with the
  frame index (d=128: 22 t / 21 h / 21 w).  Keys that leave the local window and
  become bank candidates are rotated with frame index 0 and their true (row, col)
  -- DensityKV, Supplementary "Post-RoPE Attention Geometry": the backbones zero
  the temporal RoPE coordinate of non-local memory keys.  Window keys, sink keys
  and queries use their true frame index.  Forcing-KV caches keep true indices.
* Seeds: numpy PCG64.  Keys: one generator per (workload, layer, head) from
  SeedSequence([workload, layer, head, 0]) drawing frames in order; values and
  queries: SeedSequence([workload, layer, head, stream, frame]) per frame
  (stream 1 = values, 2 = queries); head labels: SeedSequence([workload, layer,
  0, 3]).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

STREAM_K, STREAM_V, STREAM_Q, STREAM_LABELS = 0, 1, 2, 3


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload (shapes of the pages' experiments)."""

    name: str
    wid: int                # seed namespace
    layers: int
    heads: int
    head_dim: int
    dtype: str              # "f32" or "bf16": storage precision of K/V/Q
    frame_h: int
    frame_w: int
    chunk_frames: int
    n_chunks: int
    capacity: int           # M per head (DensityKV)
    tau: float = 2.0
    eps: float = 1e-3
    s: float = 2.0
    ar_a: float = 0.9
    ar_b: float = 0.44
    background_rows: int = 0    # rows [0, background_rows) use ar_a_bg
    ar_a_bg: float = 0.95
    ar_a_fg: float = 0.5
    # Forcing-KV
    seg_h: int = 4
    seg_w: int = 4
    retention: float = 0.7
    hist_frames: int = 21
    # default seed namespace offset (see WORKLOADS["tiny"])
    seed_offset: int = 0
    # history policy the workload exercises: "densitykv" or "forcingkv"
    method: str = "densitykv"

    @property
    def F(self) -> int:
        return self.frame_h * self.frame_w

    @property
    def chunk_tokens(self) -> int:
        return self.chunk_frames * self.F

    @property
    def forcing(self) -> bool:
        return self.method == "forcingkv"

    @property
    def n_segments(self) -> int:
        """Forcing-KV segments per frame (partial edge segments included)."""
        return -(-self.frame_h // self.seg_h) * -(-self.frame_w // self.seg_w)


def _w(**kw) -> Workload:
    return Workload(**kw)


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 case: 1 layer, 2 heads, d=64, 8x8 frames, 8 chunks, M=384.
    # seed_offset 58: with it no admit/evict decision of the 7-step rollout lies
    # within 1e-4 (relative) of its threshold or of its neighbour at a cut (the
    # smallest margin is 1.16e-4); most seeds give one or two such near-ties.
    "tiny": _w(name="tiny", wid=0, layers=1, heads=2, head_dim=64, dtype="f32",
               frame_h=8, frame_w=8, chunk_frames=3, n_chunks=8, capacity=384, seed_offset=58),
    # Wan-1.3B 480P single layer: 12 heads, d=128, 30x52 frames, M=9360, 20 chunks
    "wan480": _w(name="wan480", wid=1, layers=1, heads=12, head_dim=128, dtype="bf16",
                 frame_h=30, frame_w=52, chunk_frames=3, n_chunks=20, capacity=9360),
    # full rollout: 30 layers, 80 chunks, background-correlated keys
    "rollout": _w(name="rollout", wid=2, layers=30, heads=12, head_dim=128, dtype="bf16",
                  frame_h=30, frame_w=52, chunk_frames=3, n_chunks=80, capacity=9360,
                  background_rows=18),
    # Forcing-KV hybrid prune at 480P
    "forcing480": _w(name="forcing480", wid=3, layers=30, heads=12, head_dim=128, dtype="bf16",
                     frame_h=30, frame_w=52, chunk_frames=3, n_chunks=9, capacity=9360,
                     seg_h=4, seg_w=4, retention=0.7, hist_frames=21, method="forcingkv"),
    # 1080P scale-up: 68x120 frames, M=32640, 10 chunks
    "wan1080": _w(name="wan1080", wid=4, layers=1, heads=12, head_dim=128, dtype="bf16",
                  frame_h=68, frame_w=120, chunk_frames=3, n_chunks=10, capacity=32640),
    # mid-size parity case (several tiles + ragged tails, oracle finishes in seconds)
    "mid": _w(name="mid", wid=5, layers=1, heads=4, head_dim=128, dtype="bf16",
              frame_h=10, frame_w=17, chunk_frames=3, n_chunks=7, capacity=900),
    # mid-size Forcing-KV parity case
    "forcing_mid": _w(name="forcing_mid", wid=6, layers=1, heads=4, head_dim=128, dtype="bf16",
                      frame_h=10, frame_w=18, chunk_frames=3, n_chunks=6, capacity=900,
                      seg_h=4, seg_w=4, retention=0.7, hist_frames=7, method="forcingkv"),
}


def rng_for(w: Workload, layer: int, head: int, stream: int, seed_offset: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([w.wid + 1000 * seed_offset, layer, head, stream])))


# ---------------------------------------------------------------------------------
# storage precision
# ---------------------------------------------------------------------------------
def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32).reshape(x.shape)


def to_storage(w: Workload, x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return round_bf16(x) if w.dtype == "bf16" else x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array (already bf16-representable) -> uint16 bit patterns."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------------
# 3D RoPE of the backbone
# ---------------------------------------------------------------------------------
def rope_pairs(d: int):
    """(t_pairs, h_pairs, w_pairs) for head_dim d."""
    half = d // 2
    hw = d // 6
    return half - 2 * hw, hw, hw


def _axis_freqs(n_pairs: int, base: float = 10000.0) -> np.ndarray:
    j = np.arange(n_pairs, dtype=np.float64)
    return base ** (-2.0 * j / (2.0 * n_pairs))


def rope_angles(d: int, t: np.ndarray, r: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Rotation angle per (token, pair): [n_tok][d/2] float64."""
    tp, hp, wp = rope_pairs(d)
    ang = np.concatenate([
        np.outer(t, _axis_freqs(tp)),
        np.outer(r, _axis_freqs(hp)),
        np.outer(c, _axis_freqs(wp)),
    ], axis=1)
    return ang


def apply_rope(x: np.ndarray, ang) -> np.ndarray:
    """Rotate interleaved pairs (x[2k], x[2k+1]) of x [..., n_tok, d] by ang [n_tok, d/2]
    (or by a precomputed (cos, sin) pair)."""
    x = np.asarray(x, dtype=np.float32)
    if isinstance(ang, tuple):
        cos, sin = ang
    else:
        cos = np.cos(ang).astype(np.float32)
        sin = np.sin(ang).astype(np.float32)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


# ---------------------------------------------------------------------------------
# per-(layer, head) raw streams
# ---------------------------------------------------------------------------------
class _FrameDraws:
    """i.i.d. N(0,1) frames of one stream, each frame seeded on its own."""

    def __init__(self, w, layer, head, stream, seed_offset):
        self.key = (w.wid + 1000 * seed_offset, layer, head, stream)
        self.shape = (w.F, w.head_dim)

    def __getitem__(self, t):
        if isinstance(t, (list, tuple, np.ndarray)):
            return np.stack([self[int(u)] for u in t])
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([*self.key, int(t)])))
        return g.standard_normal(self.shape, dtype=np.float32)


class HeadStream:
    """Raw (pre-RoPE) keys, values and queries of one (layer, head), frames [0, T).

    Keys follow the AR(1) recurrence (one generator, frames drawn in order); values
    and queries are drawn per frame from SeedSequence([..., stream, frame])."""

    def __init__(self, w: Workload, layer: int, head: int, n_frames: int, seed_offset: int = 0):
        F, d = w.F, w.head_dim
        self.w = w
        rk = rng_for(w, layer, head, STREAM_K, seed_offset)
        K = np.empty((n_frames, F, d), dtype=np.float32)
        if w.background_rows > 0:
            rows = np.repeat(np.arange(w.frame_h), w.frame_w)
            a = np.where(rows < w.background_rows, w.ar_a_bg, w.ar_a_fg).astype(np.float32)[:, None]
            b = np.sqrt(1.0 - a.astype(np.float64) ** 2).astype(np.float32)
        else:
            a = np.float32(w.ar_a)
            b = np.float32(w.ar_b)
        K[0] = rk.standard_normal((F, d), dtype=np.float32)
        for t in range(1, n_frames):
            K[t] = a * K[t - 1] + b * rk.standard_normal((F, d), dtype=np.float32)
        self.K = K
        self.V = _FrameDraws(w, layer, head, STREAM_V, seed_offset)
        self.Q = _FrameDraws(w, layer, head, STREAM_Q, seed_offset)


def token_ids(w: Workload, frames) -> np.ndarray:
    frames = np.asarray(list(frames), dtype=np.int64)
    return (frames[:, None] * w.F + np.arange(w.F)[None, :]).reshape(-1)


def _grid(w: Workload):
    r = np.repeat(np.arange(w.frame_h), w.frame_w).astype(np.float64)
    c = np.tile(np.arange(w.frame_w), w.frame_h).astype(np.float64)
    return r, c


_ROT_CACHE: dict = {}


def frame_rotation(w: Workload, t: int):
    """(cos, sin) [F][d/2] float32 of frame index t (cached)."""
    key = (w.frame_h, w.frame_w, w.head_dim, int(t))
    if key not in _ROT_CACHE:
        if len(_ROT_CACHE) > 256:
            _ROT_CACHE.clear()
        r, c = _grid(w)
        ang = rope_angles(w.head_dim, np.full(w.F, float(t)), r, c)
        _ROT_CACHE[key] = (np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32))
    return _ROT_CACHE[key]


def rotated_frames(w: Workload, raw: np.ndarray, frames, memory: bool) -> np.ndarray:
    """Apply 3D RoPE to raw[frames] ([n][F][d]); memory=True zeroes the frame index."""
    frames = list(frames)
    out = np.empty((len(frames), w.F, w.head_dim), dtype=np.float32)
    for i, t in enumerate(frames):
        out[i] = apply_rope(raw[t], frame_rotation(w, 0 if memory else t))
    return out


def tag_values(V: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Overwrite V[..., 0:3] with the base-256 digits of the token id.

    Integers 0..255 are exact in bf16, so the pairing of a stored value with its
    key's id can be checked after any number of moves."""
    V = V.copy()
    ids = np.asarray(ids, dtype=np.int64)
    V[..., 0] = (ids % 256).astype(np.float32)
    V[..., 1] = ((ids // 256) % 256).astype(np.float32)
    V[..., 2] = ((ids // 65536) % 256).astype(np.float32)
    return V


def untag_ids(V: np.ndarray) -> np.ndarray:
    v = np.rint(np.asarray(V[..., :3], dtype=np.float64)).astype(np.int64)
    return v[..., 0] + 256 * v[..., 1] + 65536 * v[..., 2]


class LayerInputs:
    """All per-step inputs of one layer of a rollout, in storage precision (float32 arrays).

    Step i >= 1 (chunk i is being generated, chunk i-1 has just been finalised):

    * ``cand``:  DensityKV candidates = tokens of chunk i-1 that leave the local
      window (the sink frame 0 is never a candidate), keys rotated with frame 0.
    * ``window``: chunk i keys/values (true frame index), queries of chunk i.
    * ``sink``:   frame 0 keys/values.
    * ``newK/newV/new_ids``: Forcing-KV: the frames of chunk i-1 that enter the
      history (frame 0 is the sink and never does), true frame index;
      ``nextK``: the first frame of chunk i (successor of the last new frame).
    """

    def __init__(self, w: Workload, layer: int, n_chunks: Optional[int] = None,
                 tagged: bool = False, seed_offset: Optional[int] = None, heads=None):
        self.w = w
        self.layer = layer
        self.n_chunks = n_chunks if n_chunks is not None else w.n_chunks
        self.tagged = tagged
        self.heads = list(range(w.heads)) if heads is None else list(heads)
        n_frames = self.n_chunks * w.chunk_frames
        off = w.seed_offset if seed_offset is None else seed_offset
        self.streams = [HeadStream(w, layer, h, n_frames, off) for h in self.heads]

    def _frames(self, chunk: int):
        C = self.w.chunk_frames
        return list(range(chunk * C, (chunk + 1) * C))

    def _stack(self, fn):
        return np.stack([fn(s) for s in self.streams])

    def values(self, frames) -> np.ndarray:
        w = self.w
        V = self._stack(lambda s: s.V[frames].reshape(-1, w.head_dim))
        if self.tagged:
            V = tag_values(V, token_ids(w, frames)[None, :])
        return to_storage(w, V)

    def keys(self, frames, memory: bool) -> np.ndarray:
        w = self.w
        return to_storage(w, self._stack(
            lambda s: rotated_frames(w, s.K, frames, memory).reshape(-1, w.head_dim)))

    def queries(self, frames) -> np.ndarray:
        w = self.w
        out = []
        for s in self.streams:
            qs = [apply_rope(s.Q[t], frame_rotation(w, t)) for t in frames]
            out.append(np.concatenate(qs, axis=0))
        return to_storage(w, np.stack(out))

    def candidate_frames(self, step: int):
        f = self._frames(step - 1)
        return [t for t in f if t != 0]

    def step(self, i: int, forcing: bool = False) -> dict:
        assert i >= 1
        w = self.w
        cf = self.candidate_frames(i)
        cur = self._frames(i)
        out = {
            "sinkK": self.keys([0], memory=False), "sinkV": self.values([0]),
            "winK": self.keys(cur, memory=False), "winV": self.values(cur),
            "Q": self.queries(cur),
        }
        if forcing:
            prev = cf
            out["newK"] = self.keys(prev, memory=False)
            out["newV"] = self.values(prev)
            out["new_ids"] = token_ids(w, prev).astype(np.int32)
            out["nextK"] = self.keys([cur[0]], memory=False)
        else:
            out["cand_ids"] = token_ids(w, cf).astype(np.int32)
            out["candK"] = self.keys(cf, memory=True)
            out["candV"] = self.values(cf)
        return out


def head_labels(w: Workload, layer: int) -> np.ndarray:
    """Forcing-KV static(1)/dynamic(0) head labels: Bernoulli(0.5), fixed seed per layer."""
    r = rng_for(w, layer, 0, STREAM_LABELS)
    return (r.random(w.heads) < 0.5).astype(np.uint8)

