"""Rollout inputs generated on the GPU (torch's Philox generator).

The long-rollout workload (30 layers x 80 chunks at 480P) needs ~10^10 random
numbers; drawing them with NumPy on the host would take far longer than the run
itself.  This module builds the same kind of stream as ``kvgen.HeadStream`` --
per (layer, head, spatial position) AR(1) keys with the background band
correlated at ``ar_a_bg`` and the rest at ``ar_a_fg``, N(0,1) values and
queries, 3D RoPE at true positions for window / sink / queries and with the
frame index zeroed for bank candidates -- with torch on the device.  It is not
bit-identical to the NumPy streams (another generator); tests that check it
copy the generated tensors back to the host.
"""
from __future__ import annotations

import numpy as np

from . import Workload, frame_rotation, token_ids


class GpuLayerStream:
    """One layer's per-chunk inputs for all heads of workload ``w``, on ``device``.

    ``step(i)`` (i = 1, 2, ... in order) returns the DensityKV step inputs of
    chunk i, as torch tensors in storage precision (bf16):
    candK/candV/cand_ids (chunk i-1's tokens, the sink frame excluded), winK/winV
    (chunk i), sinkK/sinkV (frame 0) and Q (chunk i)."""

    def __init__(self, w: Workload, layer: int, device="cuda", seed: int = 0, tagged: bool = False):
        import torch
        self.w = w
        self.dev = device
        self.tagged = tagged
        self.g = torch.Generator(device=device)
        self.g.manual_seed(int(np.random.SeedSequence([w.wid, layer, seed]).generate_state(1)[0]))
        H, F, d = w.heads, w.F, w.head_dim
        rows = torch.arange(w.frame_h, device=device).repeat_interleave(w.frame_w)
        if w.background_rows > 0:
            a = torch.where(rows < w.background_rows, torch.tensor(w.ar_a_bg, device=device),
                            torch.tensor(w.ar_a_fg, device=device)).float()
            b = torch.sqrt(1.0 - a.double() ** 2).float()
        else:
            a = torch.full((F,), w.ar_a, device=device)
            b = torch.full((F,), w.ar_b, device=device)
        self.a, self.b = a[None, :, None], b[None, :, None]
        self.k_last = None           # raw key of the newest frame [H][F][d] fp32
        self.frames = 0              # frames drawn so far
        self.prev = None             # (raw K [H][C*F][d], V, frame list) of the previous chunk
        self.sink = None             # (K, V) of frame 0, rotated / stored
        self._rot = {}

    def _randn(self, *shape):
        import torch
        return torch.randn(*shape, device=self.dev, generator=self.g)

    def _next_raw_key(self):
        if self.k_last is None:
            k = self._randn(self.w.heads, self.w.F, self.w.head_dim)
        else:
            k = self.a * self.k_last + self.b * self._randn(self.w.heads, self.w.F, self.w.head_dim)
        self.k_last = k
        self.frames += 1
        return k

    def _rotation(self, t: int):
        import torch
        if t not in self._rot:
            if len(self._rot) > 16:
                self._rot.clear()
            cos, sin = frame_rotation(self.w, t)
            self._rot[t] = (torch.from_numpy(cos).to(self.dev), torch.from_numpy(sin).to(self.dev))
        return self._rot[t]

    def _rope(self, x, t: int):
        import torch
        cos, sin = self._rotation(t)
        x0, x1 = x[..., 0::2], x[..., 1::2]
        out = torch.empty_like(x)
        out[..., 0::2] = x0 * cos - x1 * sin
        out[..., 1::2] = x0 * sin + x1 * cos
        return out

    def _tag(self, V, frames):
        import torch
        if not self.tagged:
            return V
        ids = torch.from_numpy(token_ids(self.w, frames)).to(self.dev)
        V = V.clone()
        V[..., 0] = (ids % 256).float()
        V[..., 1] = ((ids // 256) % 256).float()
        V[..., 2] = ((ids // 65536) % 256).float()
        return V

    def _chunk(self, c: int):
        """Raw keys and stored values of chunk c (frames drawn in order)."""
        import torch
        C = self.w.chunk_frames
        frames = list(range(c * C, (c + 1) * C))
        assert self.frames == frames[0], "chunks must be drawn in order"
        K = torch.cat([self._next_raw_key() for _ in frames], dim=1)
        V = self._tag(self._randn(self.w.heads, C * self.w.F, self.w.head_dim), frames)
        return K, V, frames

    def step(self, i: int) -> dict:
        import torch
        w = self.w
        F = w.F
        bf = torch.bfloat16
        if self.prev is None:
            assert i == 1, "steps start at 1"
            self.prev = self._chunk(0)
            K0, V0, _ = self.prev
            self.sink = (self._rope(K0[:, :F], 0).to(bf), V0[:, :F].to(bf))
        Kp, Vp, fp = self.prev
        Kc, Vc, fc = self._chunk(i)
        # candidates: chunk i-1 without the sink frame, frame index zeroed
        cf = [t for t in fp if t != 0]
        sel = slice((len(fp) - len(cf)) * F, None)
        candK = torch.cat([self._rope(Kp[:, k * F:(k + 1) * F], 0) for k in range(len(fp)) if fp[k] != 0], dim=1)
        out = {
            "candK": candK.to(bf), "candV": Vp[:, sel].to(bf),
            "cand_ids": torch.from_numpy(token_ids(w, cf).astype(np.int32)).to(self.dev),
            "winK": torch.cat([self._rope(Kc[:, k * F:(k + 1) * F], t) for k, t in enumerate(fc)], dim=1).to(bf),
            "winV": Vc.to(bf),
            "sinkK": self.sink[0], "sinkV": self.sink[1],
            "Q": torch.cat([self._rope(self._randn(w.heads, F, w.head_dim), t) for t in fc], dim=1).to(bf),
        }
        self.prev = (Kc, Vc, fc)
        return out
