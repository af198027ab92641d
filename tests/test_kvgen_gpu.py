"""The torch rollout generator (kvgen.gpu), run on the CPU device: shapes and
storage type, id tags, and that a token's candidate key is its window key with the
frame index of the rotation zeroed (the same raw key, another rotation)."""
import dataclasses

import numpy as np

import kvgen
from kvgen.gpu import GpuLayerStream


def _unrotate(x, w, t):
    cos, sin = kvgen.frame_rotation(w, t)
    x = np.asarray(x, np.float64)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * cos + x1 * sin
    out[..., 1::2] = -x0 * sin + x1 * cos
    return out


def test_rollout_stream_shapes_tags_and_rotations():
    import torch
    w = dataclasses.replace(kvgen.WORKLOADS["rollout"], heads=2, frame_h=6, frame_w=5, background_rows=4)
    s = GpuLayerStream(w, 2, device="cpu", tagged=True)
    x1 = s.step(1)
    x2 = s.step(2)
    F, C = w.F, w.chunk_frames
    assert x1["candK"].shape == (2, (C - 1) * F, w.head_dim) and x1["candK"].dtype == torch.bfloat16
    assert x2["candK"].shape == (2, C * F, w.head_dim) and x2["winK"].shape == (2, C * F, w.head_dim)
    np.testing.assert_array_equal(x2["cand_ids"].numpy(), kvgen.token_ids(w, range(C, 2 * C)))
    # ids are carried by the values, window and candidates alike
    got = kvgen.untag_ids(x2["candV"].float().numpy())
    assert (got == x2["cand_ids"].numpy()[None, :]).all()
    np.testing.assert_array_equal(x1["winV"].float().numpy(), x2["candV"].float().numpy())
    # candidate k of step 2 = window k of step 1 (chunk 1), rotated with t = 0
    for k, t in enumerate(range(C, 2 * C)):
        win = _unrotate(x1["winK"][:, k * F:(k + 1) * F].float().numpy(), w, t)
        cand = _unrotate(x2["candK"][:, k * F:(k + 1) * F].float().numpy(), w, 0)
        np.testing.assert_allclose(cand, win, atol=0.06, rtol=0.02)   # two bf16 roundings apart
