"""Native softmax attention of the current chunk's queries (fp64).

DensityKV, Fig. 2 and §5: retained states are exact K/V pairs read by the
backbone's native attention together with the local window; Forcing-KV §3.3/§3.5:
Attention(Q, [K_sink, ..., K_cur], [V_sink, ..., V_cur]).

Reading: scaled dot-product attention with scale 1/sqrt(d), no mask (the current
chunk attends bidirectionally to itself, and to all history), fp64 softmax.
"""
from __future__ import annotations

import numpy as np


def attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float | None = None):
    """O = softmax(Q K^T * scale) V and the natural-log LSE per query row.

    Q [n_q][d], K [n_k][d], V [n_k][d_v]; returns (O [n_q][d_v], lse [n_q])."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(Q.shape[-1])
    S = (Q @ K.T) * scale
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    z = E.sum(axis=1, keepdims=True)
    O = (E @ V) / z
    lse = (m + np.log(z))[:, 0]
    return O, lse
