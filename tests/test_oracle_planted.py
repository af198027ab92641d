"""The pins reject plausible mistakes in the density, attention and Forcing-KV
oracles: a wrong variant is put in place of the real function and at least one
pin of that oracle must fail.  (The DensityKV admit step has its own planted
mistakes in test_oracle_densitykv.py.)"""
import math

import numpy as np
import pytest

import tests.test_oracle_attention as TA
import tests.test_oracle_density as TD
import tests.test_oracle_forcingkv as TF
from oracle import forcingkv as fkv
from oracle.density import sq_dists


def _pins(module):
    return [getattr(module, n) for n in sorted(dir(module)) if n.startswith("test_")]


def _caught(module, target, patches):
    """True if some pin of `module` fails while `patches` replace attributes of `target`."""
    saved = {k: getattr(target, k) for k in patches}
    try:
        for k, v in patches.items():
            setattr(target, k, v)
        for pin in _pins(module):
            try:
                pin()
            except AssertionError:   # (a variant that raises anything else is a broken variant: the test errors)
                return True
        return False
    finally:
        for k, v in saved.items():
            setattr(target, k, v)


# ------------------------------------------------------------------ density
def _density_variant(phi, exclude="id", dist=lambda A, B: sq_dists(A, B)):
    def density(rows, cols, *, h, eps, s, row_ids=None, col_ids=None, weights=None):
        rows = np.asarray(rows, np.float64).reshape(-1, np.shape(rows)[-1])
        cols = np.asarray(cols, np.float64).reshape(-1, np.shape(cols)[-1])
        if rows.shape[0] == 0:
            return np.zeros(0)
        if cols.shape[0] == 0:
            return np.zeros(rows.shape[0])
        P = phi(dist(rows, cols), h, eps, s)
        if weights is not None:
            P = P * np.asarray(weights, np.float64)[None, :]
        if row_ids is not None and col_ids is not None:
            if exclude == "id":
                P = np.where(np.asarray(row_ids)[:, None] == np.asarray(col_ids)[None, :], 0.0, P)
            elif exclude == "index":
                n = min(P.shape)
                P = P.copy()
                P[np.arange(n), np.arange(n)] = 0.0
        return P.sum(axis=1)
    return density


DENSITY_MISTAKES = {
    "exponent -s": _density_variant(lambda D, h, e, s: (D / h + e) ** (-s)),
    "h on the distance, not its square": _density_variant(lambda D, h, e, s: (np.sqrt(D) / h + e) ** (-s / 2)),
    "h squared": _density_variant(lambda D, h, e, s: (D / (h * h) + e) ** (-s / 2)),
    "eps outside the power": _density_variant(lambda D, h, e, s: np.where(D > 0, (D / h) ** (-s / 2), 0) + e),
    "self term kept": _density_variant(lambda D, h, e, s: (D / h + e) ** (-s / 2), exclude="none"),
    "self excluded by position": _density_variant(lambda D, h, e, s: (D / h + e) ** (-s / 2), exclude="index"),
    "squared distance via dropped cross term": _density_variant(
        lambda D, h, e, s: (D / h + e) ** (-s / 2),
        dist=lambda A, B: (A * A).sum(1)[:, None] + (B * B).sum(1)[None, :]),
}


def test_density_pins_pass_as_built():
    assert not _caught(TD, TD, {})


@pytest.mark.parametrize("name", sorted(DENSITY_MISTAKES))
def test_density_pins_catch(name):
    assert _caught(TD, TD, {"density": DENSITY_MISTAKES[name]}), name


# ------------------------------------------------------------------ attention
def _attention_variant(scale_of=lambda d: 1 / math.sqrt(d), over_queries=False, normalise=True, lse_shift=True):
    def attention(Q, K, V, scale=None):
        Q, K, V = (np.asarray(a, np.float64) for a in (Q, K, V))
        S = (Q @ K.T) * (scale_of(Q.shape[-1]) if scale is None else scale)
        ax = 0 if over_queries else 1
        m = S.max(axis=ax, keepdims=True)
        E = np.exp(S - m)
        z = E.sum(axis=ax, keepdims=True)
        O = (E / z if normalise else E) @ V
        lse = (m + np.log(z)) if lse_shift else np.log(z)
        lse = lse[:, 0] if ax == 1 else np.full(S.shape[0], float(lse.ravel()[0]))
        return O, lse
    return attention


ATTENTION_MISTAKES = {
    "scale 1/d": _attention_variant(scale_of=lambda d: 1 / d),
    "no scale": _attention_variant(scale_of=lambda d: 1.0),
    "softmax over queries": _attention_variant(over_queries=True),
    "weights not normalised": _attention_variant(normalise=False),
    "lse without the max": _attention_variant(lse_shift=False),
}


def test_attention_pins_pass_as_built():
    assert not _caught(TA, TA, {})


@pytest.mark.parametrize("name", sorted(ATTENTION_MISTAKES))
def test_attention_pins_catch(name):
    assert _caught(TA, TA, {"attention": ATTENTION_MISTAKES[name]}), name


# ------------------------------------------------------------------ Forcing-KV
def _bottom_k_ties_high(sim, k):
    order = np.lexsort((-np.arange(sim.shape[0]), sim))
    return np.sort(order[:k])


def _top_k(sim, k):
    order = np.lexsort((np.arange(sim.shape[0]), -sim))
    return np.sort(order[:k])


def _dot_not_cosine(A, B):
    return np.einsum("ij,ij->i", np.asarray(A, np.float64), np.asarray(B, np.float64))


def _segment_sum(Kt, Knext, segs):
    c = fkv.token_cosine(Kt, Knext)
    return np.array([c[s].sum() for s in segs])


_plain_prune = fkv.prune_hybrid


def _proxy_ignored(states, p, newK, newV, new_ids, nextK, sim_keys=None):
    return _plain_prune(states, p, newK, newV, new_ids, nextK)


def _proxy_keys_kept(states, p, newK, newV, new_ids, nextK, sim_keys=None):
    # the first layer's keys stored instead of this layer's own
    if sim_keys is None:
        return _plain_prune(states, p, newK, newV, new_ids, nextK)
    return _plain_prune(states, p, sim_keys[0], newV, new_ids, sim_keys[1])


FORCING_MISTAKES = {
    "first-block proxy ignored": {"prune_hybrid": _proxy_ignored},
    "first-block keys stored": {"prune_hybrid": _proxy_keys_kept},
    "ties to the higher index": {"bottom_k": _bottom_k_ties_high},
    "keeps the most similar": {"bottom_k": _top_k},
    "ceil(r n)": {"keep_count": lambda n, r: int(math.ceil(r * n - 1e-9))},
    "dot product for cosine": {"token_cosine": _dot_not_cosine},
    "segment sum for mean": {"segment_similarity": _segment_sum},
}


def test_forcing_pins_pass_as_built():
    assert not _caught(TF, fkv, {})


@pytest.mark.parametrize("name", sorted(FORCING_MISTAKES))
def test_forcing_pins_catch(name):
    assert _caught(TF, fkv, FORCING_MISTAKES[name]), name
