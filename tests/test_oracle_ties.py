"""Pins of the oracle's near-tie logic (DensityKV §3 and App. E: the admission
threshold, the synchronised-prefix cut, the eviction threshold and the capacity
cut), which decides what the GPU parity tests may let differ.

Hand-built one-head and two-head steps on 1-D keys (h = 1, eps = 1, s = 2, so
phi(a, b) = 1 / (1 + (a - b)^2) in closed form) put one deciding value at a chosen
relative distance from its threshold or its cut: 5e-5 (a near tie under the 1e-4
margin) or 5e-3 (not one).  The baselines rho0 of a hand-built bank are free
inputs, so a score or a ratio is placed by choosing them:
    score(c) = rho_B(c) / mean rho0,   ratio(i) = (rho_i + sum_A phi(c, i)) / rho0_i.

Pinned:
* ``_tie_ids`` flags exactly the ids of the decisions within the margin, and
  ``_margins`` / ``near_ties`` count them;
* a replay (``admit(..., forced=...)``) accepts the other outcome of a near-tie
  decision, including a synchronised P that moves with a near-tie feasibility in
  the head that sets it, and rejects the other outcome of a decision that is not a
  near tie; the oracle's own decisions always replay;
* planted mistakes in both (an absolute margin, the cut neighbourhood flagged
  whatever the gap, one side of a cut only, eviction ties ignored, no margin in the
  replay's order check, the P range or the capacity order unchecked, the id rule
  for equal values dropped) each fail one of these pins.
"""
import functools
import inspect
import math

import numpy as np
import pytest

import kvgen
from oracle import densitykv as dkv

TAU = 4.0
NEAR, FAR = 5e-5, 5e-3


def phi(a, b):
    return 1.0 / (1.0 + (a - b) ** 2)


def params(M=10, **kw):
    return dkv.Params(capacity=M, tau=TAU, eps=1.0, s=2.0, h=1.0, **kw)


def bank(ids, pos, rho0):
    pos = np.asarray(pos, np.float64)[:, None]
    ids = np.asarray(ids, np.int64)
    return dkv.HeadBank(ids, pos, ids[:, None].astype(np.float64), np.asarray(rho0, np.float64))


def at_score(t, r0, sign=1.0):
    """Position of a candidate whose score against a one-entry bank at 0 with
    baseline r0 is t: 1 / ((1 + x^2) r0) = t."""
    return sign * math.sqrt(1.0 / (t * r0) - 1.0)


def step(banks, ids, pos, p, forced=None):
    """pos: [H][N] candidate positions."""
    K = np.asarray(pos, np.float64)[:, :, None]
    V = np.repeat(np.asarray(ids, np.float64)[None, :, None], len(banks), 0)
    return dkv.admit(banks, np.asarray(ids, np.int64), K, V, p, forced=forced)


# ------------------------------------------------------------------ scenarios
def threshold_scenario():
    """One head, one bank entry (id 1 at 0, rho0 0.05); candidates 10..14 with
    scores tau(1+NEAR), tau(1-NEAR), tau(1+FAR), tau(1-FAR), tau/2."""
    r0 = 0.05
    targets = [TAU * (1 + NEAR), TAU * (1 - NEAR), TAU * (1 + FAR), TAU * (1 - FAR), TAU / 2]
    pos = [at_score(t, r0, (-1) ** k) for k, t in enumerate(targets)]
    return [bank([1], [0.0], [r0])], [10, 11, 12, 13, 14], [pos], targets


def eviction_scenario():
    """One head, entries 1..5 at 0..4, one far candidate (id 50 at 10, clearly
    feasible); rho0 set so that the projected ratios are tau(1+NEAR), tau(1-NEAR),
    tau(1+FAR), tau(1-FAR), tau/2; M = 10 (no capacity eviction)."""
    pos = np.arange(5, dtype=np.float64)
    c = 10.0
    rho = np.array([sum(phi(a, b) for b in pos if b != a) for a in pos])
    proj = np.array([phi(a, c) for a in pos])
    targets = np.array([TAU * (1 + NEAR), TAU * (1 - NEAR), TAU * (1 + FAR), TAU * (1 - FAR), TAU / 2])
    b = bank([1, 2, 3, 4, 5], pos, (rho + proj) / targets)
    return [b], [50], [[c]], targets


def cut_scenario(gap):
    """Two synchronised heads.  Head 0 (entry at 0, rho0 0.05): candidates 10, 11,
    12 at scores tau/4, 2 tau, 3 tau, so P = 1.  Head 1 (entry at 0, rho0 0.02):
    scores s, s(1+gap), s(1+gap+9e-5) with s = tau/8, all feasible; head 1 admits
    id 10 and the cut to id 11 is a relative gap of `gap`.  Id 12 is within the
    margin of the first rejected score but not of the last admitted one."""
    s = TAU / 8
    h0 = [at_score(t, 0.05) for t in (TAU / 4, 2 * TAU, 3 * TAU)]
    h1 = [at_score(t, 0.02, (-1) ** k) for k, t in enumerate((s, s * (1 + gap), s * (1 + gap + 9e-5)))]
    return [bank([1], [0.0], [0.05]), bank([1], [0.0], [0.02])], [10, 11, 12], [h0, h1]


def pflip_scenario(delta):
    """Two synchronised heads.  Head 0 sets P: candidates 10, 11, 12 at scores
    tau/4, tau(1+delta), 3 tau (P_0 = 1); head 1: all three clearly feasible."""
    h0 = [at_score(t, 0.05) for t in (TAU / 4, TAU * (1 + delta), 3 * TAU)]
    h1 = [at_score(t, 0.02, (-1) ** k) for k, t in enumerate((TAU / 8, TAU / 6, TAU / 5))]
    return [bank([1], [0.0], [0.05]), bank([1], [0.0], [0.02])], [10, 11, 12], [h0, h1]


def capacity_scenario(gap):
    """One head, M = 3, entries 1, 2, 3 at 0, 10, 25 and one admitted candidate
    (id 50 at 40): one capacity eviction.  rho0 makes the ratios tau/2,
    tau/2 (1-gap), tau/4, so entry 1 goes and the cut to entry 2 is a relative gap
    of `gap`.  Returns the projected densities too (densest-only cuts by them:
    0.0121, 0.0154, 0.0104, entry 2 first)."""
    pos = np.array([0.0, 10.0, 25.0])
    c = 40.0
    rho = np.array([sum(phi(a, b) for b in pos if b != a) for a in pos])
    rhat = rho + np.array([phi(a, c) for a in pos])
    targets = np.array([TAU / 2, TAU / 2 * (1 - gap), TAU / 4])
    return [bank([1, 2, 3], pos, rhat / targets)], [50], [[c]], rhat


# ------------------------------------------------------------------ _tie_ids / _margins
def test_threshold_ties_flag_exactly_the_near_scores():
    banks, ids, pos, targets = threshold_scenario()
    r = step(banks, ids, pos, params())
    np.testing.assert_allclose(r.score[0], targets, rtol=1e-12)
    assert int(r.P_h[0]) == 3
    assert r.tie_cand_ids[0] == {10, 11}
    assert r.tie_bank_ids[0] == set()
    np.testing.assert_allclose(np.sort(r.margins["adm_thr"]), [NEAR, NEAR, FAR, FAR, 0.5], rtol=1e-6)
    assert r.near_ties == 2


def test_eviction_threshold_ties_flag_exactly_the_near_ratios():
    banks, ids, pos, targets = eviction_scenario()
    r = step(banks, ids, pos, params())
    assert len(r.admitted[0]) == 1
    np.testing.assert_allclose(r.ratio[0], targets, rtol=1e-12)
    assert r.tie_bank_ids[0] == {1, 2}
    assert r.tie_cand_ids[0] == set()
    assert sorted(banks[0].ids[r.mandatory[0]].tolist()) == [1, 3]
    np.testing.assert_allclose(np.sort(r.margins["ev_thr"]), [NEAR, NEAR, FAR, FAR, 0.5], rtol=1e-6)
    assert r.near_ties == 2


@pytest.mark.parametrize("gap,flagged", [(NEAR, {10, 11, 12}), (FAR, set())])
def test_admission_cut_ties(gap, flagged):
    banks, ids, pos = cut_scenario(gap)
    r = step(banks, ids, pos, params())
    assert r.P == 1 and list(r.P_h) == [1, 3]
    assert ids[r.admitted[1][0]] == 10
    assert r.tie_cand_ids[1] == flagged
    assert r.tie_cand_ids[0] == set()
    assert r.near_ties == (1 if flagged else 0)


@pytest.mark.parametrize("gap,flagged", [(NEAR, {1, 2}), (FAR, set())])
def test_capacity_cut_ties(gap, flagged):
    banks, ids, pos, _ = capacity_scenario(gap)
    r = step(banks, ids, pos, params(M=3))
    assert len(r.admitted[0]) == 1 and int(r.n_capacity[0]) == 1
    assert banks[0].ids[r.evicted[0]].tolist() == [1]
    assert r.tie_bank_ids[0] == flagged
    assert r.near_ties == (1 if flagged else 0)


# ------------------------------------------------------------------ forced replays
def _ok(banks, ids, pos, p, A, E):
    try:
        return step(banks, ids, pos, p, forced=(A, E))
    except ValueError as e:
        raise AssertionError(f"replay rejected: {e}") from e


def _rejected(banks, ids, pos, p, A, E):
    with pytest.raises(ValueError):
        step(banks, ids, pos, p, forced=(A, E))


def test_replay_of_the_oracles_own_decisions():
    banks, ids, pos, _ = threshold_scenario()
    r = step(banks, ids, pos, params())
    A = [[ids[k] for k in r.admitted[0]]]
    E = [banks[0].ids[r.evicted[0]].tolist()]
    r2 = _ok(banks, ids, pos, params(), A, E)
    assert set(r2.banks[0].ids.tolist()) == set(r.banks[0].ids.tolist())
    np.testing.assert_allclose(np.sort(r2.rho_new[0]), np.sort(r.rho_new[0]), rtol=1e-14)


def test_replay_admission_threshold():
    banks, ids, pos, _ = threshold_scenario()
    p = params()
    # the oracle admits 11, 13, 14; the entry (ratio ~ 10) is mandatory either way
    _ok(banks, ids, pos, p, [[10, 11, 13, 14]], [[1]])        # 10 is infeasible by 5e-5: a near tie
    _ok(banks, ids, pos, p, [[13, 14]], [[1]])                # 11 feasible by 5e-5: a near tie
    _rejected(banks, ids, pos, p, [[11, 12, 13, 14]], [[1]])  # 12 infeasible by 5e-3
    _rejected(banks, ids, pos, p, [[11, 14]], [[1]])          # 13 feasible by 5e-3


def test_replay_synchronised_p_moves_with_a_near_tie_in_the_head_that_sets_it():
    p = params()
    banks, ids, pos = pflip_scenario(NEAR)
    r = step(banks, ids, pos, p)
    assert r.P == 1
    # P = 2 in every head; head 0's entry then projects to ratio 5 > tau (mandatory)
    _ok(banks, ids, pos, p, [[10, 11], [10, 11]], [[1], []])
    _rejected(banks, ids, pos, p, [[10, 11], [10]], [[1], []])   # P must stay shared
    _rejected(banks, ids, pos, p, [[], []], [[], []])             # id 10 is clearly feasible everywhere
    banks, ids, pos = pflip_scenario(FAR)
    _rejected(banks, ids, pos, p, [[10, 11], [10, 11]], [[1], []])


def test_replay_admission_cut():
    p = params()
    for gap, ok in ((NEAR, True), (FAR, False)):
        banks, ids, pos = cut_scenario(gap)
        r = step(banks, ids, pos, p)
        E = [banks[h].ids[r.evicted[h]].tolist() for h in range(2)]
        (_ok if ok else _rejected)(banks, ids, pos, p, [[10], [11]], E)


def test_replay_eviction_threshold():
    banks, ids, pos, _ = eviction_scenario()
    p = params()
    _ok(banks, ids, pos, p, [[50]], [[1, 3]])          # as the oracle
    _ok(banks, ids, pos, p, [[50]], [[3]])             # 1 kept: above tau by 5e-5
    _ok(banks, ids, pos, p, [[50]], [[1, 2, 3]])       # 2 evicted: below tau by 5e-5
    _rejected(banks, ids, pos, p, [[50]], [[1]])       # 3 kept: above tau by 5e-3
    _rejected(banks, ids, pos, p, [[50]], [[1, 3, 4]])  # 4 evicted: below tau by 5e-3


def test_replay_capacity_cut():
    p = params(M=3)
    for gap, ok in ((NEAR, True), (FAR, False)):
        banks, ids, pos, _ = capacity_scenario(gap)
        (_ok if ok else _rejected)(banks, ids, pos, p, [[50]], [[2]])
        _rejected(banks, ids, pos, p, [[50]], [[3]])          # the lowest ratio
        _rejected(banks, ids, pos, p, [[50]], [[]])           # the bank would exceed M
        _rejected(banks, ids, pos, p, [[50]], [[1, 2]])       # one eviction makes room


def test_replay_equal_values_follow_the_id_rule():
    # empty banks: every score is exactly 0, the P = M lowest ids are admitted
    p = params(M=2)
    banks = [dkv.HeadBank.empty(1)]
    ids, pos = [10, 11, 12], [[0.0, 5.0, 9.0]]
    _ok(banks, ids, pos, p, [[10, 11]], [[]])
    _rejected(banks, ids, pos, p, [[10, 12]], [[]])


def test_replay_source_order_and_densest():
    banks, ids, pos = cut_scenario(NEAR)
    p = params(cand_order="source")
    r = step(banks, ids, pos, p)
    E = [banks[h].ids[r.evicted[h]].tolist() for h in range(2)]
    _ok(banks, ids, pos, p, [[ids[k] for k in r.admitted[h]] for h in range(2)], E)
    _rejected(banks, ids, pos, p, [[11], [11]], E)     # not the lowest id
    pd = params(M=3, eviction="densest")
    for gap in (NEAR, FAR):
        banks, ids, pos, rhat = capacity_scenario(gap)
        r = step(banks, ids, pos, pd)
        first = banks[0].ids[np.argmax(rhat)]
        assert banks[0].ids[r.evicted[0]].tolist() == [first]
        _rejected(banks, ids, pos, pd, [[50]], [[banks[0].ids[np.argmin(rhat)]]])


@pytest.mark.parametrize("kw", [dict(), dict(tau=1.0), dict(tau=1.0, sync_heads=False),
                                dict(eviction="densest"), dict(eviction="source"), dict(baselines="refresh"),
                                dict(tau=1.2, cand_order="source")])
def test_replay_accepts_every_decision_of_a_seeded_rollout(kw):
    """Seeded tiny rollout (the fp32 workload at its default seed): every step's
    own decisions replay, and the replay reproduces the step."""
    w = kvgen.WORKLOADS["tiny"]
    L = kvgen.LayerInputs(w, 0, tagged=True, seed_offset=0)
    kw = dict(kw)
    p = dkv.Params(capacity=w.capacity, tau=kw.pop("tau", w.tau), eps=w.eps, s=w.s, **kw)
    banks = [dkv.HeadBank.empty(w.head_dim) for _ in range(w.heads)]
    for i in range(1, 6):
        x = L.step(i)
        r = dkv.admit(banks, x["cand_ids"], x["candK"], x["candV"], p)
        A = [x["cand_ids"][a] for a in r.admitted]
        E = [banks[h].ids[r.evicted[h]] for h in range(w.heads)]
        r2 = dkv.admit(banks, x["cand_ids"], x["candK"], x["candV"], p, forced=(A, E))
        for h in range(w.heads):
            assert set(r2.banks[h].ids.tolist()) == set(r.banks[h].ids.tolist())
        banks = r.banks


# ------------------------------------------------------------------ planted mistakes
def _variant(fn, old, new):
    src = inspect.getsource(fn)
    assert old in src, (fn.__name__, old)
    ns = dict(vars(dkv))
    exec(compile(src.replace(old, new), dkv.__file__, "exec"), ns)
    return ns[fn.__name__]


def _pins():
    """Every pin of this file as a zero-argument call (parametrised pins once per
    parameter set), except the slow seeded-rollout one and the planted-mistake
    tests themselves."""
    out = []
    for k, v in sorted(globals().items()):
        if not k.startswith("test_") or k in PLANTED_TESTS or k == "test_replay_accepts_every_decision_of_a_seeded_rollout":
            continue
        marks = [m for m in getattr(v, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            out.append(v)
            continue
        names, values = marks[0].args[:2]
        names = [n.strip() for n in names.split(",")]
        for vals in values:
            vals = vals if len(names) > 1 else (vals,)
            out.append(functools.partial(v, **dict(zip(names, vals))))
    return out


def _caught(patches):
    saved = {k: getattr(dkv, k) for k in patches}
    try:
        for k, v in patches.items():
            setattr(dkv, k, v)
        for pin in _pins():
            try:
                pin()
            except AssertionError:
                return True
            except pytest.fail.Exception:
                return True
        return False
    finally:
        for k, v in saved.items():
            setattr(dkv, k, v)


MISTAKES = {
    "absolute threshold margin": lambda: {"_tie_ids": _variant(
        dkv._tie_ids, "set(cand_ids[_rel(score[hh], p.tau) < m]", "set(cand_ids[np.abs(score[hh] - p.tau) < m]")},
    "cut flagged whatever the gap": lambda: {"_tie_ids": _variant(
        dkv._tie_ids, "            if _rel(hi, lo) < m:\n                c |=", "            if True:\n                c |=")},
    "only the admitted side of the cut": lambda: {"_tie_ids": _variant(
        dkv._tie_ids, "c |= set(cand_ids[close | (np.abs(score[hh] - hi) <= m * max(abs(hi), 1e-300))]",
        "c |= set(cand_ids[close]")},
    "eviction threshold ties ignored": lambda: {"_tie_ids": _variant(
        dkv._tie_ids, "b |= set(ids[near].tolist())", "pass")},
    "absolute margins counted": lambda: {"_margins": _variant(
        dkv._margins, 'out["adm_thr"].append(_rel(score[hh], p.tau))',
        'out["adm_thr"].append(np.abs(score[hh] - p.tau))')},
    "no margin in the replay's order checks": lambda: {"_clearly_below": lambda a, b, m: np.asarray(a) < np.asarray(b)},
    "shared P unchecked": lambda: {"_forced_violations": _variant(
        dkv._forced_violations, "elif not lo <= P_all[0] <= hi:", "elif False:")},
    "capacity order unchecked": lambda: {"_order_violations": lambda *a, **k: 0},
    "equal values not decided by id": lambda: {"_forced_violations": _variant(
        dkv._forced_violations, "((SR == SA) & (iR < iA))", "((SR == SA) & False)")},
    "survivor above tau unchecked": lambda: {"_forced_violations": _variant(
        dkv._forced_violations, "if (clear_mand & surv).any():", "if False:")},
}
PLANTED_TESTS = {"test_tie_pins_pass_as_built", "test_tie_pins_catch"}


def test_tie_pins_pass_as_built():
    assert not _caught({})


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_tie_pins_catch(name):
    assert _caught(MISTAKES[name]()), name
