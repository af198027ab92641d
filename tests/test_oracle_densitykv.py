"""Pins of the oracle's DensityKV admit step (App. B.1 "Online Bank Update", App. E).

* hand-derived scenarios (tests/golden/densitykv_hand.json, exact fractions);
* invariants of the rule on seeded rollouts: |B| <= M, the same admitted count
  in every head, no survivor above the growth bound, new baselines equal their
  post-update density, old baselines frozen, K/V pairing by carried ids;
* tau = inf with M >= history: the bank is the whole non-sink history and the
  attention equals full chunk-causal attention over every generated token;
* the incremental algebra the CUDA path uses equals the from-scratch densities;
* the App. E ablation switches (refresh baselines, densest-only eviction,
  source-order completion, source candidate order) on hand scenarios G5-G11;
* planted mistakes (strict vs non-strict bounds, tie directions, the self term,
  refreshed baselines, each ablation switch ignored or misread) each break at
  least one pin.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import kvgen
from oracle import densitykv as dkv
from oracle.attention import attention
from oracle.density import density

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "densitykv_hand.json")


def _val(s):
    return float(Fraction(s)) if "/" in s or s.lstrip("-").isdigit() else float(s)


def _run_scenario(sc):
    prm = sc["params"]
    p = dkv.Params(capacity=prm["capacity"], tau=prm["tau"], eps=prm["eps"], s=prm["s"], h=prm["h"],
                   sync_heads=prm.get("sync_heads", True), cand_order=prm.get("cand_order", "score"),
                   baselines=prm.get("baselines", "fixed"), eviction=prm.get("eviction", "ratio"))
    H = prm["heads"]
    banks = [dkv.HeadBank.empty(1) for _ in range(H)]
    for st in sc["steps"]:
        ids = np.array(st["cand_ids"])
        K = np.array(st["candK"], dtype=np.float64)[:, :, None]
        V = np.repeat(ids[None, :, None].astype(np.float64), H, 0)
        r = dkv.admit(banks, ids, K, V, p)
        yield st, r
        banks = r.banks


def _check_step(st, r):
    e = st["expect"]
    H = len(r.banks)
    cand_ids = np.array(st["cand_ids"])
    if "P" in e:
        assert r.P == e["P"]
    if "P_h" in e:
        assert list(r.P_h) == e["P_h"]
    if "scores" in e:
        for hh in range(H):
            np.testing.assert_allclose(r.score[hh], [_val(x) for x in e["scores"][hh]], rtol=1e-12)
    if "admitted_ids" in e:
        for hh in range(H):
            assert sorted(cand_ids[r.admitted[hh]].tolist()) == sorted(e["admitted_ids"][hh])
    prev_ids = None
    for hh in range(H):
        b = r.banks[hh]
        if "bank_ids" in e:
            assert sorted(b.ids.tolist()) == sorted(e["bank_ids"][hh])
        # pairing: V carries the id
        np.testing.assert_array_equal(b.V[:, 0], b.ids.astype(np.float64))
        if "rho0" in e:
            got = dict(zip(b.ids.tolist(), b.rho0.tolist()))
            for k, v in e["rho0"][hh].items():
                assert got[int(k)] == pytest.approx(_val(v), rel=1e-12, abs=1e-300)
        if "rho" in e:
            got = dict(zip(b.ids.tolist(), r.rho_new[hh].tolist()))
            for k, v in e["rho"][hh].items():
                assert got[int(k)] == pytest.approx(_val(v), rel=1e-12)
        prev_ids = b.ids
    return prev_ids


@pytest.mark.parametrize("name", [s["name"] for s in json.load(open(GOLDEN))["scenarios"]])
def test_golden_hand_scenarios(name):
    sc = [s for s in json.load(open(GOLDEN))["scenarios"] if s["name"] == name][0]
    prev_banks = None
    for st, r in _run_scenario(sc):
        _check_step(st, r)
        e = st["expect"]
        # ratio / mandatory / evicted are per old-bank entry: map through the old ids
        if prev_banks is not None:
            for hh in range(len(r.banks)):
                old_ids = prev_banks[hh].ids.tolist()
                if "ratio" in e:
                    got = dict(zip(old_ids, r.ratio[hh].tolist()))
                    for k, v in e["ratio"][hh].items():
                        assert got[int(k)] == pytest.approx(_val(v), rel=1e-12, abs=1e-300)
                if "mandatory_ids" in e:
                    assert sorted(np.array(old_ids)[r.mandatory[hh]].tolist()) == sorted(e["mandatory_ids"][hh])
                if "evicted_ids" in e:
                    assert sorted(np.array(old_ids)[r.evicted[hh]].tolist()) == sorted(e["evicted_ids"][hh])
        prev_banks = r.banks


def test_golden_values_are_reproduced_by_their_exact_derivation():
    """tests/golden/derive_densitykv_hand.py re-derives every stored expected value
    of densitykv_hand.json in exact fractions, independently of the oracle."""
    import importlib.util
    path = os.path.join(os.path.dirname(__file__), "golden", "derive_densitykv_hand.py")
    spec = importlib.util.spec_from_file_location("derive_densitykv_hand", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert mod.mismatches(json.load(open(GOLDEN))) == []


def _tiny_rollout(steps=7, tagged=True, **kw):
    w = kvgen.WORKLOADS["tiny"]
    L = kvgen.LayerInputs(w, 0, tagged=tagged)
    p = dkv.Params(capacity=kw.get("capacity", w.capacity), tau=kw.get("tau", w.tau), eps=w.eps, s=w.s,
                   sync_heads=kw.get("sync_heads", True))
    return w, L, p, dkv.rollout(L, p, steps, attend=kw.get("attend", False))


@pytest.mark.parametrize("tau", [2.0, 1.0])
def test_rollout_invariants(tau):
    w, L, p, res = _tiny_rollout(tau=tau)
    prev = None
    for rec in res:
        r = rec["admit"]
        sizes = [b.size for b in r.banks]
        assert max(sizes) <= p.capacity
        assert len({len(a) for a in r.admitted}) == 1  # same P in every head
        for hh, b in enumerate(r.banks):
            # pairing of values with keys through the carried ids
            np.testing.assert_array_equal(kvgen.untag_ids(b.V), b.ids)
            # every mandatory entry is evicted; survivors were within the bound
            assert np.all(r.evicted[hh][r.mandatory[hh]])
            assert np.all(r.ratio[hh][~r.evicted[hh]] <= p.tau)
            # new baselines = post-update density; old baselines frozen
            n_new = len(r.admitted[hh])
            np.testing.assert_allclose(b.rho0[b.size - n_new:], r.rho_new[hh][b.size - n_new:], rtol=1e-14)
            if prev is not None:
                old = dict(zip(prev[hh].ids.tolist(), prev[hh].rho0.tolist()))
                for i, v in zip(b.ids[:b.size - n_new].tolist(), b.rho0[:b.size - n_new].tolist()):
                    assert old[i] == v
            # the largest feasible prefix: one more candidate would be infeasible somewhere
        P = len(r.admitted[0])
        N = len(rec["inputs"]["cand_ids"])
        if P < min(p.capacity, N):
            assert int(r.P_h.min()) == P
        prev = r.banks
    # tau = 2 exercises mandatory and capacity evictions; tau = 1 a binding admission prefix
    if tau == 2.0:
        assert any(int(rec["admit"].n_capacity.sum()) > 0 for rec in res)
        assert any(int(sum(m.sum() for m in rec["admit"].mandatory)) > 0 for rec in res)
    else:
        assert any(0 < len(rec["admit"].admitted[0]) < len(rec["inputs"]["cand_ids"]) for rec in res)


def _switch_rollout(tau, **switches):
    w = kvgen.WORKLOADS["tiny"]
    L = kvgen.LayerInputs(w, 0, tagged=True)
    p = dkv.Params(capacity=w.capacity, tau=tau, eps=w.eps, s=w.s, **switches)
    return p, dkv.rollout(L, p, 7, attend=False)


def _lead_run(score, ids, tau):
    """Brute force: walk the candidates by id until the first one above tau."""
    n = 0
    for k in np.argsort(ids, kind="stable"):
        if not score[k] <= tau:
            break
        n += 1
    return n


@pytest.mark.parametrize("tau,switches", [
    (2.0, dict(baselines="refresh")),
    (2.0, dict(eviction="densest")),
    (2.0, dict(eviction="source")),
    (1.0, dict(cand_order="source")),
    (1.0, dict(cand_order="source", sync_heads=False)),
])
def test_ablation_switch_invariants(tau, switches):
    """What each App. E switch implies, checked on the outputs of seeded tiny
    rollouts by direct computation (sorts and loops over the step's results)."""
    p, res = _switch_rollout(tau, **switches)
    exercised = False
    for rec in res:
        r = rec["admit"]
        ids_c = np.asarray(rec["inputs"]["cand_ids"])
        N = ids_c.size
        for hh, b in enumerate(r.banks):
            old_ids = (res[rec["step"] - 2]["admit"].banks[hh].ids if rec["step"] > 1 else np.zeros(0, np.int64))
            if switches.get("baselines") == "refresh":
                np.testing.assert_allclose(b.rho0, r.rho_new[hh], rtol=1e-14)
            if switches.get("eviction") == "densest":
                assert not r.mandatory[hh].any()
                ev = r.evicted[hh]
                assert ev.sum() == max(0, old_ids.size + len(r.admitted[hh]) - p.capacity)
                rhat = r.rho_cur[hh] + r.proj[hh]
                if ev.any() and (~ev).any():
                    assert rhat[ev].min() >= rhat[~ev].max()
                    exercised = True
            if switches.get("eviction") == "source":
                np.testing.assert_array_equal(r.mandatory[hh], r.ratio[hh] > p.tau)
                cap = r.evicted[hh] & ~r.mandatory[hh]
                kept = ~r.evicted[hh]
                if cap.any() and kept.any():
                    assert old_ids[cap].max() < old_ids[kept].min()
                    exercised = True
            if switches.get("cand_order") == "source":
                run = _lead_run(r.score[hh], ids_c, p.tau)
                assert int(r.P_h[hh]) == run
                adm = np.sort(ids_c[r.admitted[hh]])
                np.testing.assert_array_equal(adm, np.sort(ids_c)[:adm.size])
                assert np.all(r.score[hh][r.admitted[hh]] <= p.tau)
                if 0 < run < N:
                    exercised = True
        if switches.get("cand_order") == "source":
            P_expect = [min(int(r.P_h.min()), p.capacity, N)] * len(r.banks) if p.sync_heads else \
                [min(int(v), p.capacity, N) for v in r.P_h]
            assert [len(a) for a in r.admitted] == P_expect
    if switches.get("baselines") != "refresh":
        assert exercised, "the rollout never reached the case the switch changes"


def _run_blocks(blocks, p, perm=None, scale=1.0):
    """Admit a list of (ids, K, V) blocks from empty banks; returns the final banks.
    ``perm`` permutes every block's candidates; ``scale`` multiplies every key."""
    H, d = blocks[0][1].shape[0], blocks[0][1].shape[-1]
    banks = [dkv.HeadBank.empty(d) for _ in range(H)]
    for ids, K, V in blocks:
        o = perm(ids.size) if perm is not None else np.arange(ids.size)
        banks = dkv.admit(banks, ids[o], K[:, o] * scale, V[:, o], p).banks
    return banks


def _bank_map(banks):
    return [{int(i): (tuple(k), r0) for i, k, r0 in zip(b.ids, b.K.round(12), b.rho0.round(12))} for b in banks]


def _random_blocks(seed, H=2, d=4, n=12, steps=4):
    rng = np.random.default_rng(seed)
    out = []
    for t in range(steps):
        ids = np.arange(100 * t, 100 * t + n)
        K = rng.standard_normal((H, n, d))
        V = np.broadcast_to(ids[None, :, None].astype(np.float64), (H, n, d)).copy()
        out.append((ids, K, V))
    return out


@pytest.mark.parametrize("tau", [2.0, 1.2])   # 2.0: mandatory and capacity evictions; 1.2: P < N
@pytest.mark.parametrize("switches", [dict(), dict(eviction="densest"), dict(eviction="source"),
                                      dict(cand_order="source"), dict(baselines="refresh")])
def test_admit_ignores_candidate_array_order(switches, tau):
    """Decisions depend on (score, id), never on where a candidate sits in the
    block: any permutation of every block leaves the same banks."""
    p = dkv.Params(capacity=20, tau=tau, eps=0.5, s=2.0, **switches)
    blocks = _random_blocks(1)
    ref = _bank_map(_run_blocks(blocks, p))
    for k in range(3):
        rng = np.random.default_rng(10 + k)
        got = _bank_map(_run_blocks(blocks, p, perm=lambda n: rng.permutation(n)))
        assert [set(g) for g in got] == [set(r) for r in ref]
        for g, r in zip(got, ref):
            for i in r:
                assert g[i][0] == r[i][0]
                assert g[i][1] == pytest.approx(r[i][1], rel=1e-12)


def test_distance_scale_enters_only_through_the_scaled_distance():
    """phi depends on ||a - b||^2 / h: scaling every key by c and h by c^2 leaves
    every density, score and decision unchanged (a check that h is applied to
    the squared distance, in every pass)."""
    blocks = _random_blocks(2)
    c = 3.0
    base = dkv.Params(capacity=20, tau=2.0, eps=0.5, s=2.0, h=4.0)
    scaled = dkv.Params(capacity=20, tau=2.0, eps=0.5, s=2.0, h=4.0 * c * c)
    a, b = _run_blocks(blocks, base), _run_blocks(blocks, scaled, scale=c)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(np.sort(x.ids), np.sort(y.ids))
        ox, oy = np.argsort(x.ids), np.argsort(y.ids)
        np.testing.assert_allclose(x.rho0[ox], y.rho0[oy], rtol=1e-12)
        np.testing.assert_allclose(x.K[ox] * c, y.K[oy], rtol=1e-15)


def test_independent_heads_equal_one_head_banks():
    """With sync_heads=False a head's bank is exactly what a one-head layer with
    that head's inputs produces: no information crosses heads."""
    blocks = _random_blocks(3, H=3)
    p = dkv.Params(capacity=20, tau=1.2, eps=0.5, s=2.0, sync_heads=False)
    together = _run_blocks(blocks, p)
    for hh in range(3):
        alone = _run_blocks([(ids, K[hh:hh + 1], V[hh:hh + 1]) for ids, K, V in blocks], p)[0]
        np.testing.assert_array_equal(together[hh].ids, alone.ids)
        np.testing.assert_array_equal(together[hh].rho0, alone.rho0)


@pytest.mark.parametrize("tau", [2.0, 1.2])
def test_head_split_with_min_exchange_equals_the_whole_layer(tau):
    """Head-parallel admission: each group of heads computes its own prefix
    min(min_h P_h, M, N), the groups exchange the MIN, and each admits under that
    bound.  The banks equal those of one admit over every head, step after step."""
    blocks = _random_blocks(4, H=4)
    p = dkv.Params(capacity=20, tau=tau, eps=0.5, s=2.0)
    groups = [(0, 1), (1, 4)]
    whole = [dkv.HeadBank.empty(4) for _ in range(4)]
    split = [dkv.HeadBank.empty(4) for _ in range(4)]
    bound_used = False
    for ids, K, V in blocks:
        r = dkv.admit(whole, ids, K, V, p)
        own = [min(int(dkv.admit(split[a:b], ids, K[a:b], V[a:b], p).P_h.min()), p.capacity, ids.size)
               for a, b in groups]
        m = min(own)
        bound_used |= max(own) > m
        new = []
        for a, b in groups:
            new += dkv.admit(split[a:b], ids, K[a:b], V[a:b], p, prefix_bound=m).banks
        for x, y in zip(r.banks, new):
            np.testing.assert_array_equal(x.ids, y.ids)
            np.testing.assert_array_equal(x.rho0, y.rho0)
        whole, split = r.banks, new
    assert bound_used or tau == 2.0     # tau 1.2 makes the groups' prefixes differ


def test_incremental_update_equals_from_scratch():
    """The CUDA path keeps densities incrementally (App. B.1, O(N M d_k) exact update):
    survivors rho + sum_A phi - sum_E phi; new c: rho_B(c) - sum_E phi + sum_{A, c' != c} phi."""
    w, L, p, res = _tiny_rollout(steps=6)
    kw = dict(h=float(w.head_dim), eps=p.eps, s=p.s)
    banks = [dkv.HeadBank.empty(w.head_dim) for _ in range(w.heads)]
    for rec in res:
        r, x = rec["admit"], rec["inputs"]
        for hh in range(w.heads):
            b = banks[hh]
            A = r.admitted[hh]
            ev = r.evicted[hh]
            cK, cid = x["candK"][hh][A].astype(np.float64), x["cand_ids"][A]
            surv = ~ev
            inc_old = (r.rho_cur[hh] + r.proj[hh]
                       - density(b.K, b.K[ev], row_ids=b.ids, col_ids=b.ids[ev], **kw))[surv]
            inc_new = (r.rho_cand[hh][A] - density(cK, b.K[ev], **kw)
                       + density(cK, cK, row_ids=cid, col_ids=cid, **kw))
            np.testing.assert_allclose(np.concatenate([inc_old, inc_new]), r.rho_new[hh], rtol=1e-11)
        banks = r.banks


def test_tau_inf_keeps_full_history_and_full_attention():
    w = kvgen.WORKLOADS["tiny"]
    steps = 5
    L = kvgen.LayerInputs(w, 0)
    p = dkv.Params(capacity=10 ** 6, tau=float("inf"), eps=w.eps, s=w.s)
    res = dkv.rollout(L, p, steps, attend=True)
    for rec in res:
        i = rec["step"]
        hist = kvgen.token_ids(w, range(1, i * w.chunk_frames))
        for hh in range(w.heads):
            assert sorted(rec["admit"].banks[hh].ids.tolist()) == hist.tolist()
        # full chunk-causal attention: every generated token up to chunk i
        x = rec["inputs"]
        for hh in range(w.heads):
            frames = list(range(0, (i + 1) * w.chunk_frames))
            # keys in the cache form: memory keys (frame index 0 in RoPE) for history,
            # true index for the sink and the current chunk
            hist_frames = list(range(1, i * w.chunk_frames))
            Kh = L.keys(hist_frames, memory=True)[hh]
            Vh = L.values(hist_frames)[hh]
            K = np.concatenate([x["sinkK"][hh], Kh, x["winK"][hh]])
            V = np.concatenate([x["sinkV"][hh], Vh, x["winV"][hh]])
            assert K.shape[0] == len(frames) * w.F
            O_ref, lse_ref = attention(x["Q"][hh], K, V)
            O, lse = rec["attn"][hh]
            np.testing.assert_allclose(O, O_ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse, lse_ref, rtol=1e-12)


def test_independent_heads_flag():
    w, L, p, res = _tiny_rollout(steps=4, sync_heads=False)
    for rec in res:
        r = rec["admit"]
        N = len(rec["inputs"]["cand_ids"])
        for hh in range(w.heads):
            assert len(r.admitted[hh]) == min(int(r.P_h[hh]), p.capacity, N)


def test_tiny_rollout_has_no_near_ties():
    w, L, p, res = _tiny_rollout(steps=7, tagged=False)
    assert sum(rec["admit"].near_ties for rec in res) == 0


# ------------------------------------------------------------------ planted mistakes
def _golden_passes():
    try:
        for sc in json.load(open(GOLDEN))["scenarios"]:
            test_golden_hand_scenarios(sc["name"])
        return True
    except AssertionError:
        return False


class _NonStrict(dkv.Params):
    """Params whose tau is nudged down by one ulp: 'ratio > tau' acts like '>='."""

    def __init__(self, *a, **k):
        super().__init__(*a, **k)
        self.tau = float(np.nextafter(self.tau, -np.inf))


class _NoRefresh(dkv.Params):
    """Params that ignore the refresh-baselines switch."""

    def __init__(self, *a, **k):
        super().__init__(*a, **k)
        self.baselines = "fixed"


def _refresh_admit(real_admit):
    def admit(banks, *a, **k):
        r = real_admit(banks, *a, **k)
        for b, rn in zip(r.banks, r.rho_new):   # baselines recomputed after every update
            b.rho0 = rn.copy()
        return r
    return admit


def test_pins_catch_planted_mistakes():
    assert _golden_passes()
    real_density = dkv.density
    mutations = {
        "tie_newer_first": ("_lex_order", lambda prim, ids: np.lexsort((-np.asarray(ids), np.asarray(prim)))),
        "self_included": ("density", lambda r, c, **k: real_density(
            r, c, **{kk: v for kk, v in k.items() if kk not in ("row_ids", "col_ids")})),
        "non_strict_evict": ("Params", _NonStrict),
        "refresh_baselines": ("admit", _refresh_admit(dkv.admit)),
        "capacity_lowest_ratio": ("_lex_order", lambda prim, ids: np.lexsort((np.asarray(ids), -np.asarray(prim)))),
        "refresh_ignored": ("Params", _NoRefresh),
        "source_order_by_score": ("_cand_key", lambda p, score: score),
        "source_prefix_counts_all_feasible": ("_feasible_prefix", lambda p, f, ids: int(f.sum())),
        "eviction_switch_ignored": ("_cut_value", lambda p, ratio, rhat, ids: ratio),
        "densest_keeps_threshold": ("_mandatory", lambda p, ratio: ratio > p.tau),
    }
    for name, (attr, repl) in mutations.items():
        real = getattr(dkv, attr)
        setattr(dkv, attr, repl)
        try:
            assert not _golden_passes(), f"planted mistake '{name}' was not caught"
        finally:
            setattr(dkv, attr, real)
    assert _golden_passes()
