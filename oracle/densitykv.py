"""DensityKV online bank update, one (layer) admit step at a time, fp64.

Follows DensityKV App. B.1 "Online Bank Update", §3 "Online Density-Constrained
Bank Update" and App. E (default policy), in the pages' order:

1. every head keeps its own bank of exact (id, key, value) entries, at most M
   (App. B.1; App. D: independent layer-head banks, M = 9,360);
2. the finalised block's tokens are candidates; each is scored by its density
   against the head's bank, normalised by the mean of the bank's frozen
   insertion baselines (the mean-normalised disturbance order of App. E, smaller
   first);
3. the admitted count P is the largest prefix feasible for every head of the
   layer (synchronised admission, App. E cross-head synchronisation); each head
   admits its own P lowest-scoring candidates;
4. bank entries whose projected density ratio crosses tau are evicted first
   (threshold-first eviction, App. E); capacity eviction then removes the
   highest-ratio entries until the bank fits M (§3: the states that must go,
   then the densest, until there is room);
5. co-admitted candidates set their insertion baselines together, after the
   update (App. B.1: mutual interactions among the admitted block do not reject
   one another; only growth from later blocks counts); baselines of older entries
   stay frozen (App. E: fixed insertion-time references).

Readings taken where the pages are silent (each is a parameter or a plain choice):

* density: ``oracle.density`` (phi = (||a-b||^2/h + eps)^(-s/2), self excluded by id);
* disturbance score of candidate c in head h: rho_B(c) / mean_{i in B} rho0_i;
  candidate feasible iff score <= tau; if the bank is empty or its mean baseline
  is 0, every candidate is feasible with score 0;
* the prefix is ordered by (score ascending, id ascending);
* P = min(min_h P_h, M, N) with P_h the number of feasible candidates of head h
  (``sync_heads=False``: each head uses its own min(P_h, M, N));
* projected ratio of entry i: (rho_i + sum_{c in A_h} phi(c, i)) / rho0_i, with
  rho_i its density within the current bank; ratio 0 when rho0_i = 0;
  mandatory iff ratio > tau;
* capacity evictions E_cap = max(0, |B| - |mandatory| + P - M) among the
  non-mandatory entries, by (ratio descending, id ascending: older first);
* after the update every density is recomputed from scratch over the new bank;
  new entries take rho0 = that density.

Ablation switches of App. E (off by default; each replaces one default above):

* ``cand_order="source"``: candidates in spatiotemporal source order (id
  ascending) instead of by score; a head's feasible prefix is the run of
  candidates from the lowest id up to, not including, its lowest-id infeasible
  one, and a head admits its P lowest ids;
* ``baselines="refresh"``: after every update every entry's rho0 becomes its
  density within the new bank (App. E "refresh baselines"), not only the new
  entries';
* ``eviction="densest"``: no ratio threshold; the bank sheds
  max(0, |B| + P - M) entries by (projected density rho_i + sum_A phi descending,
  id ascending) -- the reading of App. E "densest-only eviction";
* ``eviction="source"``: mandatory evictions as by default, then the capacity
  evictions by id ascending (oldest first) -- App. E "source-order completion".

Nothing here is incremental: the CUDA path's incremental maintenance (the exact
O(N M d_k) update of App. B.1) is checked against these from-scratch values.

Near ties.  A decision is a near tie when the value that decides it lies within a
relative margin ``tie_margin`` (1e-4) of its threshold or of the value across its
cut (``_margins``, ``_tie_ids``).  Another implementation that rounds differently
may legitimately take such a decision the other way.  ``admit(..., forced=...)``
replays a step with such an outcome: it takes every head's admitted and evicted id
sets as given, but first checks that they are an outcome of the rule under a
relative perturbation below the margin of every value that decides them
(``_forced_violations``), and raises ``ValueError`` otherwise.  The densities,
baselines and bank contents of the replay then follow from those sets exactly as
in an ordinary step.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

from .density import density


@dataclasses.dataclass
class Params:
    capacity: int
    tau: float = 2.0
    eps: float = 1e-3
    s: float = 2.0
    h: float = 0.0           # distance scale; 0 => head_dim
    sync_heads: bool = True
    cand_order: str = "score"    # "score" | "source"
    baselines: str = "fixed"     # "fixed" | "refresh"
    eviction: str = "ratio"      # "ratio" | "densest" | "source"

    def scale(self, d: int) -> float:
        return float(self.h) if self.h > 0 else float(d)


@dataclasses.dataclass
class HeadBank:
    ids: np.ndarray          # int64 [n]
    K: np.ndarray            # float64 [n][d]
    V: np.ndarray            # float64 [n][d]
    rho0: np.ndarray         # float64 [n] frozen insertion baselines

    @staticmethod
    def empty(d: int) -> "HeadBank":
        return HeadBank(np.zeros(0, np.int64), np.zeros((0, d)), np.zeros((0, d)), np.zeros(0))

    @property
    def size(self) -> int:
        return int(self.ids.shape[0])


@dataclasses.dataclass
class AdmitResult:
    banks: List[HeadBank]
    P: int
    P_h: np.ndarray                  # feasible count per head
    rho_cand: List[np.ndarray]       # rho_B(c) per head, [N]
    score: List[np.ndarray]          # disturbance score per head, [N]
    admitted: List[np.ndarray]       # candidate indices admitted per head (selection order)
    rho_cur: List[np.ndarray]        # density of old entries within the old bank
    proj: List[np.ndarray]           # sum over admitted of phi(c, i), per old entry
    ratio: List[np.ndarray]          # projected ratio per old entry
    mandatory: List[np.ndarray]      # bool per old entry
    evicted: List[np.ndarray]        # bool per old entry (mandatory or capacity)
    n_capacity: np.ndarray           # capacity evictions per head
    rho_new: List[np.ndarray]        # from-scratch density of the new bank entries
    near_ties: int                   # decisions with relative margin < tie_margin
    margins: dict
    tie_cand_ids: List[set] = None   # per head: candidate ids in a near-tie decision
    tie_bank_ids: List[set] = None   # per head: old bank ids in a near-tie decision
    forced: bool = False             # the decisions were given (a replay), not taken


def _lex_order(primary: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Indices sorted by (primary ascending, id ascending)."""
    return np.lexsort((np.asarray(ids), np.asarray(primary)))


def admit(banks: List[HeadBank], cand_ids: np.ndarray, candK: np.ndarray, candV: np.ndarray,
          p: Params, tie_margin: float = 1e-4, prefix_bound: Optional[int] = None,
          forced=None) -> AdmitResult:
    """One admit step for one layer.  candK/candV [H][N][d] (storage precision).

    ``prefix_bound`` caps the synchronised P from outside: the prefix the other
    heads of the layer allow when ``banks`` holds only some of them (heads split
    across processes); the shared P is then min(own prefix, prefix_bound).

    ``forced = (admitted_ids, evicted_ids)``, one id collection per head, replays
    the step with those decisions instead of taking them (see the module's note on
    near ties); ``ValueError`` if they are not an outcome of the rule within
    ``tie_margin``."""
    H = len(banks)
    cand_ids = np.asarray(cand_ids, dtype=np.int64)
    N = cand_ids.shape[0]
    d = candK.shape[-1]
    h = p.scale(d)
    kw = dict(h=h, eps=p.eps, s=p.s)
    M = p.capacity

    # -- step 2: candidate densities against the bank, disturbance scores ------------
    rho_cand, score, feas = [], [], []
    for hh in range(H):
        b = banks[hh]
        rc = density(candK[hh], b.K, row_ids=cand_ids, col_ids=b.ids, **kw)
        mean0 = float(b.rho0.mean()) if b.size else 0.0
        sc = rc / mean0 if mean0 > 0 else np.zeros(N)
        rho_cand.append(rc)
        score.append(sc)
        feas.append(sc <= p.tau)
    P_h = np.array([_feasible_prefix(p, f, cand_ids) for f in feas])

    # -- step 3: largest feasible prefix, synchronised across heads --------------------
    if p.sync_heads:
        P_sync = int(min(P_h.min(), M, N))
        if prefix_bound is not None:
            P_sync = min(P_sync, max(0, int(prefix_bound)))
        P_all = [P_sync] * H
    else:
        assert prefix_bound is None, "a prefix bound needs synchronised heads"
        P_all = [int(min(P_h[hh], M, N)) for hh in range(H)]
    admitted = []
    for hh in range(H):
        order = _lex_order(_cand_key(p, score[hh]), cand_ids)
        admitted.append(order[:P_all[hh]])
    if forced is not None:
        admitted = [_positions(cand_ids, forced[0][hh], "admitted candidate") for hh in range(H)]
        P_all = [len(a) for a in admitted]

    # -- step 4: projected growth, threshold-first and capacity eviction ---------------
    rho_cur, proj, ratio, mand, evicted, n_cap, cutv = [], [], [], [], [], [], []
    for hh in range(H):
        b = banks[hh]
        A = admitted[hh]
        rcur = density(b.K, b.K, row_ids=b.ids, col_ids=b.ids, **kw)
        pj = density(b.K, candK[hh][A], row_ids=b.ids, col_ids=cand_ids[A], **kw)
        rhat = rcur + pj
        with np.errstate(divide="ignore", invalid="ignore"):
            rt = np.where(b.rho0 > 0, rhat / np.where(b.rho0 > 0, b.rho0, 1.0), 0.0)
        md = _mandatory(p, rt)
        ecap = max(0, b.size - int(md.sum()) + len(A) - M)
        ev = md.copy()
        if ecap:
            rest = np.nonzero(~md)[0]
            order = _lex_order(-_cut_value(p, rt, rhat, b.ids)[rest], b.ids[rest])
            ev[rest[order[:ecap]]] = True
        if forced is not None:
            ev = np.zeros(b.size, bool)
            ev[_positions(b.ids, forced[1][hh], "evicted entry")] = True
            ecap = int((ev & ~md).sum())
        rho_cur.append(rcur)
        proj.append(pj)
        ratio.append(rt)
        cutv.append(_cut_value(p, rt, rhat, b.ids))
        mand.append(md)
        evicted.append(ev)
        n_cap.append(ecap)

    if forced is not None:
        bad = _forced_violations(p, tie_margin, banks, cand_ids, score, admitted, ratio,
                                 [rc + pj for rc, pj in zip(rho_cur, proj)], evicted, prefix_bound)
        if bad:
            raise ValueError("forced decisions are not an outcome of the rule within the near-tie "
                             "margin: " + "; ".join(bad[:8]))

    # -- step 5: new bank, baselines of co-admitted entries set together ---------------
    new_banks, rho_new = [], []
    for hh in range(H):
        b = banks[hh]
        keep = ~evicted[hh]
        A = admitted[hh]
        ids = np.concatenate([b.ids[keep], cand_ids[A]])
        K = np.concatenate([b.K[keep], np.asarray(candK[hh][A], np.float64)])
        V = np.concatenate([b.V[keep], np.asarray(candV[hh][A], np.float64)])
        rn = density(K, K, row_ids=ids, col_ids=ids, **kw)
        n_old = int(keep.sum())
        rho0 = rn.copy() if p.baselines == "refresh" else np.concatenate([b.rho0[keep], rn[n_old:]])
        new_banks.append(HeadBank(ids, K, V, rho0))
        rho_new.append(rn)

    margins = _margins(p, score, P_h, P_all, admitted, ratio, mand, evicted, n_cap, banks, cand_ids, cutv)
    near = sum(int((m < tie_margin).sum()) for m in margins.values())
    tc, tb = _tie_ids(p, score, P_h, P_all, ratio, mand, n_cap, banks, cand_ids, tie_margin, cutv)
    return AdmitResult(new_banks, P_all[0] if p.sync_heads else -1, P_h, rho_cand, score, admitted,
                       rho_cur, proj, ratio, mand, evicted, np.array(n_cap), rho_new, near, margins, tc, tb,
                       forced is not None)


def _positions(ids: np.ndarray, want, what: str) -> np.ndarray:
    """Positions in ``ids`` of the ids in ``want`` (each must occur, once)."""
    want = np.asarray(sorted(int(v) for v in want), np.int64)
    if np.unique(want).size != want.size:
        raise ValueError(f"forced decisions: a repeated {what} id")
    pos = {int(v): k for k, v in enumerate(np.asarray(ids).tolist())}
    missing = [int(v) for v in want if int(v) not in pos]
    if missing:
        raise ValueError(f"forced decisions: {what} ids not present: {missing[:8]}")
    return np.array([pos[int(v)] for v in want], np.int64)


def _clearly_below(a, b, m):
    """a is below b by a relative margin of at least m (a < b and a <= (1 - m) b,
    values >= 0): no perturbation of relative size below m makes a >= b."""
    a, b = np.asarray(a), np.asarray(b)
    return (a < b) & (a <= (1.0 - m) * b)


def _order_violations(key_first: np.ndarray, ids_first: np.ndarray, key_rest: np.ndarray,
                      ids_rest: np.ndarray, m: float) -> int:
    """How many pairs (x in first, y in rest) break the order "x before y" by
    (key descending, id ascending) beyond the margin: key(x) clearly below key(y),
    or equal keys with id(x) > id(y).  Equal keys are taken exactly (no margin): the
    same inputs give the same value in any precision, and the id then decides."""
    if key_first.size == 0 or key_rest.size == 0:
        return 0
    n = int(_clearly_below(key_first[:, None], key_rest[None, :], m).sum())
    eq = key_first[:, None] == key_rest[None, :]
    n += int((eq & (ids_first[:, None] > ids_rest[None, :])).sum())
    return n


def feasible_bounds(p: Params, score: np.ndarray, cand_ids: np.ndarray, m: float):
    """(clear, possible): a head's feasible count with tau shrunk and grown by the
    relative margin m -- the range in which another rounding of its scores may put
    it (DensityKV App. E feasible prefix, either candidate order)."""
    return (_feasible_prefix(p, score <= p.tau * (1.0 - m), cand_ids),
            _feasible_prefix(p, score < p.tau * (1.0 + m), cand_ids))


def mandatory_bounds(p: Params, ratio: np.ndarray, m: float):
    """(clear, possible): the number of threshold evictions (ratio > tau) with tau
    grown and shrunk by the relative margin m; (0, 0) for densest-only."""
    if p.eviction == "densest":
        return 0, 0
    return int((ratio >= p.tau * (1.0 + m)).sum()), int((ratio > p.tau * (1.0 - m)).sum())


def _forced_violations(p, m, banks, cand_ids, score, admitted, ratio, rhat, evicted, prefix_bound):
    """Decisions of a replay (admitted candidate positions per head, evicted flags
    per old entry) that no relative perturbation below ``m`` of the deciding values
    could produce under the rule.  Returns one message per violated condition.

    Admission, per head with scores S (all 0 when the bank is empty or its mean
    baseline is 0):
      * a head's feasible count lies between the counts with tau shrunk and grown
        by m; the shared P (synchronised heads) lies between the minima of those
        counts (capped by M, N and the outside bound);
      * every admitted candidate has S < tau (1 + m);
      * disturbance order: no rejected candidate precedes an admitted one by
        (S ascending, id ascending) beyond the margin; source order: the admitted
        candidates are exactly the P lowest ids.
    Eviction, per head with projected ratios R under the admitted set:
      * the bank fits: |B| - |E| + P <= M;
      * threshold modes: no survivor has R >= tau (1 + m); |E| lies between
        max(#{R >= tau (1+m)}, need) and max(#{R > tau (1-m)}, need), need =
        max(0, |B| + P - M); an evicted entry with R <= tau (1 - m) is a capacity
        eviction, so there are only as many evictions as make room, and it precedes
        every survivor by (R descending, id ascending)
        beyond the margin (ratio order) or has a smaller id than every survivor
        (source-order completion);
      * densest-only: |E| = need, and the evicted precede the survivors by
        (R-hat descending, id ascending) beyond the margin."""
    H = len(banks)
    M = p.capacity
    N = cand_ids.shape[0]
    out = []
    lo_h, hi_h = [], []
    for hh in range(H):
        lo, hi = feasible_bounds(p, score[hh], cand_ids, m)
        lo_h.append(lo)
        hi_h.append(hi)
    P_all = [len(a) for a in admitted]
    if p.sync_heads:
        cap = min(M, N) if prefix_bound is None else min(M, N, max(0, int(prefix_bound)))
        lo, hi = min(min(lo_h), cap), min(min(hi_h), cap)
        if len(set(P_all)) != 1:
            out.append(f"admitted counts differ across synchronised heads: {P_all}")
        elif not lo <= P_all[0] <= hi:
            out.append(f"shared P {P_all[0]} outside [{lo}, {hi}]")
    else:
        for hh in range(H):
            lo, hi = min(lo_h[hh], M, N), min(hi_h[hh], M, N)
            if not lo <= P_all[hh] <= hi:
                out.append(f"head {hh}: P {P_all[hh]} outside [{lo}, {hi}]")
    for hh in range(H):
        S = score[hh]
        A = np.asarray(admitted[hh], np.int64)
        rej = np.setdiff1d(np.arange(N), A)
        if (S[A] >= p.tau * (1.0 + m)).any():
            out.append(f"head {hh}: an admitted candidate is clearly infeasible")
        if p.cand_order == "source":
            if set(cand_ids[A].tolist()) != set(np.sort(cand_ids)[:A.size].tolist()):
                out.append(f"head {hh}: source order admits other than the {A.size} lowest ids")
        else:
            # by (S ascending, id ascending) no rejected candidate r may precede an
            # admitted a: S(r) clearly below S(a), or equal scores and the smaller id
            SR, SA, iR, iA = S[rej][:, None], S[A][None, :], cand_ids[rej][:, None], cand_ids[A][None, :]
            n = int((_clearly_below(SR, SA, m) | ((SR == SA) & (iR < iA))).sum())
            if n:
                out.append(f"head {hh}: {n} (admitted, rejected) pairs out of order")
    for hh in range(H):
        b = banks[hh]
        R, Rh, ev = ratio[hh], rhat[hh], evicted[hh]
        P = P_all[hh]
        surv = ~ev
        if b.size - int(ev.sum()) + P > M:
            out.append(f"head {hh}: the bank exceeds M")
        need = max(0, b.size + P - M)
        if p.eviction == "densest":
            if int(ev.sum()) != need:
                out.append(f"head {hh}: densest-only evicts {int(ev.sum())}, not {need}")
            if _order_violations(Rh[ev], b.ids[ev], Rh[surv], b.ids[surv], m):
                out.append(f"head {hh}: an evicted entry is clearly less dense than a survivor")
            continue
        clear_mand = R >= p.tau * (1.0 + m)
        maybe_mand = R > p.tau * (1.0 - m)
        if (clear_mand & surv).any():
            out.append(f"head {hh}: a survivor is clearly above tau")
        E = int(ev.sum())
        n_lo, n_hi = mandatory_bounds(p, R, m)
        if not max(n_lo, need) <= E <= max(n_hi, need):
            out.append(f"head {hh}: {E} evictions outside [{max(n_lo, need)}, {max(n_hi, need)}]")
        capv = ev & ~maybe_mand            # evicted entries that can only be capacity evictions
        if capv.any() and E > need:
            out.append(f"head {hh}: {E} evictions where {need} make room, one of them not above tau")
        if p.eviction == "source":
            if capv.any() and surv.any() and b.ids[capv].max() > b.ids[surv].min():
                out.append(f"head {hh}: a capacity eviction is younger than a survivor")
        elif _order_violations(R[capv], b.ids[capv], R[surv], b.ids[surv], m):
            out.append(f"head {hh}: a capacity eviction clearly ranks below a survivor")
    return out


def _feasible_prefix(p: Params, feasible: np.ndarray, cand_ids: np.ndarray) -> int:
    """Length of a head's largest feasible prefix of the candidate order: every
    feasible candidate (disturbance order puts them first), or, in source order,
    the leading run of feasible candidates by id."""
    if p.cand_order == "source":
        f = feasible[np.argsort(cand_ids, kind="stable")]
        return int(f.size if f.all() else np.argmin(f))
    return int(feasible.sum())


def _cand_key(p: Params, score: np.ndarray) -> np.ndarray:
    """Primary key of the candidate order (ties: id ascending): the disturbance
    score, or nothing (source order, i.e. by id alone)."""
    return np.zeros_like(score) if p.cand_order == "source" else score


def _mandatory(p: Params, ratio: np.ndarray) -> np.ndarray:
    """Threshold-first evictions: projected ratio above tau (none when densest-only)."""
    if p.eviction == "densest":
        return np.zeros(ratio.shape, bool)
    return ratio > p.tau


def _cut_value(p: Params, ratio: np.ndarray, rhat: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """The value whose descending order (ties: id ascending) picks the capacity
    evictions: the projected ratio (default), the projected density (densest-only),
    or minus the id (source order: oldest first)."""
    if p.eviction == "densest":
        return rhat
    if p.eviction == "source":
        return -np.asarray(ids, np.float64)
    return ratio


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        r = np.abs(a - b) / np.maximum(np.abs(b), 1e-300)
    return np.where(np.isnan(r), np.inf, r)


def _margins(p, score, P_h, P_all, admitted, ratio, mand, evicted, n_cap, banks, cand_ids, cutv):
    """Relative margins of every decision that a rounding difference could flip.

    * admission threshold: |score - tau| / tau for each candidate;
    * admission cut (when P is below a head's feasible count): relative gap between
      the last admitted and the first rejected score of that head;
    * eviction threshold: |ratio - tau| / tau per bank entry;
    * capacity cut: relative gap between the last capacity-evicted and the first
      kept non-mandatory ratio."""
    out = {"adm_thr": [], "adm_cut": [], "ev_thr": [], "ev_cut": []}
    for hh in range(len(score)):
        if banks[hh].size and banks[hh].rho0.mean() > 0:
            out["adm_thr"].append(_rel(score[hh], p.tau))
        P = P_all[hh]
        if 0 < P < int(P_h[hh]) and p.cand_order != "source":   # ids never tie
            order = _lex_order(score[hh], cand_ids)
            a, b = score[hh][order[P - 1]], score[hh][order[P]]
            out["adm_cut"].append(np.array([_rel(b, a) if a != 0 else 1.0]))
        if banks[hh].size and p.eviction != "densest":
            out["ev_thr"].append(_rel(ratio[hh], p.tau))
        if n_cap[hh] > 0 and p.eviction != "source":   # ids never tie
            cv = cutv[hh]
            rest = np.nonzero(~mand[hh])[0]
            order = _lex_order(-cv[rest], banks[hh].ids[rest])
            if n_cap[hh] < rest.size:
                a = cv[rest[order[n_cap[hh] - 1]]]
                b = cv[rest[order[n_cap[hh]]]]
                out["ev_cut"].append(np.array([_rel(b, a) if a != 0 else 1.0]))
    return {k: (np.concatenate(v) if v else np.zeros(0)) for k, v in out.items()}


def _tie_ids(p, score, P_h, P_all, ratio, mand, n_cap, banks, cand_ids, m, cutv):
    """Ids whose admit/evict decision could flip under a relative perturbation < m."""
    tc, tb = [], []
    for hh in range(len(score)):
        c, b = set(), set()
        if banks[hh].size and banks[hh].rho0.mean() > 0:
            c |= set(cand_ids[_rel(score[hh], p.tau) < m].tolist())
        P = P_all[hh]
        if 0 < P < int(P_h[hh]) and p.cand_order != "source":
            order = _lex_order(score[hh], cand_ids)
            lo, hi = score[hh][order[P - 1]], score[hh][order[P]]
            close = np.abs(score[hh] - lo) <= m * max(abs(lo), 1e-300)
            if _rel(hi, lo) < m:
                c |= set(cand_ids[close | (np.abs(score[hh] - hi) <= m * max(abs(hi), 1e-300))].tolist())
        ids = banks[hh].ids
        if banks[hh].size and p.eviction != "densest":
            near = _rel(ratio[hh], p.tau) < m
            b |= set(ids[near].tolist())
            k = int(near.sum())
            if k and p.eviction == "source":
                # each flipped threshold decision moves the capacity cut by one in
                # id order, onto entries whose own decision is not close
                raw = banks[hh].size - int(mand[hh].sum()) + P - p.capacity
                rest = np.sort(ids[~mand[hh]])
                b |= set(rest[max(0, raw - k):max(0, raw + k)].tolist())
        if n_cap[hh] > 0 and p.eviction != "source":
            cv = cutv[hh]
            rest = np.nonzero(~mand[hh])[0]
            order = _lex_order(-cv[rest], ids[rest])
            if n_cap[hh] < rest.size:
                lo = cv[rest[order[n_cap[hh] - 1]]]
                hi = cv[rest[order[n_cap[hh]]]]
                if _rel(hi, lo) < m:
                    b |= set(ids[(np.abs(cv - lo) <= m * abs(lo)) | (np.abs(cv - hi) <= m * abs(hi))].tolist())
        tc.append(c)
        tb.append(b)
    return tc, tb


def densities_from_scratch(bank: HeadBank, p: Params) -> np.ndarray:
    d = bank.K.shape[-1]
    return density(bank.K, bank.K, row_ids=bank.ids, col_ids=bank.ids, h=p.scale(d), eps=p.eps, s=p.s)


def attention_set(bank: HeadBank, sinkK, sinkV, winK, winV):
    """K/V read by the current chunk: [sink | bank | local window] (DensityKV Fig. 2)."""
    K = np.concatenate([np.asarray(sinkK, np.float64), bank.K, np.asarray(winK, np.float64)])
    V = np.concatenate([np.asarray(sinkV, np.float64), bank.V, np.asarray(winV, np.float64)])
    return K, V


def rollout(layer_inputs, p: Params, steps: int, attend: bool = True, tie_margin: float = 1e-4,
            on_step: Optional[callable] = None):
    """Run admit (+ attention) for steps 1..steps of one layer; returns per-step results."""
    from .attention import attention
    w = layer_inputs.w
    H = len(layer_inputs.heads)
    banks = [HeadBank.empty(w.head_dim) for _ in range(H)]
    results = []
    for i in range(1, steps + 1):
        x = layer_inputs.step(i)
        r = admit(banks, x["cand_ids"], x["candK"], x["candV"], p, tie_margin)
        banks = r.banks
        outs = None
        if attend:
            outs = []
            for hh in range(H):
                K, V = attention_set(banks[hh], x["sinkK"][hh], x["sinkV"][hh], x["winK"][hh], x["winV"][hh])
                outs.append(attention(x["Q"][hh], K, V))
        rec = {"step": i, "admit": r, "attn": outs, "inputs": x}
        if on_step is not None:
            on_step(rec)
        results.append(rec)
    return results
