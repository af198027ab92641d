"""Exact-fraction derivation of the expected values in densitykv_hand.json.

    python tests/golden/derive_densitykv_hand.py           # check: every stored value is re-derived
    python tests/golden/derive_densitykv_hand.py --write   # rewrite the "expect" blocks

The scenarios put 1-D keys in banks with h = 1, eps = 1, s = 2, so the
Soft-Riesz interaction phi(a, b) = (|a - b|^2 + 1)^-1 is a rational number and
every density, score and ratio of an admit step is an exact fraction.  This
script applies the admit rule of DensityKV App. B.1 "Online Bank Update", §3 and
App. E (the default policy and the ablation switches a scenario names) step by
step in Python's Fraction arithmetic, under the readings the library states:

  score(c)   = rho_B(c) / mean of the bank's baselines rho0 (0 for an empty bank
               or a zero mean), feasible iff score <= tau;
  P          = min(min over heads of the feasible count, M, N) (synchronised) or
               per head; a head admits its P lowest (score, id), or its P lowest
               ids under source candidate order, whose feasible count is the run of
               feasible candidates from the lowest id;
  ratio(i)   = (rho_i + sum over the admitted of phi) / rho0_i (0 if rho0_i = 0);
               evicted: ratio > tau (not under densest-only), then
               max(0, |B| - mandatory + P - M) more by ratio descending (default),
               projected density descending (densest-only) or id ascending
               (source-order completion), ties to the smaller id;
  new bank   = survivors + admitted; every density recomputed over it; new
               entries take rho0 = that density (every entry does under refresh).

It shares nothing with oracle/ or the CUDA library: it is the independent
derivation the oracle's hand-scenario pins are checked against.
"""
from __future__ import annotations

import json
import os
import sys
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
JSON = os.path.join(HERE, "densitykv_hand.json")


def frac(v) -> Fraction:
    return Fraction(str(v)) if not isinstance(v, str) else Fraction(v)


def text(f: Fraction) -> str:
    return str(f.numerator) if f.denominator == 1 else f"{f.numerator}/{f.denominator}"


def phi(a: Fraction, b: Fraction) -> Fraction:
    return 1 / ((a - b) ** 2 + 1)


def density(key, others):
    """sum of phi(key, k) over (id, k) in others (the caller leaves out the key itself)."""
    return sum((phi(key, k) for _, k in others), Fraction(0))


def admit_step(banks, cand_ids, candK, prm):
    """One admit step; banks: per head a list of (id, key, rho0).  Returns the new
    banks and the step's record (the quantities densitykv_hand.json stores)."""
    tau, M = frac(prm["tau"]), prm["capacity"]
    sync = prm.get("sync_heads", True)
    source_cands = prm.get("cand_order", "score") == "source"
    refresh = prm.get("baselines", "fixed") == "refresh"
    eviction = prm.get("eviction", "ratio")
    H, N = len(banks), len(cand_ids)
    scores, P_h = [], []
    for h in range(H):
        bank = [(i, k) for i, k, _ in banks[h]]
        mean0 = sum((r for _, _, r in banks[h]), Fraction(0)) / len(banks[h]) if banks[h] else Fraction(0)
        sc = [density(frac(candK[h][c]), bank) / mean0 if mean0 > 0 else Fraction(0) for c in range(N)]
        scores.append(sc)
        if source_cands:
            run = 0
            for c in sorted(range(N), key=lambda c: cand_ids[c]):
                if sc[c] > tau:
                    break
                run += 1
            P_h.append(run)
        else:
            P_h.append(sum(1 for s in sc if s <= tau))
    P_all = [min(min(P_h), M, N)] * H if sync else [min(P_h[h], M, N) for h in range(H)]
    rec = {"P_h": P_h, "scores": [[text(s) for s in sc] for sc in scores],
           "admitted_ids": [], "ratio": [], "mandatory_ids": [], "evicted_ids": [], "bank_ids": [], "rho0": [],
           "rho": []}
    if sync:
        rec["P"] = P_all[0]
    new_banks = []
    for h in range(H):
        if source_cands:
            order = sorted(range(N), key=lambda c: cand_ids[c])
        else:
            order = sorted(range(N), key=lambda c: (scores[h][c], cand_ids[c]))
        A = order[:P_all[h]]
        A_keys = [(cand_ids[c], frac(candK[h][c])) for c in A]
        old = banks[h]
        ratio, rhat = {}, {}
        for i, k, r0 in old:
            rho = density(k, [(j, kj) for j, kj, _ in old if j != i])
            rhat[i] = rho + density(k, A_keys)
            ratio[i] = rhat[i] / r0 if r0 > 0 else Fraction(0)
        mand = set() if eviction == "densest" else {i for i, _, _ in old if ratio[i] > tau}
        ecap = max(0, len(old) - len(mand) + len(A) - M)
        rest = [i for i, _, _ in old if i not in mand]
        if eviction == "densest":
            rest.sort(key=lambda i: (-rhat[i], i))
        elif eviction == "source":
            rest.sort()
        else:
            rest.sort(key=lambda i: (-ratio[i], i))
        evicted = mand | set(rest[:ecap])
        keep = [(i, k, r0) for i, k, r0 in old if i not in evicted]
        entries = [(i, k) for i, k, _ in keep] + A_keys
        rho_new = {i: density(k, [(j, kj) for j, kj in entries if j != i]) for i, k in entries}
        base = {i: r0 for i, _, r0 in keep}
        bank = [(i, k, rho_new[i] if (refresh or i not in base) else base[i]) for i, k in entries]
        new_banks.append(bank)
        rec["admitted_ids"].append(sorted(cand_ids[c] for c in A))
        rec["ratio"].append({str(i): text(ratio[i]) for i, _, _ in old})
        rec["mandatory_ids"].append(sorted(mand))
        rec["evicted_ids"].append(sorted(evicted))
        rec["bank_ids"].append(sorted(i for i, _ in entries))
        rec["rho0"].append({str(i): text(r0) for i, _, r0 in bank})
        rec["rho"].append({str(i): text(rho_new[i]) for i, _ in entries})
    return new_banks, rec


def derive(scenario):
    """Yield (step, derived record) for every step of a scenario."""
    prm = scenario["params"]
    for key in ("h", "eps", "s"):
        assert float(prm[key]) == {"h": 1.0, "eps": 1.0, "s": 2.0}[key], "the closed form needs h = eps = 1, s = 2"
    banks = [[] for _ in range(prm["heads"])]
    for st in scenario["steps"]:
        banks, rec = admit_step(banks, st["cand_ids"], st["candK"], prm)
        yield st, rec


def equal(stored: str, derived: str) -> bool:
    """A stored fraction ("p/q" or an integer) must equal the derived one exactly; a
    stored decimal (a few values are written as doubles) must agree to 1e-15."""
    a, b = frac(stored), frac(derived)
    if "." in str(stored):
        return abs(a - b) <= abs(b) * Fraction(1, 10 ** 15)
    return a == b


def mismatches(doc):
    """Every stored expected value that the derivation does not reproduce."""
    bad = []
    for sc in doc["scenarios"]:
        for n, (st, rec) in enumerate(derive(sc)):
            for key, want in st["expect"].items():
                got = rec[key]
                if key in ("scores",):
                    same = all(equal(b, a) for ga, wa in zip(got, want) for a, b in zip(ga, wa)) and \
                        [len(g) for g in got] == [len(w_) for w_ in want]
                elif key in ("ratio", "rho0", "rho"):
                    same = all(set(w_) <= set(g) and all(equal(v, g[k]) for k, v in w_.items())
                               for g, w_ in zip(got, want)) and len(got) == len(want)
                elif key in ("admitted_ids", "mandatory_ids", "evicted_ids", "bank_ids"):
                    same = [sorted(x) for x in got] == [sorted(x) for x in want]
                else:
                    same = got == want
                if not same:
                    bad.append(f"{sc['name']} step {n} {key}: stored {want}, derived {got}")
    return bad


def main(argv):
    doc = json.load(open(JSON))
    if "--write" in argv:
        for sc in doc["scenarios"]:
            for st, rec in derive(sc):
                st["expect"] = {k: rec[k] for k in st["expect"]}
        json.dump(doc, open(JSON, "w"), indent=1)
        return 0
    bad = mismatches(doc)
    for b in bad:
        print(b)
    print("ok" if not bad else f"{len(bad)} mismatches")
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
