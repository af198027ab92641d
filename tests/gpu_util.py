"""Helpers shared by the GPU tests: numpy (storage-precision float32) <-> torch."""
import numpy as np


def dev_tensor(x, dtype="bf16"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.cuda().contiguous()


def dev_ids(ids):
    import torch
    return torch.from_numpy(np.ascontiguousarray(ids, dtype=np.int32)).cuda()


def host(t):
    import torch
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float16) else t.detach().cpu().numpy()


def workspace(nbytes):
    import torch
    return torch.empty(max(int(nbytes), 256) + 256, dtype=torch.uint8, device="cuda")


def aligned_ptr(buf):
    p = buf.data_ptr()
    return (p + 255) & ~255


def import_oracle_banks(bank, banks, params, w, layer=0, densities=True):
    """Load oracle HeadBanks into a GPU bank, with from-scratch densities (or, for
    callers that only attend over the bank, with rho = rho0)."""
    import torch
    from oracle import densitykv as dkv
    for hh, b in enumerate(banks):
        if b.size == 0:
            bank.import_(layer, hh, torch.zeros(0, dtype=torch.int32, device="cuda"), None, None, None, None)
            continue
        rho = dkv.densities_from_scratch(b, params) if densities else b.rho0
        bank.import_(layer, hh, dev_ids(b.ids), dev_tensor(rho, "f32"), dev_tensor(b.rho0, "f32"),
                     dev_tensor(b.K, w.dtype), dev_tensor(b.V, w.dtype))


def export_banks(bank, layer, H):
    """Host copies (ids, rho, rho0, K, V as numpy) of every head's bank of a layer."""
    out = []
    for hh in range(H):
        ids, rho, rho0, K, V = bank.export(layer, hh)
        out.append(dict(ids=host(ids).astype(np.int64), rho=host(rho).astype(np.float64),
                        rho0=host(rho0).astype(np.float64), K=host(K), V=host(V)))
    return out


def check_admit_sampled(w, pre, post, stats, cand_ids, candK, rng, rtol=1e-4, n=12):
    """One GPU admit step at any size, checked on sampled outputs the oracle
    computes one by one and on the rule's invariants (DensityKV §3, App. B.1):
    * sizes <= M, the same admitted count P on every head, K/V pairing by id;
    * rho of sampled entries of the new bank = from-scratch oracle density within
      rtol; new entries have rho0 = rho, survivors keep their rho0;
    * admitted candidates precede rejected ones in (score, id) order, and are all
      feasible when every candidate is admitted;
    * survivors have projected ratio <= tau, and every evicted entry has a ratio
      at least every survivor's (mandatory ones above tau, capacity ones next).
    pre / post: export_banks before / after the step; candK [H][N][d] (host or
    torch); cand_ids [N]."""
    import kvgen
    from oracle.density import density
    H = len(post)
    kw = dict(h=float(w.head_dim), eps=w.eps, s=w.s)
    cand_ids = np.asarray(host(cand_ids) if hasattr(cand_ids, "cpu") else cand_ids, np.int64)
    cK = np.asarray(host(candK) if hasattr(candK, "cpu") else candK, np.float64)
    cid_pos = {int(c): k for k, c in enumerate(cand_ids)}
    assert len({s["admitted"] for s in stats}) == 1
    for hh in range(H):
        b0, b1 = pre[hh], post[hh]
        assert b0["ids"].size <= w.capacity and b1["ids"].size <= w.capacity
        assert (kvgen.untag_ids(b1["V"]) == b1["ids"]).all()
        pre_pos = {int(v): k for k, v in enumerate(b0["ids"])}
        adm = np.array([k for k, v in enumerate(b1["ids"]) if int(v) in cid_pos], np.int64)
        surv = np.array([k for k, v in enumerate(b1["ids"]) if int(v) in pre_pos], np.int64)
        assert adm.size == stats[hh]["admitted"] and adm.size + surv.size == b1["ids"].size
        evicted = np.array(sorted(set(pre_pos) - set(b1["ids"].tolist())), np.int64)
        # densities of sampled new-bank entries, from scratch
        smp = np.sort(rng.choice(b1["ids"].size, min(n, b1["ids"].size), replace=False))
        ref = density(b1["K"][smp], b1["K"], row_ids=b1["ids"][smp], col_ids=b1["ids"], **kw)
        np.testing.assert_allclose(b1["rho"][smp], ref, rtol=rtol)
        np.testing.assert_array_equal(b1["rho0"][adm], b1["rho"][adm])
        np.testing.assert_array_equal(b1["rho0"][surv], b0["rho0"][[pre_pos[int(v)] for v in b1["ids"][surv]]])
        if b0["ids"].size == 0:
            continue
        # admission order on sampled candidates (scores against the pre-step bank)
        mean0 = float(np.mean(b0["rho0"]))
        a_ids = sorted(set(b1["ids"][adm].tolist()))
        r_all = sorted(set(cand_ids.tolist()) - set(a_ids))

        def score(ids_):
            rows = cK[hh][[cid_pos[int(c)] for c in ids_]]
            return density(rows, b0["K"], row_ids=np.asarray(ids_), col_ids=b0["ids"], **kw) / mean0

        if a_ids:
            sa = score(rng.choice(a_ids, min(n, len(a_ids)), replace=False))
            if r_all:
                sr = score(rng.choice(r_all, min(n, len(r_all)), replace=False))
                assert sa.max() <= sr.min() * (1 + rtol)
            else:
                assert sa.max() <= w.tau * (1 + rtol)   # every candidate of every head was feasible
        # eviction rule on sampled survivors and evicted entries
        A_rows = cK[hh][[cid_pos[int(c)] for c in a_ids]]
        A_ids = np.asarray(a_ids, np.int64)

        def ratio(ids_):
            k = [pre_pos[int(v)] for v in ids_]
            rows = b0["K"][k]
            rh = density(rows, b0["K"], row_ids=np.asarray(ids_), col_ids=b0["ids"], **kw)
            if A_ids.size:
                rh = rh + density(rows, A_rows, row_ids=np.asarray(ids_), col_ids=A_ids, **kw)
            return rh / b0["rho0"][k]

        if surv.size:
            rs = ratio(rng.choice(b1["ids"][surv], min(n, surv.size), replace=False))
            assert rs.max() <= w.tau * (1 + rtol)
            if evicted.size:
                re_ = ratio(rng.choice(evicted, min(n, evicted.size), replace=False))
                assert re_.min() >= rs.max() * (1 - rtol)


def import_step_state(bank, banks, params, w, layer=0):
    """Load the oracle's banks before a step into the GPU bank (the stepwise
    tests start every GPU step from the oracle's state, so a near-tie decision
    taken the other way never cascades into the next step)."""
    import_oracle_banks(bank, banks, params, w, layer=layer)


def check_admit_step(bank, w, p, banks_pre, x, r, layer=0, m=1e-4, rtol=1e-4, label="", tagged=True):
    """One GPU admit step against the oracle's step r on the same inputs and the
    same starting banks (banks_pre, imported into the GPU bank before the step).

    * The GPU's decisions (admitted candidates, evicted entries per head) must be
      the oracle's, or an outcome of the rule within the near-tie margin m: the
      oracle then replays the step with them (admit(..., forced=...), which raises
      unless every differing decision is a near tie, a shared P moved by a near-tie
      feasibility included).
    * Against that oracle step or replay, every head's bank must match: id set,
      K and V rows bit for bit (by id), V carrying its own id when the inputs are
      tagged, rho and rho0 within rtol; and the
      counters: admitted, size, evictions, feasible and mandatory within the
      ranges the margin allows.
    * At most 2 flips per oracle near-tie decision plus 3 per head and unit of P
      moved (a shared P one higher admits one more candidate per head and may
      evict one more entry).
    Returns (flipped decisions, oracle near-tie decisions)."""
    import kvgen
    from oracle import densitykv as dkv
    H = len(banks_pre)
    cand_ids = np.asarray(x["cand_ids"], np.int64)
    cset = set(cand_ids.tolist())
    # ``bank`` may be a list of (bank, h0, h1): heads h0..h1-1 of the layer held by
    # each of several banks (a head-parallel split)
    parts = bank if isinstance(bank, (list, tuple)) else [(bank, 0, H)]
    g, st = [], []
    for b, h0, h1 in parts:
        g += export_banks(b, layer, h1 - h0)
        st += b.stats(layer)
    assert len(g) == H
    A_gpu, E_gpu, flips = [], [], 0
    for hh in range(H):
        got = set(g[hh]["ids"].tolist())
        A = sorted(got & cset)
        E = sorted(set(banks_pre[hh].ids.tolist()) - got)
        assert len(got) == g[hh]["ids"].size, f"{label} head {hh}: repeated ids in the GPU bank"
        A_or = set(cand_ids[r.admitted[hh]].tolist())
        E_or = set(banks_pre[hh].ids[r.evicted[hh]].tolist())
        flips += len(set(A) ^ A_or) + len(set(E) ^ E_or)
        A_gpu.append(A)
        E_gpu.append(E)
    ref = r
    if flips:
        ref = dkv.admit(banks_pre, cand_ids, x["candK"], x["candV"], p, tie_margin=m, forced=(A_gpu, E_gpu))
    dP = abs(len(A_gpu[0]) - (r.P if r.P >= 0 else len(r.admitted[0])))
    assert flips <= 2 * r.near_ties + 3 * H * dP, \
        f"{label}: {flips} flipped decisions for {r.near_ties} near ties and a P moved by {dP}"
    for hh in range(H):
        gb, ob = g[hh], ref.banks[hh]
        assert set(gb["ids"].tolist()) == set(ob.ids.tolist()), f"{label} head {hh}: bank ids"
        if tagged:
            np.testing.assert_array_equal(kvgen.untag_ids(gb["V"]), gb["ids"])
        go, oo = np.argsort(gb["ids"]), np.argsort(ob.ids)
        np.testing.assert_array_equal(gb["K"][go], ob.K[oo].astype(np.float32))
        np.testing.assert_array_equal(gb["V"][go], ob.V[oo].astype(np.float32))
        np.testing.assert_allclose(gb["rho"][go], ref.rho_new[hh][oo], rtol=rtol, err_msg=f"{label} head {hh} rho")
        np.testing.assert_allclose(gb["rho0"][go], ob.rho0[oo], rtol=rtol, err_msg=f"{label} head {hh} rho0")
        s = st[hh]
        assert s["admitted"] == len(A_gpu[hh]) and s["size"] == ob.size
        assert s["mandatory"] + s["capacity_evicted"] == len(E_gpu[hh])
        lo, hi = dkv.feasible_bounds(p, r.score[hh], cand_ids, m)
        assert lo <= s["feasible"] <= hi, f"{label} head {hh}: feasible {s['feasible']} outside [{lo}, {hi}]"
        mlo, mhi = dkv.mandatory_bounds(p, ref.ratio[hh], m)
        assert mlo <= s["mandatory"] <= mhi, f"{label} head {hh}: mandatory {s['mandatory']} outside [{mlo}, {mhi}]"
    # the kernels' own near-tie count (fp32 values) against the oracle's (fp64): a
    # value right at the margin may fall on either side, and a flipped decision
    # moves its cut
    gpu_ties = sum(s["near_ties"] for s in st)
    assert abs(gpu_ties - r.near_ties) <= 2 + 2 * flips, f"{label}: near ties {gpu_ties} (GPU) vs {r.near_ties}"
    return flips, r.near_ties
