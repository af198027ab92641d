#!/usr/bin/env python3
"""Benchmark of the KV-bank hot path: ms per chunk-layer (bank update + history
attention) on synthetic Wan2.1-1.3B-shaped data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan480|wan1080|forcing480|mid|tiny]
                    [--impl kvb|reference]

A step is one chunk-layer of the streaming rollout: one DensityKV kvb_admit of
the block that just left the local window (4680 candidates at 480P) followed by
one kvb_attend of the current chunk's 4680 queries over [sink frame | bank |
3-frame window]; for the Forcing-KV workload one kvb_prune_hybrid followed by
kvb_attend.  The bank is first brought to steady state (the timed steps are
chunks 19, 20, ... of the rollout at 480P), all inputs are resident in HBM, L2 is
flushed (a 256 MB write) before every timed step, and every step is timed with
CUDA events on the launching stream.

`--impl reference` times the fp64 CPU oracle (the parity reference, plain and
slow) on a bounded sample of the same workload and prints the same JSON line.
Under torchrun each rank runs an independent replica (the path shards by
layer and head; there is no data exchange), `value` = max-over-ranks time /
(ranks x steps).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kvgen  # noqa: E402

METRIC = "ms per chunk-layer (bank update + history attention)"
UNIT = "ms"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = str(index)
        try:
            # the process may see a remapped device 0: address the GPU by PCI bus id
            import torch
            pr = torch.cuda.get_device_properties(index)
            bus = getattr(pr, "pci_bus_id", None)
            dom = getattr(pr, "pci_domain_id", 0)
            dv = getattr(pr, "pci_device_id", 0)
            if bus is not None:
                self.index = f"{dom:08X}:{bus:02X}:{dv:02X}.0"
        except Exception:
            pass
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.file, stderr=subprocess.DEVNULL)
            # nvidia-smi needs about a second before its first sample: wait for it
            t0 = time.time()
            while time.time() - t0 < 10 and os.path.getsize(self.file.name) == 0:
                time.sleep(0.05)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [ln.strip().split(",") for ln in self.file.read().splitlines() if ln.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                smax.append(float(r[1]))
                for nm, v in zip(names, r[4:8]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        if sm:
            out.update(sm_mhz=statistics.median(sm), sm_max_mhz=max(smax), reasons=sorted(reasons), samples=len(sm))
        return out


# ------------------------------------------------------------------ distributed
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ inputs
def upload_step(x, dt):
    import torch
    out = {}
    for k, v in x.items():
        if k in ("cand_ids", "new_ids"):
            out[k] = torch.from_numpy(np.ascontiguousarray(v, dtype=np.int32)).cuda()
        else:
            t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
            out[k] = (t.to(torch.bfloat16) if dt == "bf16" else t).cuda()
    return out


def host_step(x, dt):
    """pinned host copies (for the end-to-end leg)."""
    import torch
    out = {}
    for k, v in x.items():
        if k in ("cand_ids", "new_ids"):
            t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.int32))
        else:
            t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
            t = t.to(torch.bfloat16) if dt == "bf16" else t
        out[k] = t.pin_memory()
    return out


def _cfg(w, kvb):
    return kvb.make_config(method=kvb.KVB_DENSITYKV, dtype=kvb.KVB_BF16 if w.dtype == "bf16" else kvb.KVB_F32,
                           layers=1, heads=w.heads, head_dim=w.head_dim, capacity=w.capacity,
                           max_candidates=w.chunk_tokens, tau=w.tau, eps=w.eps, s=w.s, sync_heads=1,
                           max_queries=w.chunk_tokens)


FIRST_TIMED = {"wan480": 19, "wan1080": 9, "mid": 4, "tiny": 4}


def attention_flops(w, sizes):
    """4 * Nq * Lk * d summed over heads (Lk = sink + bank_h + window)."""
    Nq = w.chunk_tokens
    return sum(4.0 * Nq * (w.F + s + w.chunk_tokens) * w.head_dim for s in sizes)


def density_flops(w, N, st_before, st_after):
    """Executed density work of one admit: 2d flops per pair over the four passes
    (candidates x bank, bank x admitted, new bank x evicted, admitted x admitted)."""
    f = 0.0
    for b0, s in zip(st_before, st_after):
        P, E = s["admitted"], s["mandatory"] + s["capacity_evicted"]
        f += 2.0 * w.head_dim * (N * b0 + b0 * P + s["size"] * E + P * P)
    return f


def density_flops_algorithmic(w, N, st_before, st_after):
    """The method's own count: N*|B| + P^2 + E*(|B| - E + P) pairs (App. B.1, O(N M d))."""
    f = 0.0
    for b0, s in zip(st_before, st_after):
        P, E = s["admitted"], s["mandatory"] + s["capacity_evicted"]
        f += 2.0 * w.head_dim * (N * b0 + P * P + E * (b0 - E + P))
    return f


def run_densitykv(args, w, rank, world):
    import torch
    import kv_cache_compression_post_b200 as kvb
    dev = torch.cuda.current_device()
    first = FIRST_TIMED.get(w.name, 4)
    n_dev_steps = args.warmup + args.steps
    total_steps = first - 1 + n_dev_steps + args.steps  # pre-roll, device-timed, end-to-end
    t0 = time.time()
    L = kvgen.LayerInputs(w, 0, n_chunks=total_steps + 2, seed_offset=rank)
    inputs = {}
    for i in range(1, first + n_dev_steps):
        inputs[i] = upload_step(L.step(i), w.dtype)
    hosted = {i: host_step(L.step(i), w.dtype) for i in range(first + n_dev_steps, total_steps + 1)}
    gen_s = time.time() - t0

    bank = kvb.Bank(_cfg(w, kvb))
    stream = torch.cuda.current_stream()
    O = torch.empty_like(inputs[1]["Q"])
    lse = torch.empty(w.heads, w.chunk_tokens, device="cuda")
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")

    def step(x):
        bank.admit(0, x["candK"], x["candV"], x["cand_ids"], stream)
        bank.attend(0, x["Q"], x["sinkK"], x["sinkV"], x["winK"], x["winV"], O, lse, stream)

    # pre-roll to steady state, then warm-up
    for i in range(1, first + args.warmup):
        step(inputs[i])
    torch.cuda.synchronize()
    if bank.status() != 0:
        raise RuntimeError(f"device status {bank.status()} after warm-up")

    sampler = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    per_step, adm_ms, att_ms, att_fl, den_fl, den_alg = [], [], [], [], [], []
    launches0 = kvb.kvb_launch_count()
    for i in range(first + args.warmup, first + n_dev_steps):
        x = inputs[i]
        flush.fill_(1.0)
        st_before = [s["size"] for s in bank.stats(0)]
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        torch.cuda.synchronize()
        e0.record(stream)
        bank.admit(0, x["candK"], x["candV"], x["cand_ids"], stream)
        e1.record(stream)
        bank.attend(0, x["Q"], x["sinkK"], x["sinkV"], x["winK"], x["winV"], O, lse, stream)
        e2.record(stream)
        torch.cuda.synchronize()
        a_ms, t_ms = e0.elapsed_time(e1), e1.elapsed_time(e2)
        st = bank.stats(0)
        adm_ms.append(a_ms)
        att_ms.append(t_ms)
        per_step.append(a_ms + t_ms)
        att_fl.append(attention_flops(w, [s["size"] for s in st]))
        den_fl.append(density_flops(w, x["cand_ids"].shape[0], st_before, st))
        den_alg.append(density_flops_algorithmic(w, x["cand_ids"].shape[0], st_before, st))
    launches = kvb.kvb_launch_count() - launches0
    clocks = sampler.stop()
    barrier(world)
    status = bank.status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    total_ms = max_over_ranks(sum(per_step), world)

    # end-to-end: host (pinned) inputs in, result out, every step
    Oh = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    h2d = d2h = 0
    dev_bufs = {k: torch.empty_like(v, device="cuda") for k, v in next(iter(hosted.values())).items()}
    barrier(world)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for i in sorted(hosted):
        hx = hosted[i]
        for k, v in hx.items():
            if dev_bufs[k].shape != v.shape:
                dev_bufs[k] = torch.empty_like(v, device="cuda")
            dev_bufs[k].copy_(v, non_blocking=True)
            h2d += v.numel() * v.element_size()
        step(dev_bufs)
        Oh.copy_(O, non_blocking=True)
        d2h += O.numel() * O.element_size()
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_total = max_over_ranks(e_start.elapsed_time(e_end), world)
    nh = len(hosted)

    peaks, peak_src = load_peaks()
    att_achieved = statistics.mean(f / (t * 1e-3) for f, t in zip(att_fl, att_ms)) / 1e12
    den_achieved = statistics.mean(f / (t * 1e-3) for f, t in zip(den_fl, adm_ms)) / 1e12
    dominant_attend = statistics.mean(att_ms) >= statistics.mean(adm_ms)
    bf16_peak = peaks["bf16_tflops"]

    def roof(achieved, kernel, per_unit, traffic=None):
        return {"bound": "tensor", "achieved": round(achieved, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                "frac": round(achieved / bf16_peak, 4), "traffic": traffic, "kernel": kernel,
                "peak_source": f"{peak_src} bf16 burst", "algorithmic": per_unit}

    roof_att = roof(att_achieved, "attend_bf16_kernel (kvb_attend, 1 launch)",
                    "4*Nq*(Ls+|B_h|+Lw)*d flops summed over heads")
    roof_den = roof(den_achieved, "kvb_admit (4 density Gram launches + selection/compaction)",
                    "2*d*(N|B| + |B|P + |B'|E + P^2) flops summed over heads")
    return {
        "ms_per_step": total_ms / (world * args.steps),
        "e2e_ms": e2e_total / (world * nh),
        "h2d": h2d // nh, "d2h": d2h // nh,
        "clocks": clocks, "launches": launches,
        "roofline": roof_att if dominant_attend else roof_den,
        "roofline_other": roof_den if dominant_attend else roof_att,
        "breakdown": {"admit_ms": round(statistics.mean(adm_ms), 4), "attend_ms": round(statistics.mean(att_ms), 4),
                      "attend_tflops": round(att_achieved, 1), "admit_density_tflops": round(den_achieved, 1),
                      "density_algorithmic_gflop": round(statistics.mean(den_alg) / 1e9, 1),
                      "density_executed_gflop": round(statistics.mean(den_fl) / 1e9, 1),
                      "attention_gflop": round(statistics.mean(att_fl) / 1e9, 1),
                      "bank_sizes": [s["size"] for s in bank.stats(0)],
                      "admitted": [s["admitted"] for s in bank.stats(0)][:1]},
        "gen_s": round(gen_s, 1),
        "first_timed_chunk": first + args.warmup,
    }


# ------------------------------------------------------------------ oracle (CPU) leg
def oracle_sample(w, reps: int = 1):
    """Time the fp64 oracle on a bounded, stated sample of one 480P chunk-layer and
    extrapolate linearly to the full chunk-layer (rows of every density / attention
    evaluation are independent, so time scales with rows)."""
    import oracle
    from oracle.attention import attention
    from oracle.density import density
    L = kvgen.LayerInputs(w, 0, n_chunks=FIRST_TIMED.get(w.name, 4) + 1, heads=[0])
    i = FIRST_TIMED.get(w.name, 4)
    x = L.step(i)
    # bank stand-in: memory keys of the six frames before the candidate block
    mem_frames = list(range(max(1, (i - 1) * w.chunk_frames - 6), (i - 1) * w.chunk_frames))
    Kb = L.keys(mem_frames, memory=True)[0][:w.capacity]
    Vb = L.values(mem_frames)[0][:w.capacity]
    Mb = Kb.shape[0]
    cand = x["candK"][0]
    N = cand.shape[0]
    rr, qr = 512, 256
    kw = dict(h=float(w.head_dim), eps=w.eps, s=w.s)
    times = []
    for _ in range(reps):
        t = time.perf_counter()
        density(cand[:rr], Kb, **kw)                                   # rho_B of candidates
        t1 = time.perf_counter()
        density(Kb[:rr], Kb, row_ids=np.arange(rr), col_ids=np.arange(Mb), **kw)  # from-scratch bank density
        t2 = time.perf_counter()
        density(Kb[:rr], cand, **kw)                                   # projected growth
        t3 = time.perf_counter()
        Kall = np.concatenate([x["sinkK"][0], Kb, x["winK"][0]])
        Vall = np.concatenate([x["sinkV"][0], Vb, x["winV"][0]])
        attention(x["Q"][0][:qr], Kall, Vall)
        t4 = time.perf_counter()
        per_head = ((t1 - t) * N / rr + (t2 - t1) * 2 * Mb / rr + (t3 - t2) * Mb / rr
                    + (t4 - t3) * w.chunk_tokens / qr)
        times.append(per_head * w.heads * 1e3)
    try:
        from threadpoolctl import threadpool_info
        blas_threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:
        blas_threads = None
    sample = (f"one head of a 480P chunk-layer (step {i}): density of {rr} of {N} candidates vs {Mb} bank keys, "
              f"from-scratch density of {rr} of {Mb} bank keys (x2: before and after the update), projected "
              f"growth of {rr} bank keys vs {N} candidates, attention of {qr} of {w.chunk_tokens} queries over "
              f"{Kall.shape[0]} keys; scaled by rows and by {w.heads} heads")
    return statistics.mean(times), sample, (os.cpu_count(), blas_threads)


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    t0 = time.time()
    ms, sample, (cores, blas) = oracle_sample(w, reps=max(1, args.steps))
    line = {"impl": "reference", "metric": METRIC, "value": round(ms, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "heads": w.heads, "head_dim": w.head_dim, "F": w.F,
                       "N": w.chunk_tokens, "M": w.capacity},
            "cpu_baseline": {"value": round(ms, 3), "unit": UNIT, "cores": cores, "blas_threads": blas,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(ms, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.time() - t0, 1)}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="wan480")
    ap.add_argument("--impl", default="kvb", choices=["kvb", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = kvgen.WORKLOADS[args.workload]
    rank, world, local = dist_init()
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    import torch
    torch.cuda.set_device(local)
    r = run_densitykv(args, w, rank, world)
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        ms, sample, (cores, blas) = oracle_sample(w, reps=1)
        cpu = {"value": round(ms, 3), "unit": UNIT, "cores": cores, "blas_threads": blas, "kind": "oracle",
               "sample": sample}
    line = {
        "metric": METRIC, "value": round(r["ms_per_step"], 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms_per_step"], 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16"
        else "f32", "data": "synthetic",
        "config": {"workload": (f"{w.name}: DensityKV admit of {w.chunk_tokens} candidates + attention of "
                                f"{w.chunk_tokens} queries over sink {w.F} + bank (M={w.capacity}) + window "
                                f"{w.chunk_tokens}; {w.heads} heads, d={w.head_dim}, 1 layer, chunks "
                                f"{r['first_timed_chunk']}..{r['first_timed_chunk'] + args.steps - 1}"),
                   "heads": w.heads, "head_dim": w.head_dim, "F": w.F, "N": w.chunk_tokens, "M": w.capacity,
                   "tau": w.tau, "parallelism": f"replicas x{world}", "l2": "flushed (256 MB write) before each step"},
        "e2e": {"value": round(r["e2e_ms"], 4), "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "roofline": r["roofline"],
        "roofline_other": r["roofline_other"],
        "breakdown": r["breakdown"],
        "clocks": r["clocks"],
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
