"""The multi-rank plumbing of bench.py on CPU (gloo, world size 2): rendezvous on
127.0.0.1, the barrier, and the max-over-ranks reduction that turns per-rank
device times into the job's time.  Each rank runs an independent replica (the
path shards by layer and head; there is no data exchange)."""
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), KVB_DIST_BACKEND="gloo")
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_init()
    bench.barrier(w)
    m = bench.max_over_ranks(1.5 * (r + 1), w)
    bench.barrier(w)
    out.put((r, w, m, dist.get_backend()))
    dist.destroy_process_group()


def test_two_rank_barrier_and_max_over_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 and r[3] == "gloo" for r in res)
    assert all(r[2] == pytest.approx(3.0) for r in res)   # every rank sees the slowest rank's time


@pytest.mark.parametrize("name", ["tiny", "forcing_mid"])
def test_cpu_baseline_record(name):
    """The oracle leg that every bench line carries: a positive time and the keys
    the line needs (threads actually used, host CPUs, the stated sample)."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import kvgen
    ms, cpu = bench.cpu_sample(kvgen.WORKLOADS[name], reps=1)
    assert ms > 0 and cpu["value"] == round(ms, 3)
    assert cpu["kind"] == "oracle" and cpu["unit"] == bench.UNIT
    assert 1 <= cpu["cores"] <= (cpu["host_cpus"] or cpu["cores"])
    assert name.split("_")[0] in cpu["sample"] or "Forcing-KV" in cpu["sample"]


def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched as the driver launches it for N > 1:
    rank 0 alone runs the oracle and prints one JSON line; the other rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, KVB_DIST_BACKEND="gloo")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
