"""The measurement arithmetic of bench.py on CPU: algorithmic flop and byte counts
per step (checked against the per-layer figures the workload is quoted with:
448.6 GFLOP of attention and at most 336 GFLOP of density work per 480P
chunk-layer) and the roofline fractions of the per-kernel table."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import kvgen  # noqa: E402

W = kvgen.WORKLOADS["wan480"]


def _stats(P, mand, cap, size):
    return {"admitted": P, "mandatory": mand, "capacity_evicted": cap, "size": size, "moved": 0}


def test_attention_flops_at_a_full_bank():
    f = bench.attention_flops(W, [W.capacity] * W.heads)
    assert f == 4.0 * 4680 * (1560 + 9360 + 4680) * 128 * 12
    assert f / 1e9 == pytest.approx(448.6, abs=0.05)


def test_density_flops_worst_case_and_pass_split():
    N, M = W.chunk_tokens, W.capacity
    before = [M] * W.heads
    after = [_stats(N, 0, N, M)] * W.heads          # P = E = N, bank full before and after
    alg = bench.density_flops_algorithmic(W, N, before, after)
    assert alg / 1e9 == pytest.approx(336.4, abs=0.1)
    pairs = bench.gram_pairs(N, before, after)
    assert pairs == [N * M * 12.0, M * N * 12.0, M * N * 12.0, N * N * 12.0]
    assert bench.density_flops(W, N, before, after) == 2.0 * 128 * sum(pairs)
    # the executed passes recompute the P x |B| projected growth on top of the method's count
    assert bench.density_flops(W, N, before, after) - alg == pytest.approx(2.0 * 128 * M * N * 12)


def test_kernel_units_of_the_movers():
    N = W.chunk_tokens
    before = [W.capacity] * W.heads
    after = [_stats(100, 20, 80, W.capacity)] * W.heads
    row = 128 * 2
    assert bench.kernel_units(W, "aug_rows_kernel", N, before, after, 0, None) == \
        ("hbm", 12 * N * (row + 64), "candidates x (K row read + 64 B augmented row written)")
    bound, units, _ = bench.kernel_units(W, "gather_evicted_kernel", N, before, after, 0, None)
    assert bound == "hbm" and units == 12 * 100 * (2 * row + 128 + 4)
    bound, units, _ = bench.kernel_units(W, "finalize_kernel", N, before, after, 0, None)
    assert units == 12 * W.capacity * 24
    assert bench.kernel_units(W, "evict_select_kernel", N, before, after, 0, None)[0] == "latency"


def test_kernel_table_fractions():
    peaks = {"bf16_tflops": 1640.9, "hbm_gbs": 6441.9}
    records = [("gram_bf16_kernel", 0.1)] * 8 + [("compact_kernel", 0.02)] * 2
    units = {"gram_bf16_kernel": ("tensor", 1e11, "t"), "compact_kernel": ("hbm", 64e6, "b")}
    rows = {r["kernel"]: r for r in bench.kernel_table(W, records, 2, units, peaks)}
    g = rows["gram_bf16_kernel"]
    assert g["launches_per_step"] == 4 and g["ms_per_step"] == pytest.approx(0.4)
    assert g["achieved"] == pytest.approx(250.0) and g["frac"] == pytest.approx(250.0 / 1640.9, abs=1e-4)
    c = rows["compact_kernel"]
    assert c["achieved"] == pytest.approx(64e6 / 0.02e-3 / 1e9, rel=1e-3)       # 3200 GB/s
    assert c["frac"] == pytest.approx(3200 / 6441.9, abs=1e-4)
    assert g["share"] + c["share"] == pytest.approx(1.0, abs=1e-3)
