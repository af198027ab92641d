"""GPU parity of the Soft-Riesz density Gram (tcgen05 bf16 path and fp32 path)
against the fp64 oracle (DensityKV §3 "Soft-Riesz Density").  Bar: 1e-4 relative."""
import numpy as np
import pytest

import kvgen
from oracle.density import density
from tests.gpu_util import aligned_ptr, dev_tensor, host, workspace

pytestmark = pytest.mark.gpu

RTOL = 1e-4


def _run(rows, cols, dtype, h=0.0, eps=1e-3, s=2.0, diag=0):
    import torch
    import kv_cache_compression_post_b200 as kvb
    H, nR, d = rows.shape
    nC = cols.shape[1]
    R = dev_tensor(rows, dtype)
    C = dev_tensor(cols, dtype) if nC else R
    out = torch.full((H, nR), float("nan"), device="cuda")
    dt = kvb.KVB_BF16 if dtype == "bf16" else kvb.KVB_F32
    nb = kvb.kvb_density_workspace_size(H, nR, nC, d, dt)
    ws = workspace(nb)
    kvb.kvb_density(R, nR, C, nC, H, d, dt, h, eps, s, diag, out, aligned_ptr(ws), nb)
    torch.cuda.synchronize()
    st = ws[aligned_ptr(ws) - ws.data_ptr():][:4].view(torch.int32).item()
    assert st == 0, f"device status {st}"
    return host(out)


def _oracle(rows, cols, h, eps, s, diag):
    out = []
    for hh in range(rows.shape[0]):
        ids = np.arange(rows.shape[1]) if diag else None
        out.append(density(rows[hh], cols[hh], h=h or rows.shape[-1], eps=eps, s=s, row_ids=ids,
                           col_ids=ids if diag else None))
    return np.array(out)


def _keys(H, n, d, seed, a=0.9):
    """AR(1)-correlated keys like the generator's (close pairs exist)."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((H, 1, d)).astype(np.float32)
    x = a * base + 0.44 * rng.standard_normal((H, n, d)).astype(np.float32)
    return kvgen.round_bf16(x)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("nR,nC", [(300, 700), (128, 128), (1, 5), (513, 129)])
def test_density_bf16_ragged(d, nR, nC):
    rows = _keys(3, nR, d, 1)
    cols = _keys(3, nC, d, 2)
    got = _run(rows, cols, "bf16")
    np.testing.assert_allclose(got, _oracle(rows, cols, 0, 1e-3, 2.0, False), rtol=RTOL)


@pytest.mark.parametrize("s", [1.0, 3.0, 2.0])
def test_density_bf16_exponents_and_scale(s):
    rows = _keys(2, 260, 128, 3)
    cols = _keys(2, 390, 128, 4)
    got = _run(rows, cols, "bf16", h=64.0, eps=0.5, s=s)
    np.testing.assert_allclose(got, _oracle(rows, cols, 64.0, 0.5, s, False), rtol=RTOL)


def test_density_bf16_pages_preset():
    """The pages' sigma / eps / p preset (h = sigma^2 = 64, eps = 1, s = p = 2)."""
    import kv_cache_compression_post_b200 as kvb
    pp = kvb.PAGES_PRESET
    rows = _keys(2, 260, 128, 7)
    cols = _keys(2, 390, 128, 8)
    got = _run(rows, cols, "bf16", h=pp["dist_scale"], eps=pp["eps"], s=pp["s"])
    np.testing.assert_allclose(got, _oracle(rows, cols, pp["dist_scale"], pp["eps"], pp["s"], False), rtol=RTOL)
    got = _run(rows, rows, "bf16", h=pp["dist_scale"], eps=pp["eps"], s=pp["s"], diag=1)
    np.testing.assert_allclose(got, _oracle(rows, rows, pp["dist_scale"], pp["eps"], pp["s"], True), rtol=RTOL)


def test_density_bf16_exclude_diagonal():
    rows = _keys(4, 700, 128, 5)
    got = _run(rows, rows, "bf16", diag=1)
    np.testing.assert_allclose(got, _oracle(rows, rows, 0, 1e-3, 2.0, True), rtol=RTOL)


def test_density_f32():
    rng = np.random.default_rng(6)
    rows = rng.standard_normal((2, 192, 64)).astype(np.float32)
    cols = rng.standard_normal((2, 384, 64)).astype(np.float32)
    got = _run(rows, cols, "f32")
    np.testing.assert_allclose(got, _oracle(rows, cols, 0, 1e-3, 2.0, False), rtol=RTOL)
    got = _run(rows, rows, "f32", diag=1)
    np.testing.assert_allclose(got, _oracle(rows, rows, 0, 1e-3, 2.0, True), rtol=RTOL)


def test_density_empty_columns():
    rows = _keys(2, 100, 128, 7)
    got = _run(rows, np.zeros((2, 0, 128), np.float32), "bf16")
    np.testing.assert_array_equal(got, 0.0)


def test_density_full_size_sampled():
    """480P shapes: 12 heads, 4680 candidates x 9360 bank keys, rows sampled."""
    H, N, M, d = 12, 4680, 9360, 128
    rows = _keys(H, N, d, 8)
    cols = _keys(H, M, d, 9)
    got = _run(rows, cols, "bf16")
    rng = np.random.default_rng(0)
    for hh in range(H):
        idx = np.sort(rng.choice(N, 24, replace=False))
        ref = density(rows[hh][idx], cols[hh], h=d, eps=1e-3, s=2.0)
        np.testing.assert_allclose(got[hh][idx], ref, rtol=RTOL)
