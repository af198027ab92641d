"""kvb_density_noalloc: the density entry point for callers that cannot allocate
device memory (a host application whose allocator owns all device memory, or a
loop that must never pay for an allocation), so cannot pass a scratch workspace.
Its scratch is a fixed array inside the library; the results must equal those of
kvb_density (which uses a caller workspace), call after call."""
import numpy as np
import pytest

import kvgen
from oracle.density import density
from tests.gpu_util import aligned_ptr, dev_tensor, host, workspace

pytestmark = pytest.mark.gpu

RTOL = 1e-4


def _keys(H, n, d, seed):
    rng = np.random.default_rng(seed)
    base = rng.standard_normal((H, 1, d)).astype(np.float32)
    return kvgen.round_bf16(0.9 * base + 0.44 * rng.standard_normal((H, n, d)).astype(np.float32))


def _with_workspace(R, C, H, nR, nC, d, diag):
    import torch
    import kv_cache_compression_post_b200 as kvb
    out = torch.full((H, nR), float("nan"), device="cuda")
    nb = kvb.kvb_density_workspace_size(H, nR, nC, d, kvb.KVB_BF16)
    ws = workspace(nb)
    kvb.kvb_density(R, nR, C, nC, H, d, kvb.KVB_BF16, 0.0, 1e-3, 2.0, diag, out, aligned_ptr(ws), nb)
    return out


def _without(R, C, H, nR, nC, d, diag, with_status=True):
    import torch
    import kv_cache_compression_post_b200 as kvb
    out = torch.full((H, nR), float("nan"), device="cuda")
    st = torch.full((1,), -7, dtype=torch.int32, device="cuda") if with_status else None
    kvb.kvb_density_noalloc(R, nR, C, nC, H, d, kvb.KVB_BF16, 0.0, 1e-3, 2.0, diag, out, st)
    torch.cuda.synchronize()
    if with_status:
        assert int(st.item()) == 0
    return out


def _oracle(rows, cols, diag, sample=None):
    """oracle.density (fp64 direct differences) of every head's rows, or of the
    row indices in `sample`, against all columns."""
    H, nR, d = rows.shape
    idx = np.arange(nR) if sample is None else np.asarray(sample)
    out = []
    for h in range(H):
        ids = np.arange(nR) if diag else None
        out.append(density(rows[h][idx], cols[h], h=float(d), eps=1e-3, s=2.0,
                           row_ids=None if ids is None else ids[idx], col_ids=ids))
    return np.stack(out)


@pytest.mark.parametrize("diag", [0, 1])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(diag):
    H, d = 3, 128
    shapes = [(300, 700), (513, 129)] if not diag else [(300, 300), (700, 700)]
    for seed, (nR, nC) in enumerate(shapes):          # two calls in a row, different sizes and data
        rows = _keys(H, nR, d, 10 + seed)
        cols = rows if diag else _keys(H, nC, d, 20 + seed)
        R, C = dev_tensor(rows, "bf16"), dev_tensor(cols, "bf16")
        ref = host(_with_workspace(R, C, H, nR, nC, d, diag))
        got = host(_without(R, C, H, nR, nC, d, diag))
        np.testing.assert_allclose(got, ref, rtol=RTOL)
        np.testing.assert_allclose(got, _oracle(rows, cols, diag), rtol=RTOL)


def test_noalloc_without_a_status_word():
    """status_out NULL: the call still computes the same densities."""
    H, nR, nC, d = 2, 257, 300, 128
    rows, cols = _keys(H, nR, d, 31), _keys(H, nC, d, 32)
    R, C = dev_tensor(rows, "bf16"), dev_tensor(cols, "bf16")
    got = host(_without(R, C, H, nR, nC, d, 0, with_status=False))
    np.testing.assert_allclose(got, _oracle(rows, cols, 0), rtol=RTOL)


def test_noalloc_largest_size_that_fits_and_the_next():
    """The documented limit: 256 + 64*H*n_rows + 64*H*n_cols + 64*H*n_rows bytes
    (each term rounded up to 256) <= 4 MiB.  With H = 1 and n_rows = n_cols = n
    (a multiple of 4) that is 256 + 192 n <= 4194304, so n = 21844 fills the array
    exactly and runs (checked on sampled rows against the oracle), and n = 21845
    (terms rounded up to 1398272 bytes: 4195072 in all) is rejected."""
    import torch
    import kv_cache_compression_post_b200 as kvb
    H, d, n = 1, 128, 21844
    rows = _keys(H, n, d, 41)
    cols = _keys(H, n, d, 42)
    R, C = dev_tensor(rows, "bf16"), dev_tensor(cols, "bf16")
    got = host(_without(R, C, H, n, n, d, 0))
    smp = np.random.default_rng(5).choice(n, 24, replace=False)
    np.testing.assert_allclose(got[:, smp], _oracle(rows, cols, 0, smp), rtol=RTOL)
    before = kvb.kvb_launch_count()
    with pytest.raises(kvb.KvbError) as e:
        kvb.kvb_density_noalloc(R, n + 1, C, n + 1, H, d, kvb.KVB_BF16, 0.0, 1e-3, 2.0, 0, 1, None,
                                torch.cuda.current_stream())
    assert e.value.status == 2
    assert kvb.kvb_launch_count() == before


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    import kv_cache_compression_post_b200 as kvb
    H, nR, nC, d = 12, 9360, 4680, 128   # the two row terms alone need 2*64*H*nR bytes > 4 MiB
    before = kvb.kvb_launch_count()
    with pytest.raises(kvb.KvbError) as e:
        kvb.kvb_density_noalloc(1, nR, 1, nC, H, d, kvb.KVB_BF16, 0.0, 1e-3, 2.0, 0, 1, None,
                                torch.cuda.current_stream())
    assert e.value.status == 2
    assert kvb.kvb_launch_count() == before
