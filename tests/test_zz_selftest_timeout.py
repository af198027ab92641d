"""The device-side failure detection, exercised without a fault: the library's
bounded mbarrier wait runs to expiry on a barrier nothing arrives on, latches
KVB_E_DEVICE_TIMEOUT, and its abort flag makes the CTA's other role give up its
own (longer) wait; the context stays usable afterwards."""
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_aborts_the_other_role():
    import torch
    import kv_cache_compression_post_b200 as kvb
    limit = 20_000_000   # 20 ms; role 1's own limit is 50x, 1 s
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((4,), -1, dtype=torch.int64, device="cuda")
    kvb.kvb_selftest_timeout(status, out, limit)
    torch.cuda.synchronize()
    assert int(status.item()) == 4                      # KVB_E_DEVICE_TIMEOUT
    done0, ns0, done1, ns1 = out.cpu().tolist()
    assert done0 == 0 and done1 == 0                    # neither barrier ever completed
    assert limit <= ns0 < 10 * limit                    # role 0 gave up at its limit
    assert ns1 < 25 * limit                             # role 1 left through the abort flag, not its 1 s limit
    # the context is intact: ordinary work and a library call still run
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 1023 * 1024 / 2
    status.zero_()
    out.fill_(-1)
    kvb.kvb_selftest_timeout(status, out, 1000)
    torch.cuda.synchronize()
    assert int(status.item()) == 4 and out.cpu().tolist()[0] == 0
