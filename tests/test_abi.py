"""The C-ABI library loads and exports every entry point include/kvb.h declares;
host-side argument checks return errors before anything is launched (no GPU)."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kvb.h")).read()
    return sorted(set(re.findall(r"^KVB_API\s+[\w\s\*]+?\b(kvb_\w+)\(", src, flags=re.M)))


def test_header_declares_entry_points():
    names = _declared()
    for n in ["kvb_bank_create", "kvb_admit", "kvb_prune_hybrid", "kvb_attend", "kvb_density"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    import ctypes
    import kv_cache_compression_post_b200 as kvb
    lib = ctypes.CDLL(kvb.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    import kv_cache_compression_post_b200 as kvb
    assert kvb.kvb_status_string(0) == "ok"
    assert "timed out" in kvb.kvb_status_string(4)
    assert kvb.kvb_status_string(99) == "unknown status"


def test_density_argument_errors_without_gpu():
    import kv_cache_compression_post_b200 as kvb
    assert kvb.kvb_density_workspace_size(0, 10, 10, 128, 0) == 0
    assert kvb.kvb_density_workspace_size(12, 4680, 9360, 128, 0) > 0
    with pytest.raises(kvb.KvbError) as e:
        kvb.kvb_density(0, 10, 0, 10, 0, 128, 0, 0.0, 1e-3, 2.0, 0, 0, 0, 0, stream=0)
    assert e.value.status == 1
    with pytest.raises(kvb.KvbError) as e:   # head_dim 96 is not a tensor-core shape here
        kvb.kvb_density(1, 10, 1, 10, 2, 96, 0, 0.0, 1e-3, 2.0, 0, 1, 256, 1 << 20, stream=0)
    assert e.value.status == 7
    with pytest.raises(kvb.KvbError) as e:   # eps must be > 0
        kvb.kvb_density(1, 10, 1, 10, 2, 128, 0, 0.0, 0.0, 2.0, 0, 1, 256, 1 << 20, stream=0)
    assert e.value.status == 1
    with pytest.raises(kvb.KvbError) as e:   # misaligned workspace
        kvb.kvb_density(1, 10, 1, 10, 2, 128, 0, 0.0, 1e-3, 2.0, 0, 1, 257, 1 << 20, stream=0)
    assert e.value.status == 2


def test_launch_trace_host_side():
    import ctypes
    import kv_cache_compression_post_b200 as kvb
    kvb.kvb_trace_enable(True)
    assert kvb.kvb_trace_read() == []          # nothing launched
    kvb.kvb_trace_enable(False)
    n = ctypes.c_int32(0)
    assert kvb.lib.kvb_trace_read(None, 0, ctypes.byref(n)) == 0 and n.value == 0
    assert kvb.lib.kvb_trace_read(None, 4, ctypes.byref(n)) == 1   # out NULL with max_records > 0
    assert kvb.lib.kvb_trace_read(None, 0, None) == 1              # n_out NULL
