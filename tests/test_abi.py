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


def test_config_validation_and_workspace_sizes():
    """kvb_workspace_size: 0 for every invalid configuration; for valid ones it
    grows with the number of layers (per-layer banks) and with max_queries
    (attention scratch), and bf16 banks are smaller than f32 ones."""
    import kv_cache_compression_post_b200 as kvb
    ok = kvb.make_config()
    base = kvb.kvb_workspace_size(ok)
    assert base > 0
    bad = [dict(heads=65), dict(heads=0), dict(head_dim=96), dict(capacity=0), dict(max_candidates=0),
           dict(max_queries=0), dict(eps=0.0), dict(tau=0.0), dict(dist_scale=-1.0), dict(layers=0),
           dict(cand_order=2), dict(cand_order=-1), dict(baselines=2), dict(evict_order=3), dict(evict_order=-1)]
    for kw in bad:
        assert kvb.kvb_workspace_size(kvb.make_config(**kw)) == 0, kw
    # E4M3 storage: DensityKV banks of bf16 only; it halves the per-layer K/V storage
    for kw in [dict(storage=2), dict(storage=-1), dict(storage=kvb.KVB_STORE_FP8_E4M3, dtype=kvb.KVB_F32)]:
        assert kvb.kvb_workspace_size(kvb.make_config(**kw)) == 0, kw
    assert kvb.kvb_workspace_size(kvb.make_config(method=kvb.KVB_FORCINGKV, frame_h=30, frame_w=52,
                                                  storage=kvb.KVB_STORE_FP8_E4M3)) == 0
    L, H, M, N, d = 30, 12, 9360, 4680, 128
    native = kvb.kvb_workspace_size(kvb.make_config(layers=L))
    fp8 = kvb.kvb_workspace_size(kvb.make_config(layers=L, storage=kvb.KVB_STORE_FP8_E4M3))
    # per layer 2*H*M*d bytes less, plus one bf16 working layer and the rounded candidates
    assert abs((native - fp8) - (2 * L * H * M * d - 4 * H * M * d - 4 * H * N * d)) <= 4096
    # the ablation switches change no buffer
    for kw in [dict(cand_order=kvb.KVB_ORDER_SOURCE), dict(baselines=kvb.KVB_BASELINES_REFRESH),
               dict(evict_order=kvb.KVB_EVICT_DENSEST), dict(evict_order=kvb.KVB_EVICT_THRESHOLD_SOURCE)]:
        assert kvb.kvb_workspace_size(kvb.make_config(**kw)) == base, kw
    two = kvb.kvb_workspace_size(kvb.make_config(layers=2))
    three = kvb.kvb_workspace_size(kvb.make_config(layers=3))
    assert two > base and abs((three - two) - (two - base)) <= 4096   # one bank per layer (+ 256-byte alignment)
    assert kvb.kvb_workspace_size(kvb.make_config(max_queries=2 * 4680)) > base
    assert kvb.kvb_workspace_size(kvb.make_config(dtype=kvb.KVB_F32)) > base
    f = kvb.make_config(method=kvb.KVB_FORCINGKV, frame_h=30, frame_w=52)
    assert kvb.kvb_workspace_size(f) > 0
    for kw in [dict(frame_h=0), dict(seg_w=0), dict(hist_frames=0), dict(retention=1.5), dict(max_new_frames=0),
               dict(bottomk_scope=2), dict(bottomk_scope=-1), dict(sim_source=2),
               # the call scope ranks max_new_frames * n_seg <= 4096 pairs at once: 40 x 104 > 4096
               dict(bottomk_scope=kvb.KVB_BOTTOMK_CALL, max_new_frames=40)]:
        c = kvb.make_config(method=kvb.KVB_FORCINGKV, frame_h=30, frame_w=52)
        for k, v in kw.items():
            setattr(c, k, v)
        assert kvb.kvb_workspace_size(c) == 0, kw
    # the Forcing-KV variants change no buffer
    for kw in [dict(bottomk_scope=kvb.KVB_BOTTOMK_CALL), dict(sim_source=kvb.KVB_SIM_FIRST_LAYER),
               dict(bottomk_scope=kvb.KVB_BOTTOMK_CALL, max_new_frames=39)]:
        c = kvb.make_config(method=kvb.KVB_FORCINGKV, frame_h=30, frame_w=52, **kw)
        assert kvb.kvb_workspace_size(c) == kvb.kvb_workspace_size(
            kvb.make_config(method=kvb.KVB_FORCINGKV, frame_h=30, frame_w=52,
                            max_new_frames=kw.get("max_new_frames", 3))), kw


def test_entry_points_reject_bad_arguments_before_any_launch():
    """Null handles and malformed operation-level arguments return KVB_E_INVAL /
    KVB_E_UNSUPPORTED without touching the device."""
    import ctypes
    import kv_cache_compression_post_b200 as kvb
    lib = kvb.lib
    assert lib.kvb_admit(None, 0, None, None, None, 1, None) == 1
    assert lib.kvb_prune_hybrid(None, 0, None, None, None, None, None, 1, None) == 1
    assert lib.kvb_attend(None, 0, None, 1, None, None, 0, None, None, 0, None, None, None) == 1
    assert lib.kvb_bank_destroy(None) == 1
    n = ctypes.c_int32(0)
    assert lib.kvb_bank_export(None, 0, 0, None, None, None, None, None, ctypes.byref(n), None) == 1
    out = ctypes.c_void_p()
    assert lib.kvb_bank_create(None, None, 0, None, ctypes.byref(out)) == 1
    assert lib.kvb_bank_create(ctypes.byref(kvb.make_config()), ctypes.c_void_p(0x1001), 1 << 40, None,
                               ctypes.byref(out)) == 2                       # misaligned workspace
    # segment cosine: 16-byte rows and aligned pointers only
    sim = ctypes.c_void_p(0x2000)
    assert lib.kvb_segment_cosine(ctypes.c_void_p(0x1008), ctypes.c_void_p(0x3000), 1, 1, 4, 4, 4, 4, 128,
                                  kvb.KVB_BF16, sim, None) == 1              # K not 16-byte aligned
    assert lib.kvb_segment_cosine(ctypes.c_void_p(0x1000), ctypes.c_void_p(0x3000), 1, 1, 4, 4, 4, 4, 4,
                                  kvb.KVB_BF16, sim, None) == 7              # 8-byte rows
    assert lib.kvb_segment_cosine(None, ctypes.c_void_p(0x3000), 1, 1, 4, 4, 4, 4, 128, kvb.KVB_BF16, sim,
                                  None) == 1


def test_plain_c_program_agrees_with_the_binding(tmp_path):
    """include/kvb.h compiles as strict C99 in a plain C program linked against
    libkvb.so; the struct layouts it sees equal the ctypes mirror's, and the
    host-only entry points return the same values through both."""
    import ctypes
    import shutil
    import subprocess
    import kv_cache_compression_post_b200 as kvb
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(kvb.LIB_PATH)
    exe = str(tmp_path / "abi_layout")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_layout.c"), "-L", libdir, "-lkvb",
                    "-Wl,-rpath," + libdir, "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    for T in (kvb.kvb_config, kvb.kvb_admit_stats, kvb.kvb_trace_record):
        assert int(got["sizeof." + T.__name__]) == ctypes.sizeof(T), T.__name__
        for name, _ in T._fields_:
            assert int(got[f"{T.__name__}.{name}"]) == getattr(T, name).offset, (T.__name__, name)
    # every field the C program prints exists in the mirror
    mirrored = {f"{T.__name__}.{n}" for T in (kvb.kvb_config, kvb.kvb_admit_stats, kvb.kvb_trace_record)
                for n, _ in T._fields_}
    assert {k for k in got if "." in k and not k.startswith(("sizeof", "workspace", "status"))} == mirrored
    ref = kvb.make_config(heads=12, head_dim=128, capacity=9360, max_candidates=4680, max_queries=4680)
    assert int(got["workspace.wan480"]) == kvb.kvb_workspace_size(ref) > 0
    assert int(got["workspace.invalid"]) == 0
    assert got["status.0"] == kvb.kvb_status_string(0)


def test_selftest_timeout_argument_errors_without_gpu():
    import ctypes
    import kv_cache_compression_post_b200 as kvb
    fake = ctypes.c_void_p(256)   # never dereferenced: the checks return before any launch
    assert kvb.lib.kvb_selftest_timeout(None, fake, 1000, None) == 1
    assert kvb.lib.kvb_selftest_timeout(fake, None, 1000, None) == 1
    assert kvb.lib.kvb_selftest_timeout(fake, fake, 999, None) == 1
    assert kvb.lib.kvb_selftest_timeout(fake, fake, 100_000_001, None) == 1


def test_admit_halves_argument_errors_without_gpu():
    import ctypes
    import kv_cache_compression_post_b200 as kvb
    fake = ctypes.c_void_p(256)   # never dereferenced: the checks return before any launch
    assert kvb.lib.kvb_admit_begin(None, 0, fake, fake, fake, 10, fake, None) == 1    # no bank
    assert kvb.lib.kvb_admit_begin(fake, 0, fake, fake, fake, 10, None, None) == 1    # no prefix_out
    assert kvb.lib.kvb_admit_finish(None, 0, None, None) == 1


def test_plain_c_caller_of_the_whole_path_builds(tmp_path):
    """tests/c/c_user.c drives create / admit / attend / stats / status through
    the header alone; it compiles as strict C99 and links against libkvb.so and
    the CUDA runtime (running it needs a B200)."""
    import shutil
    import subprocess
    import kv_cache_compression_post_b200 as kvb
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if shutil.which("gcc") is None or not os.path.exists(os.path.join(cuda, "include", "cuda_runtime.h")):
        pytest.skip("no C compiler or CUDA headers")
    libdir = os.path.dirname(kvb.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "c_user.c"),
                    "-L", libdir, "-lkvb", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    "-Wl,-rpath," + libdir, "-o", str(tmp_path / "c_user")], check=True)
    assert os.path.getsize(tmp_path / "c_user") > 0


def test_pages_preset_is_a_valid_configuration():
    """sigma = 8, p = 2, eps = 1 in the library's parameters: h = 64, s = 2, eps = 1;
    phi of two keys at squared distance 64 is then exactly 1/2."""
    import numpy as np
    import kv_cache_compression_post_b200 as kvb
    from oracle.density import density
    pre = kvb.PAGES_PRESET
    assert kvb.kvb_workspace_size(kvb.make_config(**pre)) == kvb.kvb_workspace_size(kvb.make_config()) > 0
    a, b = np.zeros((1, 128)), np.zeros((1, 128))
    b[0, 0] = 8.0
    assert density(a, b, h=pre["dist_scale"], eps=pre["eps"], s=pre["s"])[0] == 0.5
