"""The plain C99 caller (tests/c/c_user.c) of the whole DensityKV path, built
against include/kvb.h and libkvb.so and run on the GPU: create, admit, attend,
counters, device status, destroy, with no Python in the process.  Its inputs are
zeros, so the result is known in closed form: the bank starts empty, every
candidate is feasible with score 0, and each head admits min(N, M) = 256 of its
256 candidates."""
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plain_c_caller_runs_the_path(tmp_path):
    import kv_cache_compression_post_b200 as kvb
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(kvb.LIB_PATH)
    exe = str(tmp_path / "c_user")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "c_user.c"),
                    "-L", libdir, "-lkvb", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    "-Wl,-rpath," + libdir, "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("head ")]
    assert lines == ["head 0: admitted 256, bank size 256", "head 1: admitted 256, bank size 256"], r.stdout
