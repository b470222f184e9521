"""The parity suites, run once more against the index-checking debug build.

The debug build (``python -m bit_jl_key_b200.build --debug-index``, compiled
with -DJL_DEBUG_INDEX into libjlkey_debug.so) checks every global access its
kernels make through a raw pointer against the extent that the call's shapes
give that buffer; an access outside it is skipped and reported as
JL_DERR_INDEX through jl_device_error.  Every GPU test asserts at teardown
(tests/conftest.py) that jl_device_error() is 0, so a pass here means the small cases of every
kernel touched memory only inside the buffers they were given, and still
matched the oracle.  (Tensor-map copies are bounded by the hardware against
their maps and need no software check.)  The full-size cases are left out.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

SUITES = ["tests/test_gpu_parity.py", "tests/test_gpu_paged.py", "tests/test_gpu_dequant.py",
          "tests/test_gpu_search.py", "tests/test_gpu_turbo.py", "tests/test_gpu_turbo_paged.py",
          "tests/test_gpu_turbo_dequant.py", "tests/test_gpu_context_parallel.py"]


def test_parity_suites_pass_under_index_checks():
    from bit_jl_key_b200 import build
    lib = build.build(debug_index=True)
    env = dict(os.environ, JLKEY_LIBRARY=lib)
    probe = subprocess.run(
        [sys.executable, "-c", "import bit_jl_key_b200 as jl; print(jl.LIB_PATH, jl.jl_build_flags())"],
        env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert probe.returncode == 0, probe.stderr
    path, flags = probe.stdout.split()
    assert os.path.samefile(path, lib) and int(flags) == 1
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
         *SUITES, "-k", "not fullsize and not full_size and not sampled and not nccl"],
        env=env, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    print(r.stdout[-1500:])
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
