"""The bounds-checked library, libdf11_check.so: the same C-ABI with the
kernels compiled with -DDF11_CHECK=1, so that every decode-table, stage,
exponent-buffer and look-ahead index and every read of a container section
(stream, gaps, chunk counts, out_off, plane) and write of the output is
checked against its bound.  An access outside is skipped and
DF11_DEV_ERR_BOUNDS is set in the launch's error word; nothing traps.

The small-case GPU suites (decode, GPU encode, the decode fused into the
GEMM, the rANS decode) run against it in a child process (the binding picks
its library once, at import, from DF11_LIBRARY).  Their parity tests demand an error word of 0,
their corruption tests demand no DF11_DEV_ERR_BOUNDS, and
test_bounds_checks_are_live demands that a bound made 0 bytes is reported."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_gpu_decode.py", "tests/test_gpu_encode.py", "tests/test_gpu_gemm.py", "tests/test_gpu_rans.py"]


@pytest.fixture(scope="module")
def check_env():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from entropy_decoding_b200 import build
    build.build()
    build.build(check=True)
    return dict(os.environ, DF11_LIBRARY="check")


def test_child_loads_the_check_library(check_env):
    code = ("from entropy_decoding_b200 import df11\n"
            "assert df11.CHECKED and df11.LIB_PATH.endswith('libdf11_check.so')\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libdf11_check.so' in maps and '/libdf11.so' not in maps\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=check_env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]


def test_small_suites_under_bounds_checks(check_env):
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu and not slow", *SUITES]
    r = subprocess.run(cmd, cwd=ROOT, env=check_env, capture_output=True, text=True, timeout=3000)
    assert r.returncode == 0, r.stdout[-6000:] + r.stderr[-3000:]
    assert " passed" in r.stdout
