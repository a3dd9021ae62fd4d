"""GPU: the tcgen05 FP8 decode kernel (decode_tc_kernel), a run-time alternative to decode_kernel
for FP8 pools with head_dim 128 (environment variable HSWA_DECODE_TC = 2 sends every layer to
it). The library reads the variable once per process, so the FP8 decode cases run in a child
pytest with it set; they compare against the fp64 oracle on the dequantized entries (ring and
paged layers, split boundaries and merges, the config-4 head shape, all-subnormal codes)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_fp8_decode_cases_through_the_tcgen05_kernel():
    env = dict(os.environ, HSWA_DECODE_TC="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_gpu_fp8.py"), "-q", "-x",
                        "-k", "decode", "-p", "no:cacheprovider"],
                       env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
