"""GPU: the narrow-window prefill path (1 <= W <= 129: a query tile's band spans at most two key
tiles, which stay resident while the query heads of one KV head pass through two slots).

Cases the other prefill tests do not reach: an odd number of query heads per KV head (slot 1
gets one head fewer), one query head per KV head (slot 1 idle), a window so small that whole
warps have no key in the previous tile, the largest window on this path with an aligned ring
prefix, and several units per CTA with mixed prefixes.
"""
import pytest

from hswa_testlib import compare
from test_gpu_prefill import run_swa_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_q,W,hq,hkv,d,starts", [
    (300, 128, 3, 1, 128, [131, 0]),     # G = 3: slots take heads {0, 2} and {1}
    (257, 64, 2, 2, 64, [0, 200]),       # G = 1: slot 1 idle; rows >= 64 of a tile see nothing in tile t-1
    (384, 129, 10, 2, 128, [256, 640]),  # W = 129 (largest narrow window), prefix rows by cp.async
    (130, 2, 8, 1, 64, [5, 0]),          # W = 2, G = 8, a 2-row tail tile
    (1000, 128, 8, 1, 128, [0, 131072]), # many units, prefix far into the sequence
    (300, 128, 8, 2, 128, [126, 127]),   # W = 128 at the rotated-mask boundary (first row 126 / 127)
    (300, 128, 4, 1, 64, [128, 255]),    # rotated mask with an aligned and an unaligned ring prefix
])
def test_narrow_window_cases(n_q, W, hq, hkv, d, starts):
    got, ref = run_swa_case(107, 2, n_q, W, hq, hkv, d, starts)
    compare(got, ref, f"n_q={n_q} W={W} hq={hq} hkv={hkv}")
