"""The FMA-pipe exponential used by the prefill softmax, emulated step by step in float32
(numpy) and compared with float64 exp2 over the range the kernel feeds it (x <= 8)."""
import numpy as np

C3, C2, C1, C0 = (np.float32(0.05583828315138817), np.float32(0.2426394820213318),
                  np.float32(0.6931367516517639), np.float32(0.9999245405197144))


def exp2_poly(x):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (C3 * f + C2).astype(np.float32)
    p = (p * f + C1).astype(np.float32)
    p = (p * f + C0).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-120, 8, 2_000_001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, -1.0, 7.99, -119.5], np.float32)])
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1)
    assert rel.max() < 1.1e-4


def test_clamped_tail_is_negligible():
    x = np.array([-np.inf, -1e30, -200.0, -126.0], np.float32)
    got = exp2_poly(x)
    assert np.all(got > 0) and np.all(got < 1e-37)
