"""CPU: bench.py's FP8 reference helper gives exactly the oracle's dequantized values."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fp8_values_equal_the_oracle_dequantization():
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    oracle.build()
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(3000, 4, 32, generator=g) * 3).to(torch.bfloat16)
    scales = np.array([6.0 / 448, 0.02, 1.0, 256.0], dtype=np.float32)  # normal, subnormal and saturated codes
    got = bench.fp8_values(oracle, x, scales)
    for h in range(4):
        ref = oracle.e4m3_dequantize(oracle.e4m3_quantize(x[:, h].contiguous(), float(scales[h])), float(scales[h]))
        assert np.array_equal(got[:, h], ref)
