"""CPU pins of the oracle's FP8 E4M3 functions (the storage format of an FP8 KV cache).

The format is the OCP 8-bit floating point E4M3 ("MiMo v2.5 inference optimisation", closing
section: quantization cuts the bits of each cached entry and stacks with the sliding window's
cut in entries). The oracle's decode and encode are pinned against the values the format
states (largest finite 448, smallest normal 2^-6, smallest subnormal 2^-9, S.1111.111 the only
NaN, no infinities), against torch's independent float8_e4m3fn conversion on all 256 codes and
on random values inside the finite range, and against the round-to-nearest-even and saturation
rules on every midpoint and beyond the range. The fp64-key attention entry is pinned to the
bf16 one, which the attention pins cover.
"""
import math

import numpy as np
import torch

import oracle


def test_stated_values_of_the_format():
    d = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0          # largest finite magnitude 1.75 * 2^8
    assert d[0x08] == 2.0 ** -6                             # smallest normal
    assert d[0x07] == 0.875 * 2.0 ** -6                     # largest subnormal
    assert d[0x01] == 2.0 ** -9                             # smallest subnormal
    assert d[0x38] == 1.0                                   # exponent field 7 = bias
    assert d[0x00] == 0.0 and not math.copysign(1, d[0x00]) < 0
    assert d[0x80] == 0.0 and math.copysign(1, d[0x80]) < 0
    nan = np.isnan(d)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]         # S.1111.111 only; no infinities
    assert np.isfinite(d[~nan]).all() and (~nan).sum() == 254
    assert (np.diff(d[:0x7F]) > 0).all()                    # positive codes increase with the code
    assert np.array_equal(d[0x80:0xFF], -d[0x00:0x7F])      # the sign bit mirrors


def test_decode_equals_torch_float8_e4m3fn_on_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes.numpy())
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_encode_round_trip_midpoints_and_saturation():
    vals = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = [c for c in range(256) if not np.isnan(vals[c])]
    assert all(int(oracle.e4m3_encode(vals[c])) == c for c in finite)
    # midpoints between neighbouring positive values go to the code with the even mantissa
    pos = [c for c in range(0x7F)]
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (vals[a] + vals[b]) / 2
        want = a if a % 2 == 0 else b
        assert int(oracle.e4m3_encode(mid)) == want, (a, b)
        assert int(oracle.e4m3_encode(-mid)) == want | 0x80
        assert int(oracle.e4m3_encode(np.nextafter(mid, 0))) == a
        assert int(oracle.e4m3_encode(np.nextafter(mid, np.inf))) == b
    # beyond the largest finite value: saturate to +-448, never NaN
    for x in (448.0, 463.9, 464.0, 470.0, 1e4, 1e30):
        assert int(oracle.e4m3_encode(x)) == 0x7E and int(oracle.e4m3_encode(-x)) == 0xFE
    assert int(oracle.e4m3_encode(float("nan"))) == 0x7F


def test_encode_equals_torch_inside_the_finite_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 50, 2000), rng.normal(0, 0.01, 2000),
                        rng.uniform(-463.9, 463.9, 2000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x.astype(np.float64)), ref)


def test_quantize_is_encode_of_the_fp32_product_with_the_fp32_reciprocal():
    rng = np.random.default_rng(6)
    x = torch.from_numpy(rng.normal(0, 3, 5000).astype(np.float32)).to(torch.bfloat16)
    for scale in (1.0, 0.0625, 0.37, 3.0):
        inv = np.float32(1.0) / np.float32(scale)
        prod = x.float().numpy() * inv  # fp32 product
        want = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(oracle.e4m3_quantize(x, scale), want)
        deq = oracle.e4m3_dequantize(oracle.e4m3_quantize(x, scale), scale)
        assert np.all(np.abs(deq - x.double().numpy()) <= np.maximum(np.abs(x.double().numpy()) / 16, 2.0 ** -10 * scale))


def test_fp64_kv_attention_equals_the_bf16_entry_on_bf16_values():
    rng = np.random.default_rng(7)
    q = torch.from_numpy(rng.normal(0, 1, (9, 4, 32)).astype(np.float32)).to(torch.bfloat16)
    k = torch.from_numpy(rng.normal(0, 1, (40, 2, 32)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.normal(0, 1, (40, 2, 32)).astype(np.float32)).to(torch.bfloat16)
    pos = np.arange(31, 40)
    for window in (0, 5, 17):
        a = oracle.attention(q, pos, k, v, window)
        b = oracle.attention_kv64(q, pos, k.double().numpy(), v.double().numpy(), window)
        assert np.array_equal(a, b)
