"""Seeded, counter-based synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no attention arithmetic. It only turns (seed, stream, index)
triples into bf16 values, so that any row of any tensor can be regenerated on
its own, on the CPU or on the GPU, and the two devices agree bit for bit.

Recipe
------
* 64-bit counter hash: the SplitMix64 output function (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014; the constants
  are the ones published with Vigna's public-domain splitmix64). A draw is
  ``mix64(key + (i + 1) * GAMMA)`` with ``key = mix64(seed ^ mix64(stream + GAMMA))``.
* The top 32 bits of a draw are a uniform integer ``u`` in [0, 2**32).
* ``u`` is mapped to a bf16 value by inverse-CDF table lookup: the table lists
  every bf16 value ``v_k`` that a real N(0, sigma^2) sample rounds to (round to
  nearest even) with non-zero probability at 2**-32 resolution, and the
  threshold between ``v_k`` and ``v_{k+1}`` is ``round(Phi(m_k / sigma) * 2**32)``
  with ``m_k`` the midpoint of the two values.  The result is "a normal sample
  rounded to bf16", with bin probabilities quantised to 2**-32.

Every step is integer arithmetic or an exact table lookup, so
``torch`` on the CPU and on CUDA produce identical bits.
"""
from __future__ import annotations

import math
from functools import lru_cache

import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB

# stream tags (the first word of a stream id)
TAG_Q = 1
TAG_K = 2
TAG_V = 3
TAG_K_NEW = 4
TAG_V_NEW = 5
TAG_MISC = 9


def _s64(x: int) -> int:
    """uint64 -> the int64 with the same bits."""
    x &= MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def mix64_int(z: int) -> int:
    """SplitMix64 output mix on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * _M1) & MASK64
    z = ((z ^ (z >> 27)) * _M2) & MASK64
    return z ^ (z >> 31)


def stream_id(tag: int, *parts: int) -> int:
    """Fold a tag and integers (layer, sequence, ...) into one 64-bit stream id."""
    h = mix64_int(tag + GAMMA)
    for p in parts:
        h = mix64_int((h ^ (p & MASK64)) + GAMMA)
    return h


def stream_key(seed: int, stream: int) -> int:
    return mix64_int((seed & MASK64) ^ mix64_int(stream + GAMMA))


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 tensors holding uint64 bits."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix64_t(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def uniform_u32(key: int, index: torch.Tensor) -> torch.Tensor:
    """Top 32 bits of draw ``index`` of the stream with this key (int64 tensor)."""
    z = index.to(torch.int64) * _s64(GAMMA) + _s64(key + GAMMA)
    z = _mix64_t(z)
    return _lsr(z, 32)


def _bf16_bits_to_float(bits: int) -> float:
    import struct
    return struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]


@lru_cache(maxsize=None)
def normal_table(sigma: float):
    """(thresholds int64[n-1], values bf16-bits int16[n]) for N(0, sigma^2) rounded to bf16.

    Values are enumerated in increasing order over all finite bf16 numbers with
    |v| <= 9 sigma; a value keeps a bin only if its quantised probability is
    non-zero. A uniform u selects values[#thresholds <= u].
    """
    vals = []
    # negative values: bits 0x8000|e (descending magnitude), zero, positive ascending
    pos = []
    for b in range(0x0000, 0x7F80):  # finite non-negative bf16 (0 .. max finite)
        x = _bf16_bits_to_float(b)
        if x > 9.0 * sigma:
            break
        pos.append((x, b))
    neg = [(-x, b | 0x8000) for (x, b) in reversed(pos) if b != 0]
    vals = neg + pos
    two32 = float(1 << 32)
    thr = []
    for k in range(len(vals) - 1):
        mid = 0.5 * (vals[k][0] + vals[k + 1][0])
        phi = 0.5 * math.erfc(-mid / (sigma * math.sqrt(2.0)))
        thr.append(int(round(phi * two32)))
    # keep value k iff its bin [thr[k-1], thr[k]) is non-empty (thr[-1] = 0, thr[n-1] = 2**32)
    full = [0] + thr + [1 << 32]
    kept_vals = []
    kept_thr = []
    for k in range(len(vals)):
        if full[k + 1] > full[k]:
            kept_vals.append(vals[k][1])
            kept_thr.append(full[k + 1])
    kept_thr = kept_thr[:-1]  # the last upper edge is 2**32
    t = torch.tensor(kept_thr, dtype=torch.int64)
    v = torch.tensor([b - 0x10000 if b >= 0x8000 else b for b in kept_vals], dtype=torch.int16)
    return t, v


_DEV_TABLES: dict = {}


def _table_on(sigma: float, device: torch.device):
    key = (sigma, str(device))
    if key not in _DEV_TABLES:
        t, v = normal_table(sigma)
        _DEV_TABLES[key] = (t.to(device), v.to(device))
    return _DEV_TABLES[key]


_FAST = None


def _fast_lib():
    """The C build of the same generator (CPU only); None if gcc is unavailable."""
    global _FAST
    if _FAST is None:
        import ctypes
        import os
        import subprocess
        here = os.path.dirname(os.path.abspath(__file__))
        src, lib = os.path.join(here, "fastgen.c"), os.path.join(here, "libfastgen.so")
        try:
            if not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
                tmp = lib + f".tmp{os.getpid()}"
                subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, src])
                os.replace(tmp, lib)
            L = ctypes.CDLL(lib)
            L.fastgen_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                              ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            L.fastgen_normal_bf16.restype = ctypes.c_int
            _FAST = L
        except Exception:  # pragma: no cover - torch path below still works
            _FAST = False
    return _FAST or None


def normal_bf16(seed: int, stream: int, start: int, count: int, sigma: float = 1.0,
                device="cpu", chunk: int = 1 << 26, use_c: bool = True) -> torch.Tensor:
    """``count`` bf16 values: draws ``start .. start+count-1`` of (seed, stream), N(0, sigma^2)."""
    device = torch.device(device)
    key = stream_key(seed, stream)
    if device.type == "cpu" and use_c and count >= 4096 and _fast_lib() is not None:
        import os
        thr, val = normal_table(float(sigma))
        out = torch.empty(count, dtype=torch.int16)
        _fast_lib().fastgen_normal_bf16(key, start, count, thr.data_ptr(), thr.numel(), val.data_ptr(),
                                        out.data_ptr(), os.cpu_count() or 1)
        return out.view(torch.bfloat16)
    thr, val = _table_on(float(sigma), device)
    out = torch.empty(count, dtype=torch.int16, device=device)
    for c0 in range(0, count, chunk):
        n = min(chunk, count - c0)
        idx = torch.arange(start + c0, start + c0 + n, dtype=torch.int64, device=device)
        u = uniform_u32(key, idx)
        sel = torch.searchsorted(thr, u, right=True)
        out[c0:c0 + n] = val[sel]
        del idx, u, sel
    return out.view(torch.bfloat16)


def normal_bf16_rows(seed: int, stream: int, row_start: int, n_rows: int, row_elems: int,
                     sigma: float = 1.0, device="cpu") -> torch.Tensor:
    """Rows ``row_start .. row_start+n_rows-1`` of a logical [rows][row_elems] tensor."""
    x = normal_bf16(seed, stream, row_start * row_elems, n_rows * row_elems, sigma, device)
    return x.view(n_rows, row_elems)


def uniform_int(seed: int, stream: int, count: int, lo: int, hi: int, device="cpu") -> torch.Tensor:
    """Integers uniform in [lo, hi] (inclusive) via 32-bit draws and a multiply-shift."""
    key = stream_key(seed, stream)
    idx = torch.arange(count, dtype=torch.int64, device=device)
    u = uniform_u32(key, idx)
    span = hi - lo + 1
    assert 0 < span <= (1 << 31)
    return lo + ((u * span) >> 32)


def uniform_float64(seed: int, stream: int, count: int, device="cpu") -> torch.Tensor:
    """Doubles in [0, 1) with 32-bit resolution (for host-side workload shapes)."""
    key = stream_key(seed, stream)
    idx = torch.arange(count, dtype=torch.int64, device=device)
    return uniform_u32(key, idx).to(torch.float64) / float(1 << 32)


def permutation(seed: int, stream: int, n: int) -> torch.Tensor:
    """A seeded permutation of 0..n-1 (argsort of distinct 64-bit draws), on the CPU."""
    key = stream_key(seed, stream)
    idx = torch.arange(n, dtype=torch.int64)
    z = _mix64_t(idx * _s64(GAMMA) + _s64(key + GAMMA))
    # order by the draw, ties (impossible in practice) broken by index
    return torch.argsort(z, stable=True)
