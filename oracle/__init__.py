"""fp64 CPU oracle for hybrid sliding-window attention (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` and
``--impl reference`` legs of ``bench.py`` may import this package. The product
path (``hybrid_sliding_window_swa_b200``) never imports it and shares no code
with it. The arithmetic lives in ``oracle.c`` (plain C, fp64); this module only
builds it with gcc and marshals numpy/torch arrays through ctypes, except for
``prefix_cache_replay``, a brute-force integer model written out in Python.

Every function here restates a passage of the source pages; see ``oracle.h``
for the citations and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (host code only)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.orc_mask_count.restype = i64
        L.orc_mask_count.argtypes = [i64, i64]
        L.orc_attention.restype = i32
        L.orc_attention.argtypes = [p, p, i64, i32, p, p, i64, i64, i32, i32, i64, p, i32]
        L.orc_window_safe_len.restype = i32
        L.orc_window_safe_len.argtypes = [p, p, p, ctypes.c_int32, i64, p]
        L.orc_ring_trace.restype = i32
        L.orc_ring_trace.argtypes = [i64, i64, p]
        L.orc_kv_bytes.restype = i64
        L.orc_kv_bytes.argtypes = [i64, i64, i64, i64, i64]
        L.orc_hybrid_kv_ratio.restype = ctypes.c_double
        L.orc_hybrid_kv_ratio.argtypes = [i64, i64, i64, i64]
        L.orc_attention_kv64.restype = i32
        L.orc_attention_kv64.argtypes = [p, p, i64, i32, p, p, i64, i64, i32, i32, i64, p, i32]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_e4m3_quantize.restype = i32
        L.orc_e4m3_quantize.argtypes = [p, i64, ctypes.c_float, p]
        _lib = L
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 data (torch bf16 tensor or uint16/int16 numpy array) -> contiguous uint16 numpy."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype in (np.uint16, np.int16)
    return a.view(np.uint16)


def default_threads() -> int:
    return os.cpu_count() or 1


def mask_count(n: int, window: int) -> int:
    """Pairs (i, j) with j in W(i) for i < n (window 0 = full causal)."""
    return int(_load().orc_mask_count(n, window))


def attention(q, q_pos, k, v, window: int, key_base: int = 0, n_threads: int | None = None) -> np.ndarray:
    """fp64 attention rows.

    q: [n_rows, Hq, d] bf16; q_pos: [n_rows] absolute positions;
    k, v: [n_keys, Hkv, d] bf16 holding positions key_base .. key_base+n_keys-1;
    window >= 1 (sliding window) or 0 (full causal). Returns [n_rows, Hq, d] float64.
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    assert qb.ndim == 3 and kb.ndim == 3 and vb.shape == kb.shape
    n_rows, hq, d = qb.shape
    n_keys, hkv, d2 = kb.shape
    assert d == d2
    pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64))
    assert pos.shape == (n_rows,)
    out = np.empty((n_rows, hq, d), dtype=np.float64)
    rc = _load().orc_attention(qb.ctypes.data, pos.ctypes.data, n_rows, hq, kb.ctypes.data,
                               vb.ctypes.data, key_base, n_keys, hkv, d, window,
                               out.ctypes.data, n_threads or default_threads())
    if rc != 0:
        raise ValueError("oracle attention: a needed key position is outside the given keys")
    return out


def attention_kv64(q, q_pos, k, v, window: int, key_base: int = 0, n_threads: int | None = None) -> np.ndarray:
    """``attention`` with float64 keys and values [n_keys, Hkv, d] (dequantized FP8 entries, or a mix
    of those and bf16 ones); q is bf16 [n_rows, Hq, d]."""
    qb = _bits(q)
    k64 = np.ascontiguousarray(np.asarray(k, dtype=np.float64))
    v64 = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    assert qb.ndim == 3 and k64.ndim == 3 and v64.shape == k64.shape
    n_rows, hq, d = qb.shape
    n_keys, hkv, d2 = k64.shape
    assert d == d2
    pos = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64))
    out = np.empty((n_rows, hq, d), dtype=np.float64)
    rc = _load().orc_attention_kv64(qb.ctypes.data, pos.ctypes.data, n_rows, hq, k64.ctypes.data, v64.ctypes.data,
                                    key_base, n_keys, hkv, d, window, out.ctypes.data, n_threads or default_threads())
    if rc != 0:
        raise ValueError("oracle attention: a needed key position is outside the given keys")
    return out


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of FP8 E4M3 codes (uint8 array)."""
    c = np.asarray(codes, dtype=np.uint8)
    L = _load()
    return np.array([L.orc_e4m3_decode(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes of float64 values (nearest, ties to even, saturating at +-448)."""
    a = np.asarray(x, dtype=np.float64)
    L = _load()
    return np.array([L.orc_e4m3_encode(float(v)) for v in a.ravel()], dtype=np.uint8).reshape(a.shape)


def e4m3_quantize(x, scale: float) -> np.ndarray:
    """E4M3 codes of bf16 data x (torch bf16 tensor or uint16 bits) stored with scale `scale`:
    encode(fp32(x) * fp32(1 / scale))."""
    b = _bits(x)
    out = np.empty(b.shape, dtype=np.uint8)
    rc = _load().orc_e4m3_quantize(b.ctypes.data, b.size, float(scale), out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle e4m3_quantize: bad arguments")
    return out


def e4m3_dequantize(codes, scale: float) -> np.ndarray:
    """The values an FP8 cache holds: decode(code) * scale, in float64 (exact)."""
    return e4m3_decode(codes) * np.float64(np.float32(scale))


def window_safe_len(match_len, cached_len, slot_valid, window: int) -> np.ndarray:
    """Window-safe prefix-match length per request, by definition (int64)."""
    m = np.ascontiguousarray(np.asarray(match_len, dtype=np.int64))
    c = np.ascontiguousarray(np.asarray(cached_len, dtype=np.int64))
    words = (window + 31) // 32
    sv = np.ascontiguousarray(np.asarray(slot_valid, dtype=np.uint32)).reshape(-1)
    assert m.shape == c.shape and sv.size == m.size * words
    out = np.empty(m.shape, dtype=np.int64)
    rc = _load().orc_window_safe_len(m.ctypes.data, c.ctypes.data, sv.ctypes.data, window,
                                     m.size, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle window_safe_len: bad arguments")
    return out


def ring_trace(n_appended: int, w: int) -> np.ndarray:
    """Position held by each of the w ring slots after appending positions 0..n_appended-1."""
    out = np.empty(w, dtype=np.int64)
    assert _load().orc_ring_trace(n_appended, w, out.ctypes.data) == 0
    return out


def kv_bytes(layers: int, kv_heads: int, tokens: int, head_dim: int, elem_bytes: int = 2) -> int:
    return int(_load().orc_kv_bytes(layers, kv_heads, tokens, head_dim, elem_bytes))


def hybrid_kv_ratio(n_swa: int, n_full: int, window: int, n_tokens: int) -> float:
    return float(_load().orc_hybrid_kv_ratio(n_swa, n_full, window, n_tokens))


def pool_bytes(n_swa_layers: int, n_full_layers: int, window: int, n_kv_heads: int,
               head_dim: int, page_size: int, max_seqs: int, pages_per_full_layer: int,
               elem_bytes: int = 2) -> tuple[int, int]:
    """(SWA ring bytes, full paged-pool bytes) of the dual pool, from the KV-bytes formula:
    each sequence keeps W token-slots per SWA layer; each full layer keeps
    pages * page_size token-slots."""
    swa = kv_bytes(n_swa_layers, n_kv_heads, window * max_seqs, head_dim, elem_bytes)
    full = kv_bytes(n_full_layers, n_kv_heads, pages_per_full_layer * page_size, head_dim, elem_bytes)
    return swa, full


def prefix_cache_replay(window: int, ops):
    """Brute-force model of the SWA-aware prefix cache ("MiMo v2.5 inference optimisation",
    section "KV cache redesign": a prefix-cache match is cut to the window-safe length because
    only part of a cached sequence's window KV may survive).

    State, by definition: a cached position is a token prefix (a tuple); every cached position
    keeps its full-attention KV. Each insert names an owner (the ring row that keeps the
    sequence's window KV; -1 when the caller does not say). A position's holders are the owners of
    the inserts whose last `window` positions include it, counted once per insert, minus those
    whose copy was evicted after their insert; it holds sliding-window KV while it has a holder.
    `ops` is a list of ("insert", tokens[, owner]), ("release", tokens[, owner]),
    ("evict", tokens, lo, hi), ("match", tokens) and ("match_slots", tokens). A release undoes one
    earlier insert of exactly the same tokens by the same owner (ValueError when none is left; the
    empty sequence is a no-op). Returns one result per match, in order: "match" gives (m, L),
    m = the longest cached prefix of tokens, L = max { L in [0, m] : every position in
    [max(0, L - window), L) holds sliding-window KV }; "match_slots" gives (m, L, slots) with
    slots[s] = the set of holders of the position p of [max(0, L - window), L) with p mod window
    = s (empty for the other slots). Quadratic in sequence length: for small cases only.
    """
    cached = set()
    holders = {}   # token prefix -> list of owners (one entry per holding insert)
    inserted = {}  # (exact token tuple, owner) -> inserts not yet released
    out = []
    for op in ops:
        kind, toks = op[0], tuple(int(t) for t in op[1])
        n = len(toks)
        win = range(max(0, n - window), n)
        if kind == "insert":
            owner = int(op[2]) if len(op) > 2 else -1
            for p in range(n):
                cached.add(toks[:p + 1])
            for p in win:
                holders.setdefault(toks[:p + 1], []).append(owner)
            inserted[(toks, owner)] = inserted.get((toks, owner), 0) + 1
        elif kind == "release":
            owner = int(op[2]) if len(op) > 2 else -1
            if n == 0:
                continue
            if inserted.get((toks, owner), 0) == 0:
                raise ValueError("release of a sequence with no insert by this owner left to undo")
            inserted[(toks, owner)] -= 1
            for p in win:
                h = holders.get(toks[:p + 1], [])
                if owner in h:
                    h.remove(owner)
        elif kind == "evict":
            lo, hi = op[2], op[3]
            for p in range(max(0, lo), min(n, hi)):
                if toks[:p + 1] in cached:
                    holders[toks[:p + 1]] = []
        elif kind in ("match", "match_slots"):
            m = 0
            while m < n and toks[:m + 1] in cached:
                m += 1
            best = 0
            for L in range(0, m + 1):
                if all(len(holders.get(toks[:q + 1], [])) > 0 for q in range(max(0, L - window), L)):
                    best = L
            if kind == "match":
                out.append((m, best))
            else:
                slots = [set() for _ in range(window)]
                for q in range(max(0, best - window), best):
                    slots[q % window] = set(holders[toks[:q + 1]])
                out.append((m, best, slots))
        else:
            raise ValueError(kind)
    return out
