"""hybrid_sliding_window_swa_b200 -- hybrid sliding-window attention on NVIDIA B200.

Thin Python binding over ``libhswa.so`` (C ABI in ``include/hswa.h``). Every function
here has the name of the C entry point it calls and only marshals arguments
(torch tensors -> device pointers, the current CUDA stream); all computation runs
in the library's sm_100a kernels. There is no fallback: if the library is missing
or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhswa.so")

HSWA_OK = 0
HSWA_ERR_INVALID_ARG = -1
HSWA_ERR_UNSUPPORTED_SHAPE = -2
HSWA_ERR_OUT_OF_MEMORY = -3
HSWA_ERR_CUDA = -4
HSWA_ERR_TIMEOUT = -5
HSWA_ERR_DEVICE_BOUNDS = -6

HSWA_KV_BF16 = 0
HSWA_KV_FP8_E4M3 = 1

EXPORTED = [
    "kv_pool_layout", "kv_pool_create", "kv_pool_destroy", "kv_pool_append",
    "swa_prefill_fwd", "full_prefill_fwd", "hybrid_decode_workspace_size", "hybrid_decode_fwd",
    "window_safe_len", "hswa_pool_check_error", "hswa_last_error", "hybrid_decode_fwd_noalloc",
    "hswa_selftest_wait_timeout", "hswa_tree_create", "hswa_tree_destroy", "hswa_tree_insert",
    "hswa_tree_release", "hswa_tree_evict_swa", "hswa_tree_match", "hswa_tree_match_batch", "hswa_tree_stats",
    "hswa_tree_match_slots", "kv_pool_gather_ring", "kv_pool_set_scales", "hswa_shard_kv_heads",
    "hswa_shard_sequences",
]

# scratch bytes available to hybrid_decode_fwd_noalloc (HSWA_NOALLOC_SCRATCH_BYTES in hswa.h)
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


class HswaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"hswa error {code}: {msg}")
        self.code = code


class PoolDescC(ctypes.Structure):
    _fields_ = [
        ("n_swa_layers", ctypes.c_int32), ("n_full_layers", ctypes.c_int32), ("window", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("max_seqs", ctypes.c_int32), ("kv_format", ctypes.c_int32), ("pages_per_full_layer", ctypes.c_int64),
    ]


_lib = None


def load_library(path: str | None = None):
    """Load libhswa.so (raises if it is absent: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("HSWA_LIBRARY") or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libhswa.so not found at {path}; build it with "
                          f"`python -m hybrid_sliding_window_swa_b200._build`")
    L = ctypes.CDLL(path)
    p, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "kv_pool_layout": [ctypes.POINTER(PoolDescC), ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)],
        "kv_pool_create": [ctypes.POINTER(PoolDescC), p, sz, ctypes.POINTER(p)],
        "kv_pool_destroy": [p],
        "kv_pool_append": [p, i32, i32, p, p, i32, p, p, p, i32, p],
        "swa_prefill_fwd": [p, i32, p, p, p, p, i32, i32, p, p, i32, p],
        "full_prefill_fwd": [p, i32, p, p, i32, i32, p, p, i32, i32, p],
        "hybrid_decode_workspace_size": [p, i32, i32, i32, i64, ctypes.POINTER(sz)],
        "hybrid_decode_fwd": [p, i32, p, p, p, p, i32, i32, p, i64, p, p, i32, i32, p, sz, p],
        "window_safe_len": [p, p, p, ctypes.c_int32, ctypes.c_int32, p, p],
        "hswa_pool_check_error": [p, ctypes.POINTER(ctypes.c_int)],
        "hybrid_decode_fwd_noalloc": [p, i32, p, p, p, p, i32, i32, p, i64, p, p, i32, i32, p],
        "hswa_selftest_wait_timeout": [p, i64, p],
        "hswa_tree_create": [ctypes.c_int32, ctypes.POINTER(p)],
        "hswa_tree_destroy": [p],
        "hswa_tree_insert": [p, p, i64, ctypes.c_int32, ctypes.POINTER(i64)],
        "hswa_tree_release": [p, p, i64, ctypes.c_int32],
        "hswa_tree_match_slots": [p, p, i64, ctypes.POINTER(i64), ctypes.POINTER(i64), p],
        "kv_pool_gather_ring": [p, i32, ctypes.c_int32, p, p],
        "kv_pool_set_scales": [p, i32, p, p],
        "hswa_shard_kv_heads": [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                ctypes.POINTER(ctypes.c_int32)],
        "hswa_shard_sequences": [p, ctypes.c_int32, ctypes.c_int32, p, p],
        "hswa_tree_evict_swa": [p, p, i64, i64, i64, ctypes.POINTER(i64)],
        "hswa_tree_match": [p, p, i64, ctypes.POINTER(i64), ctypes.POINTER(i64)],
        "hswa_tree_match_batch": [p, p, p, ctypes.c_int32, p, p],
        "hswa_tree_stats": [p, ctypes.POINTER(i64), ctypes.POINTER(i64)],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.hswa_last_error.argtypes = []
    L.hswa_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(rc: int):
    if rc != HSWA_OK:
        msg = load_library().hswa_last_error().decode(errors="replace")
        raise HswaError(rc, msg)


def _ptr(t: torch.Tensor | None, dtype=None, name: str = "tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass(frozen=True)
class PoolDesc:
    n_swa_layers: int
    n_full_layers: int
    window: int
    n_kv_heads: int
    head_dim: int
    max_seqs: int
    pages_per_full_layer: int
    page_size: int = 64
    kv_format: int = HSWA_KV_BF16

    def c(self) -> PoolDescC:
        return PoolDescC(self.n_swa_layers, self.n_full_layers, self.window, self.n_kv_heads, self.head_dim,
                         self.page_size, self.max_seqs, self.kv_format, self.pages_per_full_layer)

    @property
    def fp8(self) -> bool:
        return self.kv_format == HSWA_KV_FP8_E4M3


def kv_pool_layout(desc: PoolDesc) -> tuple[int, int, int]:
    """(bytes_total, bytes_swa, bytes_full) of the dual pool."""
    L = load_library()
    t, s, f = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    d = desc.c()
    _check(L.kv_pool_layout(ctypes.byref(d), ctypes.byref(t), ctypes.byref(s), ctypes.byref(f)))
    return t.value, s.value, f.value


class KVPool:
    """A dual-pool KV cache carved out of one caller-owned torch uint8 CUDA buffer."""

    def __init__(self, desc: PoolDesc, memory: torch.Tensor, handle):
        self.desc = desc
        self.memory = memory
        self.handle = handle

    def _views(self):
        d = self.desc
        _, swa, _full = kv_pool_layout(d)
        e = 1 if d.fp8 else 2
        ring_half = d.max_seqs * d.n_swa_layers * d.n_kv_heads * d.window * d.head_dim
        page_half = d.n_full_layers * d.pages_per_full_layer * d.n_kv_heads * d.page_size * d.head_dim
        mem = self.memory
        ring = mem[: 2 * e * ring_half]
        pages = mem[swa: swa + 2 * e * page_half]
        if not d.fp8:
            ring, pages = ring.view(torch.bfloat16), pages.view(torch.bfloat16)
        ring = ring.view(2, d.max_seqs, d.n_swa_layers, d.n_kv_heads, d.window, d.head_dim)
        pages = pages.view(2, d.n_full_layers, d.pages_per_full_layer, d.n_kv_heads, d.page_size, d.head_dim)
        return ring, pages

    @property
    def data(self) -> torch.Tensor:
        """uint8 view of the K/V regions only (the library's error word that follows them excluded)."""
        _, swa, full = kv_pool_layout(self.desc)
        return self.memory[: swa + full]

    @property
    def ring(self) -> torch.Tensor:
        """[2 (K,V)][max_seqs][n_swa_layers][Hkv][W][d] view of the rolling buffers (bf16, or uint8
        E4M3 codes in an FP8 pool)."""
        return self._views()[0]

    @property
    def pages(self) -> torch.Tensor:
        """[2 (K,V)][n_full_layers][pages][Hkv][page_size][d] view of the paged pool (bf16, or uint8
        E4M3 codes in an FP8 pool)."""
        return self._views()[1]

    def set_scales(self, layer: int, k_scale, v_scale):
        """FP8 pools: K and V scales of `layer`, one per KV head (see kv_pool_set_scales)."""
        kv_pool_set_scales(self, layer, k_scale, v_scale)

    def destroy(self):
        if self.handle is not None:
            load_library().kv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def kv_pool_create(desc: PoolDesc, memory: torch.Tensor | None = None, device=None) -> KVPool:
    """Carve a pool from ``memory`` (uint8 CUDA tensor of >= bytes_total) or allocate one with torch."""
    L = load_library()
    total, _, _ = kv_pool_layout(desc)
    if memory is None:
        memory = torch.empty(total, dtype=torch.uint8, device=device or "cuda")
    _ptr(memory, torch.uint8, "memory")
    h = ctypes.c_void_p()
    d = desc.c()
    _check(L.kv_pool_create(ctypes.byref(d), ctypes.c_void_p(memory.data_ptr()), memory.numel(), ctypes.byref(h)))
    return KVPool(desc, memory, h)


def kv_pool_set_scales(pool: KVPool, layer: int, k_scale, v_scale):
    """FP8 pools: K and V scales of `layer` (sequences of n_kv_heads floats > 0; host values)."""
    import numpy as np
    ks = np.ascontiguousarray(np.asarray(k_scale, dtype=np.float32).reshape(-1))
    vs = np.ascontiguousarray(np.asarray(v_scale, dtype=np.float32).reshape(-1))
    if ks.size != pool.desc.n_kv_heads or vs.size != pool.desc.n_kv_heads:
        raise ValueError("one K and one V scale per KV head")
    _check(load_library().kv_pool_set_scales(pool.handle, layer, ks.ctypes.data_as(ctypes.c_void_p),
                                             vs.ctypes.data_as(ctypes.c_void_p)))


def kv_pool_destroy(pool: KVPool):
    pool.destroy()


def kv_pool_append(pool: KVPool, layer: int, k: torch.Tensor, v: torch.Tensor, start_pos: torch.Tensor,
                   seq_ids: torch.Tensor | None = None, page_table: torch.Tensor | None = None, stream=None):
    """Commit k, v [n_seqs, n_tok, Hkv, d] at positions start_pos[b] + t of layer ``layer``."""
    n_seqs, n_tok = k.shape[0], k.shape[1]
    pt_stride = page_table.shape[1] if page_table is not None else 0
    _check(load_library().kv_pool_append(
        pool.handle, layer, n_seqs, _ptr(seq_ids, torch.int32, "seq_ids"), _ptr(start_pos, torch.int64, "start_pos"),
        n_tok, _ptr(k, torch.bfloat16, "k"), _ptr(v, torch.bfloat16, "v"),
        _ptr(page_table, torch.int32, "page_table"), pt_stride, _stream(stream)))


def kv_pool_gather_ring(pool: KVPool, layer: int, dst_seq: int, src_seq: torch.Tensor, stream=None):
    """Assemble ring row dst_seq of layer ``layer`` slot by slot from the rows src_seq[s] (int32 [W]
    on the device; -1 leaves a slot as it is)."""
    _check(load_library().kv_pool_gather_ring(pool.handle, layer, dst_seq, _ptr(src_seq, torch.int32, "src_seq"),
                                              _stream(stream)))


def swa_prefill_fwd(pool: KVPool, layer: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    o: torch.Tensor | None = None, start_pos: torch.Tensor | None = None,
                    seq_ids: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Sliding-window attention of a chunk: q [B, n_q, Hq, d], k/v [B, n_q, Hkv, d] -> o like q."""
    B, n_q, hq, _ = q.shape
    if o is None:
        o = torch.empty_like(q)
    _check(load_library().swa_prefill_fwd(
        pool.handle, layer, _ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
        _ptr(v, torch.bfloat16, "v"), _ptr(o, torch.bfloat16, "o"), B, n_q,
        _ptr(start_pos, torch.int64, "start_pos"), _ptr(seq_ids, torch.int32, "seq_ids"), hq, _stream(stream)))
    return o


def full_prefill_fwd(pool: KVPool, layer: int, q: torch.Tensor, page_table: torch.Tensor,
                     o: torch.Tensor | None = None, start_pos: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Full causal attention of a chunk over the paged pool (the chunk must be appended first)."""
    B, n_q, hq, _ = q.shape
    if o is None:
        o = torch.empty_like(q)
    _check(load_library().full_prefill_fwd(
        pool.handle, layer, _ptr(q, torch.bfloat16, "q"), _ptr(o, torch.bfloat16, "o"), B, n_q,
        _ptr(start_pos, torch.int64, "start_pos"), _ptr(page_table, torch.int32, "page_table"),
        page_table.shape[1], hq, _stream(stream)))
    return o


def hybrid_decode_workspace_size(pool: KVPool, n_seqs: int, n_q_per_seq: int, n_q_heads: int,
                                 max_ctx_len: int) -> int:
    out = ctypes.c_size_t()
    _check(load_library().hybrid_decode_workspace_size(pool.handle, n_seqs, n_q_per_seq, n_q_heads,
                                                       max_ctx_len, ctypes.byref(out)))
    return out.value


def hybrid_decode_fwd(pool: KVPool, layer: int, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                      ctx_len: torch.Tensor, max_ctx_len: int, workspace: torch.Tensor,
                      seq_ids: torch.Tensor | None = None, page_table: torch.Tensor | None = None,
                      o: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One decode step: q [n_seqs, n_qt, Hq, d], k_new/v_new [n_seqs, n_qt, Hkv, d] -> o like q."""
    n_seqs, n_qt, hq, _ = q.shape
    if o is None:
        o = torch.empty_like(q)
    pt_stride = page_table.shape[1] if page_table is not None else 0
    _check(load_library().hybrid_decode_fwd(
        pool.handle, layer, _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _ptr(o, torch.bfloat16, "o"), n_seqs, n_qt,
        _ptr(ctx_len, torch.int64, "ctx_len"), max_ctx_len, _ptr(seq_ids, torch.int32, "seq_ids"),
        _ptr(page_table, torch.int32, "page_table"), pt_stride, hq, _ptr(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)))
    return o


def window_safe_len(match_len: torch.Tensor, cached_len: torch.Tensor, slot_valid: torch.Tensor, window: int,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Window-safe prefix-match length per request (int64, exact)."""
    n = match_len.numel()
    if out is None:
        out = torch.empty(n, dtype=torch.int64, device=match_len.device)
    sv = slot_valid.view(torch.int32) if slot_valid.dtype == torch.uint32 else slot_valid
    _check(load_library().window_safe_len(
        _ptr(match_len, torch.int64, "match_len"), _ptr(cached_len, torch.int64, "cached_len"),
        _ptr(sv, torch.int32, "slot_valid"), window, n, _ptr(out, torch.int64, "out"), _stream(stream)))
    return out


def hswa_pool_check_error(pool: KVPool) -> int:
    """Synchronise and return (then clear) the pool's device error code (0 = none)."""
    code = ctypes.c_int()
    _check(load_library().hswa_pool_check_error(pool.handle, ctypes.byref(code)))
    return code.value


def hswa_selftest_wait_timeout(pool: KVPool, limit_ns: int = 50_000_000, stream=None):
    """Run one bounded wait that is meant to run out (see include/hswa.h)."""
    _check(load_library().hswa_selftest_wait_timeout(pool.handle, limit_ns, _stream(stream)))


def hswa_last_error() -> str:
    return load_library().hswa_last_error().decode(errors="replace")


def hybrid_decode_fwd_noalloc(pool: KVPool, layer: int, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                              ctx_len: torch.Tensor, max_ctx_len: int, o: torch.Tensor,
                              seq_ids: torch.Tensor | None = None, page_table: torch.Tensor | None = None,
                              stream=None) -> torch.Tensor:
    """hybrid_decode_fwd for callers that cannot allocate device memory at call time: the split-KV
    scratch is the library's fixed built-in array, so the caller passes only inputs and the output.
    Calls that overlap on the GPU share that array and race; run them one after another."""
    n_seqs, n_qt, hq, _ = q.shape
    pt_stride = page_table.shape[1] if page_table is not None else 0
    _check(load_library().hybrid_decode_fwd_noalloc(
        pool.handle, layer, _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), _ptr(o, torch.bfloat16, "o"), n_seqs, n_qt,
        _ptr(ctx_len, torch.int64, "ctx_len"), max_ctx_len, _ptr(seq_ids, torch.int32, "seq_ids"),
        _ptr(page_table, torch.int32, "page_table"), pt_stride, hq, _stream(stream)))
    return o


def hswa_shard_kv_heads(n_kv_heads: int, n_ranks: int, rank: int) -> tuple[int, int]:
    """[head_begin, head_end) of the KV heads rank `rank` owns when prefill is split over n_ranks."""
    b, e = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().hswa_shard_kv_heads(n_kv_heads, n_ranks, rank, ctypes.byref(b), ctypes.byref(e)))
    return b.value, e.value


def hswa_shard_sequences(ctx_len, n_ranks: int):
    """(rank of each sequence, total context per rank) for decode split over n_ranks (numpy arrays)."""
    import numpy as np
    lens = np.ascontiguousarray(np.asarray(ctx_len, dtype=np.int64).reshape(-1))
    ranks = np.zeros(lens.size, dtype=np.int32)
    loads = np.zeros(n_ranks, dtype=np.int64)
    _check(load_library().hswa_shard_sequences(lens.ctypes.data_as(ctypes.c_void_p), lens.size, n_ranks,
                                               ranks.ctypes.data_as(ctypes.c_void_p),
                                               loads.ctypes.data_as(ctypes.c_void_p)))
    return ranks, loads


def _tokens(tokens):
    """int32 host token array (numpy view, or a copy when the input is not int32/contiguous)."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(tokens), dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.c_void_p)


class PrefixTree:
    """SWA-aware prefix cache over a token trie (host code; see include/hswa.h, hswa_tree_*)."""

    def __init__(self, window: int):
        h = ctypes.c_void_p()
        _check(load_library().hswa_tree_create(window, ctypes.byref(h)))
        self.handle, self.window = h, window

    def close(self):
        if self.handle:
            load_library().hswa_tree_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def insert(self, tokens, owner: int = -1) -> int:
        """Cache tokens for `owner` (the ring row holding its window, or -1); returns positions added."""
        a, ptr = _tokens(tokens)
        added = ctypes.c_int64()
        _check(load_library().hswa_tree_insert(self.handle, ptr, a.size, owner, ctypes.byref(added)))
        return added.value

    def release(self, tokens, owner: int = -1):
        a, ptr = _tokens(tokens)
        _check(load_library().hswa_tree_release(self.handle, ptr, a.size, owner))

    def evict_swa(self, tokens, pos_lo: int, pos_hi: int) -> int:
        a, ptr = _tokens(tokens)
        n = ctypes.c_int64()
        _check(load_library().hswa_tree_evict_swa(self.handle, ptr, a.size, pos_lo, pos_hi, ctypes.byref(n)))
        return n.value

    def match(self, tokens) -> tuple[int, int]:
        """(match length, window-safe length) of one request."""
        a, ptr = _tokens(tokens)
        m, s = ctypes.c_int64(), ctypes.c_int64()
        _check(load_library().hswa_tree_match(self.handle, ptr, a.size, ctypes.byref(m), ctypes.byref(s)))
        return m.value, s.value

    def match_slots(self, tokens):
        """(match length, window-safe length L, int32 numpy [W]: per ring slot, the owner holding the
        position of [max(0, L - W), L) in that slot, else -1)."""
        import numpy as np
        a, ptr = _tokens(tokens)
        m, s = ctypes.c_int64(), ctypes.c_int64()
        owners = np.full(self.window, -1, dtype=np.int32)
        _check(load_library().hswa_tree_match_slots(self.handle, ptr, a.size, ctypes.byref(m), ctypes.byref(s),
                                                    owners.ctypes.data_as(ctypes.c_void_p)))
        return m.value, s.value, owners

    def match_batch(self, requests):
        """(match lengths, window-safe lengths) as int64 numpy arrays for a list of token sequences."""
        import numpy as np
        lens = np.array([len(r) for r in requests], dtype=np.int64)
        offsets = np.zeros(len(requests) + 1, dtype=np.int64)
        np.cumsum(lens, out=offsets[1:])
        flat = np.ascontiguousarray(np.concatenate([np.asarray(r, dtype=np.int32) for r in requests])
                                    if requests else np.zeros(0, np.int32), dtype=np.int32)
        m = np.zeros(len(requests), dtype=np.int64)
        s = np.zeros(len(requests), dtype=np.int64)
        _check(load_library().hswa_tree_match_batch(
            self.handle, flat.ctypes.data_as(ctypes.c_void_p), offsets.ctypes.data_as(ctypes.c_void_p),
            len(requests), m.ctypes.data_as(ctypes.c_void_p), s.ctypes.data_as(ctypes.c_void_p)))
        return m, s

    def stats(self) -> tuple[int, int]:
        """(cached positions, positions holding sliding-window KV)."""
        n, h = ctypes.c_int64(), ctypes.c_int64()
        _check(load_library().hswa_tree_stats(self.handle, ctypes.byref(n), ctypes.byref(h)))
        return n.value, h.value

