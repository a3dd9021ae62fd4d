"""GPU: hybrid_decode_fwd_noalloc, the decode entry point for callers that cannot allocate device
memory when they call the library (it uses the library's fixed built-in scratch array instead of
a caller workspace).

Called straight through the C ABI (ctypes), twice in a row on different problems, each time
compared with hybrid_decode_fwd run with an ordinary caller-provided workspace. The second call
finds the scratch array holding the first call's leftovers, which must not change its result.
This file sorts last so that a run stopping at its first failure has already run everything else;
it builds its own inputs, so it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import hybrid_sliding_window_swa_b200 as hs
import oracle
import synth

pytestmark = pytest.mark.gpu

ATOL_MAX = 2e-2   # the attention tolerance of the other GPU tests
ATOL_MEAN = 2e-3


def _rows(seed, tag, layer, seq, pos0, n, h, d):
    x = synth.normal_bf16_rows(seed, synth.stream_id(tag, layer, seq), pos0, n, h * d, 1.0, "cpu")
    return x.view(n, h, d)


def _problem(seed, lens, n_qt, hq, hkv, d, window):
    """A pool with one SWA layer (ring) and one full layer (pages) holding these context lengths."""
    n = len(lens)
    max_ctx = max(lens)
    pps = (max_ctx + n_qt + 63) // 64
    total_pages = n * pps + 2
    desc = hs.PoolDesc(n_swa_layers=1, n_full_layers=1, window=window, n_kv_heads=hkv, head_dim=d,
                       max_seqs=n, pages_per_full_layer=total_pages)
    pool = hs.kv_pool_create(desc)
    pool.data.zero_()
    perm = synth.permutation(seed, synth.stream_id(synth.TAG_MISC, 50), total_pages)
    pt = perm[: n * pps].view(n, pps).to(torch.int32).contiguous().cuda()
    sid = torch.arange(n, dtype=torch.int32).cuda()
    for b, L in enumerate(lens):
        lo = max(0, L - window)
        if L > lo:
            k, v = _rows(seed, synth.TAG_K, 0, b, lo, L - lo, hkv, d), _rows(seed, synth.TAG_V, 0, b, lo, L - lo, hkv, d)
            hs.kv_pool_append(pool, 0, k[None].cuda(), v[None].cuda(), torch.tensor([lo]).cuda(), seq_ids=sid[b:b + 1])
        if L > 0:
            k, v = _rows(seed, synth.TAG_K, 1, b, 0, L, hkv, d), _rows(seed, synth.TAG_V, 1, b, 0, L, hkv, d)
            hs.kv_pool_append(pool, 1, k[None].cuda(), v[None].cuda(), torch.tensor([0]).cuda(),
                              page_table=pt[b:b + 1].contiguous())
    inputs = {}
    for layer in (0, 1):
        q = torch.stack([_rows(seed, synth.TAG_Q, layer, b, L, n_qt, hq, d) for b, L in enumerate(lens)]).cuda()
        kn = torch.stack([_rows(seed, synth.TAG_K, layer, b, L, n_qt, hkv, d) for b, L in enumerate(lens)]).cuda()
        vn = torch.stack([_rows(seed, synth.TAG_V, layer, b, L, n_qt, hkv, d) for b, L in enumerate(lens)]).cuda()
        inputs[layer] = (q, kn, vn)
    ctx = torch.tensor(lens, dtype=torch.int64).cuda()
    return pool, pt, sid, ctx, max_ctx, inputs


def _noalloc_via_c_abi(pool, layer, q, kn, vn, o, ctx, max_ctx, sid, pt):
    lib = hs.load_library()
    vp = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    rc = lib.hybrid_decode_fwd_noalloc(
        pool.handle, layer, vp(q), vp(kn), vp(vn), vp(o), q.shape[0], q.shape[1], vp(ctx), max_ctx, vp(sid),
        vp(pt), pt.shape[1] if pt is not None else 0, q.shape[2],
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == hs.HSWA_OK, lib.hswa_last_error().decode()


def _check_close(a, b, what):
    err = (a.float() - b.float()).abs()
    assert torch.isfinite(a.float()).all(), what
    assert err.max().item() <= ATOL_MAX and err.mean().item() <= ATOL_MEAN, f"{what}: {err.max().item():.3e}"


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row():
    cases = [
        # several splits per sequence on the full layer: the scratch holds split partials
        dict(seed=901, lens=[9000, 17, 4096, 12345], n_qt=4, hq=16, hkv=2, d=128, window=128),
        # a different shape: the second call meets the first call's leftovers in the scratch
        dict(seed=902, lens=[3, 700, 20000], n_qt=2, hq=8, hkv=8, d=64, window=64),
    ]
    for call, c in enumerate(cases):
        pool, pt, sid, ctx, max_ctx, inputs = _problem(c["seed"], c["lens"], c["n_qt"], c["hq"], c["hkv"], c["d"],
                                                       c["window"])
        need = hs.hybrid_decode_workspace_size(pool, len(c["lens"]), c["n_qt"], c["hq"], max_ctx)
        assert need <= hs.NOALLOC_SCRATCH_BYTES
        for layer in (0, 1):
            q, kn, vn = inputs[layer]
            ws = torch.empty(need, dtype=torch.uint8, device="cuda")
            kw = dict(seq_ids=sid) if layer == 0 else dict(page_table=pt)
            ref = hs.hybrid_decode_fwd(pool, layer, q, kn, vn, ctx, max_ctx, ws, **kw)
            out = torch.full_like(q, float("nan"))
            _noalloc_via_c_abi(pool, layer, q, kn, vn, out, ctx, max_ctx, sid if layer == 0 else None,
                               pt if layer == 1 else None)
            torch.cuda.synchronize()
            assert hs.hswa_pool_check_error(pool) == 0
            _check_close(out, ref, f"call {call} layer {layer}")
            # and directly against the fp64 oracle, on inputs regenerated on the CPU
            d, W, hq, hkv, n_qt = c["d"], c["window"], c["hq"], c["hkv"], c["n_qt"]
            for b, L in enumerate(c["lens"]):
                base = max(0, L - W + 1) if layer == 0 else 0
                kk = _rows(c["seed"], synth.TAG_K, layer, b, base, L + n_qt - base, hkv, d)
                vv = _rows(c["seed"], synth.TAG_V, layer, b, base, L + n_qt - base, hkv, d)
                qq = _rows(c["seed"], synth.TAG_Q, layer, b, L, n_qt, hq, d)
                want = oracle.attention(qq, L + np.arange(n_qt), kk, vv, W if layer == 0 else 0, key_base=base)
                err = np.abs(out[b].float().cpu().double().numpy() - want)
                assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, f"call {call} layer {layer} seq {b}"


def test_noalloc_rejects_calls_beyond_its_scratch():
    desc = hs.PoolDesc(n_swa_layers=0, n_full_layers=1, window=128, n_kv_heads=8, head_dim=128, max_seqs=1,
                       pages_per_full_layer=4)
    pool = hs.kv_pool_create(desc)
    n, n_qt, hq, max_ctx = 256, 4, 64, 1 << 20  # full layer, 1M tokens: far above 64 MiB of partials
    assert hs.hybrid_decode_workspace_size(pool, n, n_qt, hq, max_ctx) > hs.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(n, n_qt, hq, 128, dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros(n, n_qt, 8, 128, dtype=torch.bfloat16, device="cuda")
    ctx = torch.zeros(n, dtype=torch.int64, device="cuda")
    pt = torch.zeros(n, 4, dtype=torch.int32, device="cuda")
    lib = hs.load_library()
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = lib.hybrid_decode_fwd_noalloc(pool.handle, 0, vp(q), vp(kn), vp(kn), vp(q), n, n_qt, vp(ctx), max_ctx, None,
                                       vp(pt), 4, hq, None)
    assert rc == hs.HSWA_ERR_OUT_OF_MEMORY
    assert "scratch" in lib.hswa_last_error().decode()
