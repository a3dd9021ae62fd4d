"""GPU: FP8 (E4M3) KV storage in both pools ("MiMo v2.5 inference optimisation", closing section:
quantization cuts the bits of each cached entry and stacks with the sliding window's cut in
entries).

An FP8 pool stores code = E4M3(fp32(x) * fp32(1 / s)) per element, s the scale of the entry's
(layer, KV head, K or V), and reads it back as E4M3_value(code) * s. The commit is checked bit for
bit against the oracle's encoder. Attention on FP8 pools is checked against the fp64 oracle run on
the dequantized entries (the values the cache holds), at the same tolerance as the bf16 paths;
a decode step's new tokens enter as they will be stored (quantized), like every cached key.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import ATOL_MAX, ATOL_MEAN, kv_rows, page_table_for, q_rows

pytestmark = pytest.mark.gpu

FP8 = hs.HSWA_KV_FP8_E4M3


def _scales(seed, n, lo=0.25, hi=2.5):
    u = synth.uniform_float64(seed, synth.stream_id(synth.TAG_MISC, 61, n), n).numpy()
    return (lo + (hi - lo) * u).astype(np.float32)


def _deq(x_bf16, scales):
    """Values an FP8 cache holds for bf16 rows x [n, Hkv, d] stored with per-head scales."""
    out = np.empty(tuple(x_bf16.shape), dtype=np.float64)
    for g in range(x_bf16.shape[1]):
        out[:, g] = oracle.e4m3_dequantize(oracle.e4m3_quantize(x_bf16[:, g].contiguous(), scales[g]), scales[g])
    return out


def _close(got, ref, what):
    g = got.detach().float().cpu().double().numpy()
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, f"{what}: max {err.max():.3e} mean {err.mean():.3e}"


@pytest.mark.parametrize("d", [64, 128])
def test_append_stores_the_oracle_codes(d):
    hkv, W, n = 4, 128, 300
    desc = hs.PoolDesc(1, 1, W, hkv, d, 2, 16, kv_format=FP8)
    pool = hs.kv_pool_create(desc)
    ks, vs = _scales(1, hkv), _scales(2, hkv)
    ks[0] = 2.0 ** -10  # |x| / s beyond 448 for |x| > 0.44: saturates at +-448
    for layer in (0, 1):
        pool.set_scales(layer, ks, vs)
    k, v = kv_rows(71, 0, 0, 0, n, hkv, d)
    k[5, 1, :4] = torch.tensor([1e-4, -3e-3, 2e-2, 300.0], dtype=torch.bfloat16)  # subnormal, normal, large
    sid = torch.tensor([1], dtype=torch.int32, device="cuda")
    hs.kv_pool_append(pool, 0, k[None].cuda(), v[None].cuda(), torch.tensor([0], device="cuda"), seq_ids=sid)
    pt = torch.arange(16, dtype=torch.int32).flip(0).view(1, 16).contiguous().cuda()
    hs.kv_pool_append(pool, 1, k[None].cuda(), v[None].cuda(), torch.tensor([0], device="cuda"), page_table=pt)
    assert hs.hswa_pool_check_error(pool) == 0
    ring, pages = pool.ring.cpu(), pool.pages.cpu()
    for g in range(hkv):
        wk = oracle.e4m3_quantize(k[:, g].contiguous(), ks[g])
        wv = oracle.e4m3_quantize(v[:, g].contiguous(), vs[g])
        pos = np.arange(n - W, n)  # the ring keeps the last W positions, slot = pos mod W
        assert np.array_equal(ring[0, 1, 0, g, pos % W].numpy(), wk[pos])
        assert np.array_equal(ring[1, 1, 0, g, pos % W].numpy(), wv[pos])
        phys = pt[0].cpu().long()[np.arange(n) // 64]
        assert np.array_equal(pages[0, 0, phys, g, np.arange(n) % 64].numpy(), wk)
        assert np.array_equal(pages[1, 0, phys, g, np.arange(n) % 64].numpy(), wv)
    assert (ring[0, 1, 0, 0].numpy() == 0x7E).any() or (ring[0, 1, 0, 0].numpy() == 0xFE).any()


def _decode_case(seed, lens, n_qt, hq, hkv, d, W, kind, ks=None, vs=None):
    n = len(lens)
    max_ctx = max(lens)
    pps = (max_ctx + n_qt + 63) // 64
    total_pages = n * pps + 3 if kind == "full" else 1
    desc = hs.PoolDesc(1, 1, W, hkv, d, n + 1, total_pages, kv_format=FP8)
    pool = hs.kv_pool_create(desc)
    pool.data.fill_(0x7F)  # NaN codes wherever nothing was committed
    layer = 0 if kind == "swa" else 1
    ks = _scales(seed, hkv) if ks is None else ks
    vs = _scales(seed + 1, hkv) if vs is None else vs
    pool.set_scales(layer, ks, vs)
    sid = (torch.arange(n, dtype=torch.int32) * 3 % (n + 1)).contiguous()
    pt = page_table_for(seed, n, pps, total_pages).cuda() if kind == "full" else None
    for b, L in enumerate(lens):
        lo = max(0, L - W) if kind == "swa" else 0
        if L > lo:
            k, v = kv_rows(seed, layer, b, lo, L - lo, hkv, d)
            kw = dict(seq_ids=sid[b:b + 1].cuda()) if kind == "swa" else dict(page_table=pt[b:b + 1].contiguous())
            hs.kv_pool_append(pool, layer, k[None].cuda(), v[None].cuda(), torch.tensor([lo], device="cuda"), **kw)
    qs = [q_rows(seed, layer, b, L, n_qt, hq, d) for b, L in enumerate(lens)]
    kvn = [kv_rows(seed, layer, b, L, n_qt, hkv, d) for b, L in enumerate(lens)]
    q = torch.stack(qs).cuda()
    kn = torch.stack([x[0] for x in kvn]).cuda()
    vn = torch.stack([x[1] for x in kvn]).cuda()
    ctx = torch.tensor(lens, dtype=torch.int64).cuda()
    ws = torch.empty(hs.hybrid_decode_workspace_size(pool, n, n_qt, hq, max_ctx), dtype=torch.uint8, device="cuda")
    kw = dict(seq_ids=sid.cuda()) if kind == "swa" else dict(page_table=pt)
    o = hs.hybrid_decode_fwd(pool, layer, q, kn, vn, ctx, max_ctx, ws, **kw)
    assert hs.hswa_pool_check_error(pool) == 0
    window = W if kind == "swa" else 0
    for b, L in enumerate(lens):
        base = max(0, L - W + 1) if kind == "swa" else 0
        k, v = kv_rows(seed, layer, b, base, L + n_qt - base, hkv, d)
        ref = oracle.attention_kv64(qs[b], L + np.arange(n_qt), _deq(k, ks), _deq(v, vs), window, key_base=base)
        _close(o[b], ref, f"{kind} L={L}")


@pytest.mark.parametrize("W", [128, 5, 300])
def test_fp8_decode_ring(W):
    _decode_case(301, [0, 1, 3, 127, 128, 129, 1000, 4099, 70000], 4, 16, 2, 128, W, "swa")


@pytest.mark.parametrize("lens,n_qt,hq,hkv,d", [
    ([0, 5, 64, 65, 8191, 8192, 8193, 17000], 4, 16, 2, 128),  # split boundaries and a 3-split merge
    ([20000, 1, 12345], 4, 32, 4, 128),                         # 8 rows per KV head
    ([300, 5000], 1, 8, 1, 64),                                 # d = 64, G = 8, one token
    ([1024, 777, 50000], 2, 4, 4, 64),                          # G = 1
    ([70000, 3000], 4, 64, 8, 128),                             # config-4 head shape
])
def test_fp8_decode_paged(lens, n_qt, hq, hkv, d):
    _decode_case(302, lens, n_qt, hq, hkv, d, 128, "full")


@pytest.mark.parametrize("kind", ["full", "swa"])
def test_fp8_decode_subnormal_codes(kind):
    """Scales of 256 put nearly every N(0, 1) entry in E4M3's subnormal range (|x / s| < 2^-6):
    values m 2^-9 s, m = 1 .. 7. A kernel that lost them (flushed to zero) would be off by the
    size of O itself, far outside the tolerance."""
    hkv = 2
    big = np.full(hkv, 256.0, dtype=np.float32)
    _decode_case(303, [17, 64, 300, 5000], 4, 16, hkv, 128, 128, kind, ks=big, vs=big)


def test_fp8_pool_layout_and_scale_arguments():
    desc = hs.PoolDesc(2, 3, 128, 8, 128, 4, 100)
    t16, s16, f16 = hs.kv_pool_layout(desc)
    t8, s8, f8 = hs.kv_pool_layout(hs.PoolDesc(2, 3, 128, 8, 128, 4, 100, kv_format=FP8))
    assert s8 * 2 == s16 and f8 * 2 == f16
    assert t8 == s8 + f8 + (4 * 4 * 5 * 8 + 255) // 256 * 256 + 256
    bf = hs.kv_pool_create(hs.PoolDesc(1, 0, 64, 2, 64, 1, 0))
    with pytest.raises(hs.HswaError):
        bf.set_scales(0, [1.0, 1.0], [1.0, 1.0])  # scales apply to FP8 pools only
    p8 = hs.kv_pool_create(hs.PoolDesc(1, 0, 64, 2, 64, 1, 0, kv_format=FP8))
    for bad in ([0.0, 1.0], [1.0, float("nan")], [-1.0, 1.0], [1e-45, 1.0]):
        with pytest.raises(hs.HswaError):
            p8.set_scales(0, bad, [1.0, 1.0])
    with pytest.raises(hs.HswaError):
        p8.set_scales(1, [1.0, 1.0], [1.0, 1.0])  # no layer 1


@pytest.mark.parametrize("W,P,n_q,hq,hkv,d", [
    (128, 1024, 700, 8, 2, 128),   # narrow kernel, prefix tile on a 128 boundary
    (128, 1000, 300, 16, 2, 128),  # narrow kernel, unaligned prefix
    (100, 777, 260, 4, 4, 64),     # narrow kernel, d = 64, G = 1
    (300, 1500, 640, 8, 2, 128),   # general kernel, several ring tiles
    (256, 4096, 384, 8, 4, 128),   # general kernel, W a multiple of 128
])
def test_fp8_swa_prefill_reads_the_quantized_ring(W, P, n_q, hq, hkv, d):
    # the chunk's own keys and values are the bf16 inputs; the prefix comes from the FP8 ring
    seed = 311
    pool = hs.kv_pool_create(hs.PoolDesc(1, 0, W, hkv, d, 2, 0, kv_format=FP8))
    pool.data.fill_(0x7F)
    ks, vs = _scales(seed, hkv), _scales(seed + 1, hkv)
    pool.set_scales(0, ks, vs)
    sid = torch.tensor([1], dtype=torch.int32, device="cuda")
    kp, vp = kv_rows(seed, 0, 0, P - W, W, hkv, d)
    hs.kv_pool_append(pool, 0, kp[None].cuda(), vp[None].cuda(), torch.tensor([P - W], device="cuda"), seq_ids=sid)
    q = q_rows(seed, 0, 0, P, n_q, hq, d)
    kc, vc = kv_rows(seed, 0, 0, P, n_q, hkv, d)
    o = hs.swa_prefill_fwd(pool, 0, q[None].cuda(), kc[None].cuda(), vc[None].cuda(),
                           start_pos=torch.tensor([P], device="cuda"), seq_ids=sid)
    assert hs.hswa_pool_check_error(pool) == 0
    base = P - W + 1
    kpre, vpre = kv_rows(seed, 0, 0, base, W - 1, hkv, d)
    keys = np.concatenate([_deq(kpre, ks), kc.double().numpy()])
    vals = np.concatenate([_deq(vpre, vs), vc.double().numpy()])
    _close(o[0], oracle.attention_kv64(q, P + np.arange(n_q), keys, vals, W, key_base=base), f"W={W} P={P}")


@pytest.mark.parametrize("P,n_q,hq,hkv", [
    (2048, 640, 16, 2),    # 40 units
    (8190, 2050, 32, 4),   # 272 units (several per CTA), unaligned chunk start and end
    (0, 384, 8, 8),        # no prefix, G = 1 (query-tile pairs)
])
def test_fp8_full_prefill_over_quantized_pages(P, n_q, hq, hkv):
    seed, d = 312, 128
    total = P + n_q
    n_pages = (total + 63) // 64
    phys = n_pages + 5
    pool = hs.kv_pool_create(hs.PoolDesc(0, 1, 128, hkv, d, 1, phys, kv_format=FP8))
    pool.data.fill_(0x7F)  # NaN codes in every page row nobody wrote
    ks, vs = _scales(seed, hkv), _scales(seed + 1, hkv)
    pool.set_scales(0, ks, vs)
    perm = synth.permutation(seed, synth.stream_id(synth.TAG_MISC, 62), phys)[:n_pages]
    pt = perm.view(1, n_pages).to(torch.int32).contiguous().cuda()
    k, v = kv_rows(seed, 0, 0, 0, total, hkv, d)
    hs.kv_pool_append(pool, 0, k[None].cuda(), v[None].cuda(), torch.tensor([0], device="cuda"), page_table=pt)
    q = q_rows(seed, 0, 0, P, n_q, hq, d)
    o = hs.full_prefill_fwd(pool, 0, q[None].cuda(), pt, start_pos=torch.tensor([P], device="cuda"))
    assert hs.hswa_pool_check_error(pool) == 0
    rows = np.unique(np.concatenate([np.arange(0, n_q, 7), [n_q - 1]]))
    ref = oracle.attention_kv64(q[rows], P + rows, _deq(k, ks), _deq(v, vs), 0)
    _close(o[0, rows], ref, f"full P={P}")


def test_fp8_full_prefill_head_dim_64_is_refused():
    pool = hs.kv_pool_create(hs.PoolDesc(0, 1, 128, 1, 64, 1, 4, kv_format=FP8))
    q = torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16, device="cuda")
    pt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(hs.HswaError) as e:
        hs.full_prefill_fwd(pool, 0, q, pt)
    assert e.value.code == hs.HSWA_ERR_UNSUPPORTED_SHAPE
