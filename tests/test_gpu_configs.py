"""GPU: the prefill and decode workloads at their full sizes against the fp64 oracle.

At these sizes every launch runs the persistent multi-unit paths: a CTA of the general prefill
kernel takes about 28 units of the 16K-token, W=4096 chunk in turn, the narrow kernel about 7
units of the W=128 chunk, and the decode kernel's 296 CTAs pull thousands of (sequence, split,
KV head) items from the work counter. That exercises the barrier phases carried from one unit
to the next, the reuse of Q slots and TMEM columns, and the split merge at 256K tokens, none of
which the small cases reach. The oracle regenerates its inputs from the seeded generator on the
CPU (it never sees a GPU tensor) and computes sampled rows (all heads of each): the first and
last rows, rows at the window and tile edges, and seeded random rows.

Workloads ("Sliding Window Attention (SWA) no riron to jisso", section "Mistral: SWA and GQA";
"MiMo v2.5 inference optimisation", sections "architecture" and "KV cache redesign"):
  * Mistral-shaped SWA prefill of one 16K chunk: B=2, N=16384, W=4096, Hq=32, Hkv=8, d=128,
    inputs N(0, 1/2);
  * one 16K chunk after a 131072-token prefix on a W=128 layer (ring prefix), Hq=64, Hkv=8;
  * a full layer over a paged prefix (16384 cached + 4096 chunk tokens, randomly permuted
    64-token pages), Hq=64, Hkv=8: 1024 work units, 7 per CTA;
  * the hybrid decode batch: 256 sequences, context lengths log-uniform in [1K, 256K], 4 query
    tokens each, a W=128 ring layer and a paged full layer, Hq=64, Hkv=8, on a bf16 pool and on
    an FP8 (E4M3) pool.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import compare, kv_rows, q_rows

pytestmark = pytest.mark.gpu


def _sample_rows(seed, n, fixed, n_random):
    rng = np.random.default_rng(seed)
    extra = rng.choice(n, size=min(n, n_random), replace=False)
    return sorted({int(r) for r in fixed if 0 <= r < n} | {int(r) for r in extra})


def _q_rows_cpu(seed, layer, seq, pos0, rows, hq, d, sigma=1.0):
    """Query rows pos0 + r for r in rows, generated one by one on the CPU."""
    return torch.stack([q_rows(seed, layer, seq, pos0 + r, 1, hq, d, sigma)[0] for r in rows])


def test_swa_prefill_16k_chunk_W4096_full_size():
    B, N, W, Hq, Hkv, d = 2, 16384, 4096, 32, 8, 128
    sigma = 2 ** -0.5
    seed = 3101
    pool = hs.kv_pool_create(hs.PoolDesc(1, 0, W, Hkv, d, B, 0))
    q = torch.stack([q_rows(seed, 0, b, 0, N, Hq, d, sigma, "cuda") for b in range(B)])
    kv = [kv_rows(seed, 0, b, 0, N, Hkv, d, sigma, "cuda") for b in range(B)]
    k = torch.stack([x[0] for x in kv])
    v = torch.stack([x[1] for x in kv])
    del kv
    o = hs.swa_prefill_fwd(pool, 0, q, k, v)
    assert hs.hswa_pool_check_error(pool) == 0
    rows = _sample_rows(seed, N, [0, 1, 127, 128, W - 2, W - 1, W, 8191, 8192, N - 1], 64)
    for b in range(B):
        kc, vc = kv_rows(seed, 0, b, 0, N, Hkv, d, sigma)
        qc = _q_rows_cpu(seed, 0, b, 0, rows, Hq, d, sigma)
        ref = oracle.attention(qc, np.array(rows), kc, vc, W)
        compare(o[b, rows], ref, f"16K chunk W=4096, sequence {b}")


def test_swa_layer_W128_chunk_after_131072_prefix_full_size():
    P, Nc, W, Hq, Hkv, d = 131072, 16384, 128, 64, 8, 128
    seed = 3102
    pool = hs.kv_pool_create(hs.PoolDesc(1, 0, W, Hkv, d, 3, 0))
    sid = torch.tensor([2], dtype=torch.int32, device="cuda")  # ring row 2 of 3
    kp, vp = kv_rows(seed, 0, 0, P - W, W, Hkv, d, device="cuda")
    hs.kv_pool_append(pool, 0, kp[None], vp[None], torch.tensor([P - W], device="cuda"), seq_ids=sid)
    q = q_rows(seed, 0, 0, P, Nc, Hq, d, device="cuda")[None]
    k, v = kv_rows(seed, 0, 0, P, Nc, Hkv, d, device="cuda")
    o = hs.swa_prefill_fwd(pool, 0, q, k[None], v[None], start_pos=torch.tensor([P], device="cuda"), seq_ids=sid)
    assert hs.hswa_pool_check_error(pool) == 0
    rows = _sample_rows(seed, Nc, [0, 1, 126, 127, 128, 129, 255, 256, 8191, 8192, Nc - 1], 48)
    kc, vc = kv_rows(seed, 0, 0, P - W + 1, Nc + W - 1, Hkv, d)
    qc = _q_rows_cpu(seed, 0, 0, P, rows, Hq, d)
    ref = oracle.attention(qc, P + np.array(rows), kc, vc, W, key_base=P - W + 1)
    compare(o[0, rows], ref, "W=128 chunk after 131072")


def test_full_layer_paged_prefix_1024_units():
    P, Nc, Hq, Hkv, d = 16384, 4096, 64, 8, 128
    seed = 3103
    total = P + Nc
    n_pages = total // 64
    phys = n_pages + 7
    pool = hs.kv_pool_create(hs.PoolDesc(0, 1, 128, Hkv, d, 1, phys))
    pool.data.fill_(0xFF)  # unused page rows hold NaN bit patterns
    perm = synth.permutation(seed, synth.stream_id(synth.TAG_MISC, 31), phys)[:n_pages]
    pt = perm.view(1, n_pages).to(torch.int32).contiguous().cuda()
    for c0 in range(0, total, 4096):
        kf, vf = kv_rows(seed, 0, 0, c0, 4096, Hkv, d, device="cuda")
        hs.kv_pool_append(pool, 0, kf[None], vf[None], torch.tensor([c0], device="cuda"), page_table=pt)
    q = q_rows(seed, 0, 0, P, Nc, Hq, d, device="cuda")[None]
    o = hs.full_prefill_fwd(pool, 0, q, pt, start_pos=torch.tensor([P], device="cuda"))
    assert hs.hswa_pool_check_error(pool) == 0
    rows = _sample_rows(seed, Nc, [0, 1, 127, 128, 255, 256, 2047, 2048, Nc - 1], 16)
    kc, vc = kv_rows(seed, 0, 0, 0, total, Hkv, d)
    qc = _q_rows_cpu(seed, 0, 0, P, rows, Hq, d)
    ref = oracle.attention(qc, P + np.array(rows), kc, vc, 0)
    compare(o[0, rows], ref, "full layer, 16384 + 4096 keys")


def _decode_batch(seed, kv_format=hs.HSWA_KV_BF16, k_scales=None, v_scales=None):
    """The 256-sequence decode batch on a fresh pool (a W=128 ring layer 0, a paged full layer 1)."""
    n, nq, Hq, Hkv, d, W = 256, 4, 64, 8, 128, 128
    u = synth.uniform_float64(seed, synth.stream_id(synth.TAG_MISC, 41), n)
    lens = torch.floor(torch.exp(math.log(1024) + u * (math.log(262144) - math.log(1024)))).to(torch.int64)
    lens[int(torch.argmax(lens))] = 262144 - nq  # the longest sequence at the top of the range
    pps = (lens + nq + 63) // 64
    total_pages = int(pps.sum())
    pool = hs.kv_pool_create(hs.PoolDesc(1, 1, W, Hkv, d, n, total_pages, kv_format=kv_format))
    if kv_format == hs.HSWA_KV_FP8_E4M3:
        pool.data.fill_(0x7F)  # NaN codes wherever nothing was committed
        for layer in (0, 1):
            pool.set_scales(layer, k_scales, v_scales)
    perm = synth.permutation(seed, synth.stream_id(synth.TAG_MISC, 42), total_pages).to(torch.int32)
    pt = torch.zeros(n, int(pps.max()), dtype=torch.int32)
    off = 0
    for b in range(n):
        pt[b, :pps[b]] = perm[off:off + int(pps[b])]
        off += int(pps[b])
    pt = pt.cuda()
    sid = synth.permutation(seed, synth.stream_id(synth.TAG_MISC, 43), n).to(torch.int32).cuda()
    for b in range(n):
        L = int(lens[b])
        for c0 in range(0, L, 65536):
            m = min(65536, L - c0)
            kf, vf = kv_rows(seed, 1, b, c0, m, Hkv, d, device="cuda")
            hs.kv_pool_append(pool, 1, kf[None], vf[None], torch.tensor([c0], device="cuda"), page_table=pt[b:b + 1])
        kr, vr = kv_rows(seed, 0, b, L - W, W, Hkv, d, device="cuda")
        hs.kv_pool_append(pool, 0, kr[None], vr[None], torch.tensor([L - W], device="cuda"), seq_ids=sid[b:b + 1])
    ctx = lens.cuda()
    maxL = int(lens.max())
    ws = torch.empty(hs.hybrid_decode_workspace_size(pool, n, nq, Hq, maxL), dtype=torch.uint8, device="cuda")
    ws.fill_(0xAB)
    outs = {}
    for layer in (0, 1):
        q = torch.stack([q_rows(seed, layer, b, int(lens[b]), nq, Hq, d, device="cuda") for b in range(n)])
        kn = torch.stack([kv_rows(seed, layer, b, int(lens[b]), nq, Hkv, d, device="cuda")[0] for b in range(n)])
        vn = torch.stack([kv_rows(seed, layer, b, int(lens[b]), nq, Hkv, d, device="cuda")[1] for b in range(n)])
        kw = dict(seq_ids=sid) if layer == 0 else dict(page_table=pt)
        outs[layer] = hs.hybrid_decode_fwd(pool, layer, q, kn, vn, ctx, maxL, ws, **kw)
    assert hs.hswa_pool_check_error(pool) == 0
    return lens, outs, (nq, Hq, Hkv, d, W)


def test_hybrid_decode_256_sequences_full_size():
    seed = 3104
    lens, outs, (nq, Hq, Hkv, d, W) = _decode_batch(seed)
    order = torch.argsort(lens, descending=True).tolist()
    # full layer: every row of the 4 longest sequences (32 splits at 256K, merged)
    for b in order[:4]:
        L = int(lens[b])
        kc, vc = kv_rows(seed, 1, b, 0, L + nq, Hkv, d)
        qc = q_rows(seed, 1, b, L, nq, Hq, d)
        compare(outs[1][b], oracle.attention(qc, L + np.arange(nq), kc, vc, 0), f"full layer, L={L}")
        del kc, vc
    # ring layer: every row of 8 sequences, longest and shortest among them
    for b in order[:3] + order[-3:] + order[100:102]:
        L = int(lens[b])
        kc, vc = kv_rows(seed, 0, b, L - W + 1, W - 1 + nq, Hkv, d)
        qc = q_rows(seed, 0, b, L, nq, Hq, d)
        compare(outs[0][b], oracle.attention(qc, L + np.arange(nq), kc, vc, W, key_base=L - W + 1),
                f"ring layer, L={L}")


def test_hybrid_decode_256_sequences_fp8_full_size():
    """The same batch on an FP8 (E4M3) pool, against the oracle over the values the cache holds:
    E4M3_value(E4M3(fp32(x) / s)) * s per entry, the new tokens included (they enter as they will
    be stored)."""
    seed = 3105
    u = synth.uniform_float64(seed, synth.stream_id(synth.TAG_MISC, 62, 16), 16).numpy()
    ks = (0.25 + 2.25 * u[:8]).astype(np.float32)
    vs = (0.25 + 2.25 * u[8:]).astype(np.float32)
    lens, outs, (nq, Hq, Hkv, d, W) = _decode_batch(seed, hs.HSWA_KV_FP8_E4M3, ks, vs)
    lut = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))  # the oracle's value of every code

    def deq(x, scales):
        out = np.empty(tuple(x.shape), dtype=np.float64)
        for g in range(x.shape[1]):
            out[:, g] = lut[oracle.e4m3_quantize(x[:, g].contiguous(), scales[g])] * np.float64(scales[g])
        return out

    order = torch.argsort(lens, descending=True).tolist()
    # full layer: every row of the 2 longest sequences (32 and more splits merged) and 2 shorter ones
    for b in order[:2] + order[60:61] + order[-1:]:
        L = int(lens[b])
        kc, vc = kv_rows(seed, 1, b, 0, L + nq, Hkv, d)
        qc = q_rows(seed, 1, b, L, nq, Hq, d)
        ref = oracle.attention_kv64(qc, L + np.arange(nq), deq(kc, ks), deq(vc, vs), 0)
        compare(outs[1][b], ref, f"FP8 full layer, L={L}")
        del kc, vc, ref
    # ring layer: every row of 6 sequences
    for b in order[:3] + order[-3:]:
        L = int(lens[b])
        kc, vc = kv_rows(seed, 0, b, L - W + 1, W - 1 + nq, Hkv, d)
        qc = q_rows(seed, 0, b, L, nq, Hq, d)
        ref = oracle.attention_kv64(qc, L + np.arange(nq), deq(kc, ks), deq(vc, vs), W, key_base=L - W + 1)
        compare(outs[0][b], ref, f"FP8 ring layer, L={L}")
