"""GPU: sliding-window and full prefill on tensor cores against the fp64 oracle.

Cases span several 128-row tiles, ragged tails, prefixes that are and are not
128-aligned (rolling-buffer rows via TMA and via cp.async), GQA ratios, head_dim
64/128, and the degenerate windows W = 1 and W >= N.
"""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import compare, kv_rows, page_table_for, q_rows

pytestmark = pytest.mark.gpu


def run_swa_case(seed, B, n_q, W, hq, hkv, d, starts, sigma=1.0, layer=0, rows=None):
    """SWA chunk prefill with per-sequence prefixes held in the ring; returns (gpu out, oracle out)."""
    desc = hs.PoolDesc(n_swa_layers=layer + 1, n_full_layers=0, window=W, n_kv_heads=hkv, head_dim=d,
                       max_seqs=B + 1, pages_per_full_layer=0)
    pool = hs.kv_pool_create(desc)
    pool.data.fill_(0xFF)  # NaN bit patterns everywhere the kernel must not read
    seq_ids = torch.arange(B, dtype=torch.int32).flip(0) + 1  # ring rows 1..B, reversed
    qs, ks, vs = [], [], []
    for b in range(B):
        P = starts[b]
        lo = max(0, P - W)
        if P > lo:  # commit the prefix window [P - W, P) into the ring
            kp, vp = kv_rows(seed, layer, b, lo, P - lo, hkv, d, sigma)
            hs.kv_pool_append(pool, layer, kp[None].cuda(), vp[None].cuda(),
                              torch.tensor([lo], dtype=torch.int64).cuda(), seq_ids=seq_ids[b:b + 1].cuda())
        k, v = kv_rows(seed, layer, b, P, n_q, hkv, d, sigma)
        ks.append(k); vs.append(v)
        qs.append(q_rows(seed, layer, b, P, n_q, hq, d, sigma))
    q = torch.stack(qs).cuda(); k = torch.stack(ks).cuda(); v = torch.stack(vs).cuda()
    sp = torch.tensor(starts, dtype=torch.int64).cuda()
    any_prefix = any(s > 0 for s in starts)
    o = hs.swa_prefill_fwd(pool, layer, q, k, v, start_pos=sp if any_prefix else None,
                           seq_ids=seq_ids.cuda() if any_prefix else None)
    assert hs.hswa_pool_check_error(pool) == 0
    outs, refs = [], []
    for b in range(B):
        P = starts[b]
        base = max(0, P - W + 1)
        kk, vv = kv_rows(seed, layer, b, base, P + n_q - base, hkv, d, sigma)
        r = np.arange(n_q) if rows is None else np.asarray(rows)
        refs.append(oracle.attention(qs[b][r], P + r, kk, vv, W, key_base=base))
        outs.append(o[b, r])
    return torch.stack(outs), np.stack(refs)


@pytest.mark.parametrize("W", [128, 512, 1])
def test_single_swa_layer_n512_gqa4(W):
    # B=1, N=512, Hq=4, Hkv=1, d=64, inputs N(0,1) rounded to bf16; W=512 is full causal
    got, ref = run_swa_case(101, 1, 512, W, 4, 1, 64, [0])
    compare(got, ref, f"W={W}")


def test_w_ge_n_equals_full_causal_on_gpu():
    got_a, _ = run_swa_case(102, 1, 300, 300, 2, 1, 64, [0])
    got_b, ref = run_swa_case(102, 1, 300, 4096, 2, 1, 64, [0])
    compare(got_b, ref, "W=4096")
    assert torch.equal(got_a.view(torch.int16), got_b.view(torch.int16))


def test_w1_returns_own_value():
    got, ref = run_swa_case(103, 1, 200, 1, 4, 2, 128, [0])
    compare(got, ref, "W=1")
    _, v = kv_rows(103, 0, 0, 0, 200, 2, 128)
    # o_i = v_i up to the bf16 output rounding of an fp32 1.0 * v (exact)
    assert torch.equal(got[0].cpu()[:, ::2].contiguous().view(torch.int16), v.view(torch.int16))


@pytest.mark.parametrize("n_q,W,hq,hkv,d", [(300, 100, 8, 2, 128), (1000, 256, 4, 4, 64), (129, 129, 2, 1, 128),
                                            (700, 1000, 16, 2, 64)])
def test_ragged_and_unaligned_windows(n_q, W, hq, hkv, d):
    got, ref = run_swa_case(104, 2, n_q, W, hq, hkv, d, [0, 0])
    compare(got, ref, f"n_q={n_q} W={W}")


@pytest.mark.parametrize("starts,W,n_q", [([128, 1024], 128, 300),       # aligned: ring tiles by TMA
                                          ([131, 5000], 128, 260),       # unaligned: cp.async ring rows
                                          ([40, 0], 128, 200),           # prefix shorter than W
                                          ([4096, 8192], 512, 640),      # W multiple of 128, several ring tiles
                                          ([77, 300], 100, 150),         # W not a multiple of 128
                                          ([1, 2], 1, 64)])              # W = 1 with a prefix
def test_chunk_after_prefix_reads_the_ring(starts, W, n_q):
    got, ref = run_swa_case(105, 2, n_q, W, 8, 2, 128, starts)
    compare(got, ref, f"starts={starts} W={W}")


def test_chunked_equals_one_shot():
    # the same sequence prefilled as one chunk or as two chunks through the ring
    seed, W, hq, hkv, d, N, split = 106, 256, 4, 2, 128, 900, 384
    one, _ = run_swa_case(seed, 1, N, W, hq, hkv, d, [0])
    second, ref = run_swa_case(seed, 1, N - split, W, hq, hkv, d, [split])
    compare(second, ref[:, :], "second chunk")
    # the second chunk's rows equal rows split.. of the one-shot output up to accumulation order
    diff = (one[0, split:].float() - second[0].float()).abs().max().item()
    assert diff <= 2e-2


def run_full_case(seed, B, n_q, hq, hkv, d, starts, layer=0, total_pages=None, rows=None):
    lens = [s + n_q for s in starts]
    max_pages = max((l + 63) // 64 for l in lens)
    total_pages = total_pages or B * max_pages + 3
    desc = hs.PoolDesc(n_swa_layers=0, n_full_layers=layer + 1, window=1, n_kv_heads=hkv, head_dim=d,
                       max_seqs=0, pages_per_full_layer=total_pages)
    pool = hs.kv_pool_create(desc)
    pool.data.fill_(0xFF)
    pt = page_table_for(seed, B, max_pages, total_pages).cuda()
    qs = []
    for b in range(B):
        k, v = kv_rows(seed, layer, b, 0, lens[b], hkv, d)
        hs.kv_pool_append(pool, layer, k[None].cuda(), v[None].cuda(), torch.zeros(1, dtype=torch.int64).cuda(),
                          page_table=pt[b:b + 1].contiguous())
        qs.append(q_rows(seed, layer, b, starts[b], n_q, hq, d))
    q = torch.stack(qs).cuda()
    o = hs.full_prefill_fwd(pool, layer, q, pt, start_pos=torch.tensor(starts, dtype=torch.int64).cuda())
    assert hs.hswa_pool_check_error(pool) == 0
    outs, refs = [], []
    for b in range(B):
        k, v = kv_rows(seed, layer, b, 0, lens[b], hkv, d)
        r = np.arange(n_q) if rows is None else np.asarray(rows)
        refs.append(oracle.attention(qs[b][r], starts[b] + r, k, v, 0))
        outs.append(o[b, r])
    return torch.stack(outs), np.stack(refs)


@pytest.mark.parametrize("starts,n_q,hq,hkv,d", [([0, 0], 256, 4, 1, 64), ([1000, 0], 300, 8, 2, 128),
                                                 ([130, 64], 129, 16, 2, 128), ([5000, 3333], 512, 8, 8, 64)])
def test_full_prefill_paged(starts, n_q, hq, hkv, d):
    got, ref = run_full_case(107, 2, n_q, hq, hkv, d, starts)
    compare(got, ref, f"full starts={starts}")


def test_full_prefill_page_permutation_invariance():
    # the same logical K/V under two different random page tables gives identical output
    a, _ = run_full_case(108, 1, 200, 4, 1, 128, [700], total_pages=40)
    b, _ = run_full_case(108, 1, 200, 4, 1, 128, [700], total_pages=64)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
