"""GPU: the hybrid 70-layer schedule (60 sliding-window layers + 10 full layers, "MiMo v2.5
inference optimisation", section "architecture") run on one chunk after a cached prefix, every
layer checked against the oracle on sampled rows, and the dual-pool footprint checked against
(60 W + 10 N) token-slots."""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import compare, kv_rows, q_rows

pytestmark = pytest.mark.gpu


def test_seventy_layer_chunk_after_prefix():
    seed, n_swa, n_full, W = 31, 60, 10, 128
    Hq, Hkv, d = 8, 2, 128
    P, Nc = 1536, 512            # cached prefix, then one chunk
    N = P + Nc
    pages = N // 64
    desc = hs.PoolDesc(n_swa_layers=n_swa, n_full_layers=n_full, window=W, n_kv_heads=Hkv, head_dim=d, max_seqs=1,
                       pages_per_full_layer=pages)
    _, swa_bytes, full_bytes = hs.kv_pool_layout(desc)
    slot_bytes = 2 * Hkv * d * 2
    assert swa_bytes + full_bytes == (n_swa * W + n_full * N) * slot_bytes
    pool = hs.kv_pool_create(desc)
    pool.data.fill_(0xFF)
    pt = torch.arange(pages, dtype=torch.int32).flip(0).view(1, pages).contiguous().cuda()
    sid = torch.zeros(1, dtype=torch.int32).cuda()
    start = torch.tensor([P], dtype=torch.int64).cuda()
    rows = np.array([0, 1, 127, 128, 300, Nc - 1])
    # layer order: the pages give only the counts, so SWA and full layers are interleaved 6:1
    order = []
    for blk in range(n_full):
        order += [("swa", blk * 6 + i) for i in range(6)] + [("full", n_swa + blk)]
    assert len(order) == 70
    for kind, layer in order:
        q = q_rows(seed, layer, 0, P, Nc, Hq, d)
        if kind == "swa":
            kp, vp = kv_rows(seed, layer, 0, P - W, W, Hkv, d)
            hs.kv_pool_append(pool, layer, kp[None].cuda(), vp[None].cuda(), torch.tensor([P - W]).cuda(), seq_ids=sid)
            k, v = kv_rows(seed, layer, 0, P, Nc, Hkv, d)
            o = hs.swa_prefill_fwd(pool, layer, q[None].cuda(), k[None].cuda(), v[None].cuda(), start_pos=start,
                                   seq_ids=sid)
            kk, vv = kv_rows(seed, layer, 0, P - W + 1, Nc + W - 1, Hkv, d)
            ref = oracle.attention(q[rows], P + rows, kk, vv, W, key_base=P - W + 1)
        else:
            k, v = kv_rows(seed, layer, 0, 0, N, Hkv, d)
            hs.kv_pool_append(pool, layer, k[None].cuda(), v[None].cuda(), torch.zeros(1, dtype=torch.int64).cuda(),
                              page_table=pt)
            o = hs.full_prefill_fwd(pool, layer, q[None].cuda(), pt, start_pos=start)
            ref = oracle.attention(q[rows], P + rows, k, v, 0)
        compare(o[0, rows], ref, f"{kind} layer {layer}")
    assert hs.hswa_pool_check_error(pool) == 0
