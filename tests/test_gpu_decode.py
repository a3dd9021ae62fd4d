"""GPU: hybrid decode (1 token + drafts per sequence, split-KV) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import compare, kv_rows, page_table_for, q_rows

pytestmark = pytest.mark.gpu


def run_decode_case(seed, lens, n_qt, hq, hkv, d, W, kind, layer_swa=0, n_swa=1, n_full=1,
                    rows_of=None, max_ctx=None):
    """kind 'swa' uses ring layer `layer_swa`; kind 'full' uses the pool's first full layer."""
    n = len(lens)
    max_ctx = max_ctx or max(lens)
    pages_per_seq = (max_ctx + n_qt + 63) // 64
    total_pages = n * pages_per_seq + 5 if kind == "full" else 1
    desc = hs.PoolDesc(n_swa_layers=n_swa, n_full_layers=n_full, window=W, n_kv_heads=hkv, head_dim=d,
                       max_seqs=n + 2, pages_per_full_layer=total_pages)
    pool = hs.kv_pool_create(desc)
    pool.data.fill_(0xFF)
    layer = layer_swa if kind == "swa" else n_swa
    seq_ids = (torch.arange(n, dtype=torch.int32) * 7 % (n + 2)).contiguous()
    pt = page_table_for(seed, n, pages_per_seq, total_pages).cuda() if kind == "full" else None
    for b, L in enumerate(lens):
        if kind == "swa":
            lo = max(0, L - W)
            if L > lo:
                k, v = kv_rows(seed, layer, b, lo, L - lo, hkv, d)
                hs.kv_pool_append(pool, layer, k[None].cuda(), v[None].cuda(), torch.tensor([lo]).cuda(),
                                  seq_ids=seq_ids[b:b + 1].cuda())
        elif L > 0:
            k, v = kv_rows(seed, layer, b, 0, L, hkv, d)
            hs.kv_pool_append(pool, layer, k[None].cuda(), v[None].cuda(), torch.tensor([0]).cuda(),
                              page_table=pt[b:b + 1].contiguous())
    qs, kn, vn = [], [], []
    for b, L in enumerate(lens):
        qs.append(q_rows(seed, layer, b, L, n_qt, hq, d))
        k, v = kv_rows(seed, layer, b, L, n_qt, hkv, d)
        kn.append(k); vn.append(v)
    q = torch.stack(qs).cuda(); k_new = torch.stack(kn).cuda(); v_new = torch.stack(vn).cuda()
    ctx = torch.tensor(lens, dtype=torch.int64).cuda()
    ws = torch.empty(hs.hybrid_decode_workspace_size(pool, n, n_qt, hq, max_ctx), dtype=torch.uint8, device="cuda")
    ws.fill_(0xAB)
    o = hs.hybrid_decode_fwd(pool, layer, q, k_new, v_new, ctx, max_ctx, ws,
                             seq_ids=seq_ids.cuda() if kind == "swa" else None, page_table=pt)
    assert hs.hswa_pool_check_error(pool) == 0
    window = W if kind == "swa" else 0
    outs, refs = [], []
    for b, L in enumerate(lens):
        base = max(0, L - W + 1) if kind == "swa" else 0
        k, v = kv_rows(seed, layer, b, base, L + n_qt - base, hkv, d)
        refs.append(oracle.attention(qs[b], L + np.arange(n_qt), k, v, window, key_base=base))
        outs.append(o[b])
    return torch.stack(outs), np.stack(refs), o


@pytest.mark.parametrize("W", [128, 4, 1, 300])
def test_swa_decode_ring(W):
    lens = [0, 1, 3, 127, 128, 129, 1000, 4099, 70000]
    got, ref, _ = run_decode_case(201, lens, 4, 16, 2, 128, W, "swa")
    compare(got, ref, f"swa W={W}")


@pytest.mark.parametrize("lens,n_qt,hq,hkv,d", [
    ([0, 5, 64, 65, 8191, 8192, 8193, 17000], 4, 16, 2, 128),  # split boundaries (8192-key splits)
    ([20000, 1, 12345], 4, 32, 4, 128),                         # 8 rows per KV head
    ([300, 5000], 1, 8, 1, 64),                                 # single token, MHA-like group of 8
    ([1024, 777, 50000], 2, 4, 4, 64),                          # G = 1
])
def test_full_decode_paged(lens, n_qt, hq, hkv, d):
    got, ref, _ = run_decode_case(202, lens, n_qt, hq, hkv, d, 128, "full")
    compare(got, ref, f"full lens={lens}")


def test_decode_rows_equal_prefill_rows():
    # draft t of a decode step equals row L+t of a full-causal chunk prefill over the same keys
    from test_gpu_prefill import run_full_case
    L, n_qt = 700, 4
    got_dec, ref_dec, _ = run_decode_case(203, [L], n_qt, 8, 2, 128, 128, "full", n_swa=0)
    got_pre, ref_pre = run_full_case(203, 1, n_qt, 8, 2, 128, [L])
    assert np.array_equal(ref_dec, ref_pre)  # same logical inputs on both paths
    compare(got_dec, ref_dec, "decode")
    assert (got_dec.float() - got_pre.float()).abs().max().item() <= 2e-2


def test_ctx_len_above_declared_max_is_reported():
    desc = hs.PoolDesc(n_swa_layers=0, n_full_layers=1, window=128, n_kv_heads=1, head_dim=64, max_seqs=1,
                       pages_per_full_layer=4)
    pool = hs.kv_pool_create(desc)
    pool.data.zero_()
    q = torch.zeros(1, 1, 1, 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(hs.hybrid_decode_workspace_size(pool, 1, 1, 1, 100), dtype=torch.uint8, device="cuda")
    pt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    hs.hybrid_decode_fwd(pool, 0, q, q, q, torch.tensor([200], device="cuda"), 100, ws, page_table=pt)
    assert hs.hswa_pool_check_error(pool) == hs.HSWA_ERR_DEVICE_BOUNDS


def test_context_too_long_for_the_split_merge_is_rejected_before_launch():
    # max_ctx_len near 2^31 means ~262K splits of one sequence: their merge factors need far more
    # shared memory than a block may use, so both entry points refuse before launching anything
    import ctypes
    desc = hs.PoolDesc(n_swa_layers=0, n_full_layers=1, window=128, n_kv_heads=8, head_dim=128, max_seqs=1,
                       pages_per_full_layer=4)
    pool = hs.kv_pool_create(desc)
    q = torch.zeros(1, 4, 64, 128, dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros(1, 4, 8, 128, dtype=torch.bfloat16, device="cuda")
    ctx = torch.zeros(1, dtype=torch.int64, device="cuda")
    pt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    lib = hs.load_library()
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    big = (1 << 31) - 8192
    rc = lib.hybrid_decode_fwd(pool.handle, 0, vp(q), vp(kn), vp(kn), vp(q), 1, 4, vp(ctx), big, None, vp(pt), 4, 64,
                               None, 0, None)
    assert rc == hs.HSWA_ERR_UNSUPPORTED_SHAPE and "shared memory" in lib.hswa_last_error().decode()
    rc = lib.hybrid_decode_fwd_noalloc(pool.handle, 0, vp(q), vp(kn), vp(kn), vp(q), 1, 4, vp(ctx), big, None,
                                       vp(pt), 4, 64, None)
    assert rc == hs.HSWA_ERR_UNSUPPORTED_SHAPE and "shared memory" in lib.hswa_last_error().decode()
    assert hs.hswa_pool_check_error(pool) == 0


@pytest.mark.skipif(torch.cuda.device_count() < 2, reason="needs two GPUs")
def test_calls_with_another_device_current_are_rejected():
    desc = hs.PoolDesc(n_swa_layers=1, n_full_layers=0, window=128, n_kv_heads=1, head_dim=64, max_seqs=1,
                       pages_per_full_layer=0)
    with torch.cuda.device(0):
        pool = hs.kv_pool_create(desc, device="cuda:0")
        q = torch.zeros(1, 128, 1, 64, dtype=torch.bfloat16, device="cuda:0")
    with torch.cuda.device(1):
        with pytest.raises(hs.HswaError) as e:
            hs.swa_prefill_fwd(pool, 0, q, q, q)
        assert e.value.code == hs.HSWA_ERR_INVALID_ARG and "device" in str(e.value)
