"""GPU: seeded generator agreement, window_safe_len (bit-exact) and KV commit placement (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import kv_rows, page_table_for

pytestmark = pytest.mark.gpu


def test_generator_cpu_and_gpu_agree_bitwise():
    s = synth.stream_id(synth.TAG_K, 2, 5)
    for sigma in (1.0, 2 ** -0.5):
        a = synth.normal_bf16(99, s, 12345, 1 << 20, sigma, "cpu")
        b = synth.normal_bf16(99, s, 12345, 1 << 20, sigma, "cuda").cpu()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def _wsl_requests(seed, n, w, max_len):
    """Requests shaped like the decode workload: C uniform in [0, max_len] (1/8 forced <= W),
    m = C half the time else uniform, masks all-valid / sparse evictions / one evicted slot C mod W."""
    C = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 1), n, 0, max_len).numpy()
    small = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 2), n, 0, w).numpy()
    kind = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 3), n, 0, 7).numpy()
    C = np.where(kind == 0, small, C)
    mu = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 4), n, 0, max_len).numpy()
    coin = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 5), n, 0, 1).numpy()
    M = np.where(coin == 0, C, mu)
    mk = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 6), n, 0, 3).numpy()
    ev = synth.uniform_int(seed, synth.stream_id(synth.TAG_MISC, 7), n * w, 0, 63).numpy().reshape(n, w)
    bits = np.ones((n, w), dtype=np.int64)
    bits = np.where((mk[:, None] == 2) & (ev == 0), 0, bits)
    one = (mk == 3)
    bits[one, (C[one] % w)] = 0
    words = (w + 31) // 32
    packed = np.zeros((n, words), dtype=np.uint32)
    for s in range(w):
        packed[:, s // 32] |= (bits[:, s].astype(np.uint32) << np.uint32(s % 32))
    return M.astype(np.int64), C.astype(np.int64), packed


@pytest.mark.parametrize("w,n,max_len", [(128, 4096, 262144), (8, 3000, 40), (1, 500, 10), (33, 2000, 200),
                                         (4096, 256, 20000)])
def test_window_safe_len_bit_exact(w, n, max_len):
    M, C, packed = _wsl_requests(7 + w, n, w, max_len)
    ref = oracle.window_safe_len(M, C, packed, w)
    got = hs.window_safe_len(torch.from_numpy(M).cuda(), torch.from_numpy(C).cuda(),
                             torch.from_numpy(packed.view(np.int32)).cuda(), w)
    assert np.array_equal(got.cpu().numpy(), ref)


def test_window_safe_len_exhaustive_small():
    for w in (1, 2, 3, 5):
        ms, cs, rows = [], [], []
        for mask in range(1 << w):
            for c in range(0, 3 * w + 2):
                for m in range(0, 3 * w + 3):
                    ms.append(m); cs.append(c); rows.append(mask)
        packed = np.array(rows, dtype=np.uint32).reshape(-1, 1)
        ref = oracle.window_safe_len(ms, cs, packed, w)
        got = hs.window_safe_len(torch.tensor(ms).cuda(), torch.tensor(cs).cuda(),
                                 torch.from_numpy(packed.view(np.int32)).cuda(), w)
        assert np.array_equal(got.cpu().numpy(), ref)


@pytest.mark.parametrize("w,hkv,d", [(4, 1, 64), (128, 8, 128), (100, 2, 64)])
def test_ring_append_places_slot_pos_mod_w(w, hkv, d):
    seed, layer, n_seqs = 3, 1, 3
    desc = hs.PoolDesc(n_swa_layers=2, n_full_layers=0, window=w, n_kv_heads=hkv, head_dim=d, max_seqs=4,
                       pages_per_full_layer=0)
    pool = hs.kv_pool_create(desc)
    pool.data.zero_()
    seq_ids = torch.tensor([2, 0, 3], dtype=torch.int32)
    # append in several calls of different lengths: positions 0..T-1 per sequence
    T = 3 * w + 5
    pos = 0
    for n_tok in (1, w - 1 if w > 1 else 1, 2 * w + 3, T):
        n_tok = min(n_tok, T - pos)
        if n_tok <= 0:
            break
        ks, vs = zip(*[kv_rows(seed, layer, b, pos, n_tok, hkv, d) for b in range(n_seqs)])
        hs.kv_pool_append(pool, layer, torch.stack(ks).cuda(), torch.stack(vs).cuda(),
                          torch.full((n_seqs,), pos, dtype=torch.int64).cuda(), seq_ids=seq_ids.cuda())
        pos += n_tok
    torch.cuda.synchronize()
    assert hs.hswa_pool_check_error(pool) == 0
    ring = pool.ring.cpu()
    held = oracle.ring_trace(pos, w)  # position held by each slot
    for b in range(n_seqs):
        k_all, v_all = kv_rows(seed, layer, b, 0, pos, hkv, d)
        for s_ in range(w):
            p_ = held[s_]
            assert torch.equal(ring[0, seq_ids[b], layer, :, s_].view(torch.int16), k_all[p_].view(torch.int16))
            assert torch.equal(ring[1, seq_ids[b], layer, :, s_].view(torch.int16), v_all[p_].view(torch.int16))
    # untouched ring rows stay zero
    assert int(ring[:, 1].abs().sum()) == 0 and int(ring[:, :, 0].abs().sum()) == 0


def test_page_append_follows_page_table():
    seed, hkv, d = 4, 2, 128
    desc = hs.PoolDesc(n_swa_layers=1, n_full_layers=2, window=128, n_kv_heads=hkv, head_dim=d, max_seqs=1,
                       pages_per_full_layer=40)
    pool = hs.kv_pool_create(desc)
    pool.data.zero_()
    n_seqs, n_tok = 2, 300  # 5 pages each, last one partial
    pt = page_table_for(seed, n_seqs, 8, 40)
    layer = 2  # second full layer
    ks, vs = zip(*[kv_rows(seed, layer, b, 0, n_tok, hkv, d) for b in range(n_seqs)])
    # commit in two chunks with an unaligned boundary
    for a, n in ((0, 77), (77, n_tok - 77)):
        hs.kv_pool_append(pool, layer, torch.stack([k[a:a + n] for k in ks]).cuda(),
                          torch.stack([v[a:a + n] for v in vs]).cuda(),
                          torch.full((n_seqs,), a, dtype=torch.int64).cuda(), page_table=pt.cuda())
    assert hs.hswa_pool_check_error(pool) == 0
    pages = pool.pages.cpu()
    for b in range(n_seqs):
        for p_ in range(n_tok):
            page = int(pt[b, p_ // 64])
            assert torch.equal(pages[0, 1, page, :, p_ % 64].view(torch.int16), ks[b][p_].view(torch.int16))
            assert torch.equal(pages[1, 1, page, :, p_ % 64].view(torch.int16), vs[b][p_].view(torch.int16))
    assert int(pages[:, 0].abs().sum()) == 0  # the other full layer is untouched


def test_bad_page_id_is_recorded_not_written():
    desc = hs.PoolDesc(n_swa_layers=0, n_full_layers=1, window=1, n_kv_heads=1, head_dim=64, max_seqs=0,
                       pages_per_full_layer=4)
    pool = hs.kv_pool_create(desc)
    pool.data.zero_()
    k = torch.ones(1, 64, 1, 64, dtype=torch.bfloat16, device="cuda")
    pt = torch.tensor([[7]], dtype=torch.int32, device="cuda")  # page 7 does not exist
    hs.kv_pool_append(pool, 0, k, k, torch.zeros(1, dtype=torch.int64, device="cuda"), page_table=pt)
    assert hs.hswa_pool_check_error(pool) == hs.HSWA_ERR_DEVICE_BOUNDS
    assert hs.hswa_pool_check_error(pool) == 0  # cleared
    assert int(pool.pages.float().abs().sum()) == 0
