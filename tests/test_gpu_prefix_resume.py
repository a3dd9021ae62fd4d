"""GPU: resuming a request from a prefix-cache match on the dual pool.

"MiMo v2.5 inference optimisation", section "KV cache redesign": a prefix-cache match is cut to
the window-safe length L, so that the W positions before L still have their sliding-window KV,
and prefill resumes at L. Here two cached sequences on one token path, A (1000 tokens, ring row
0) and its prefix A2 (900 tokens, ring row 1), sit in the prefix tree and in the pool (rings hold
their windows, the full layer's pages hold A's positions, which A2 shares). One position of A's
window is evicted (and its ring slot overwritten with NaN). A request R shares 950 tokens with A,
then continues with its own. The tree gives L and, per ring slot, the ring row that holds the
position the resumed window needs there; kv_pool_gather_ring builds R's ring from them (R's ring
starts as NaN). R's page table shares A's pages before L, with a private copy of the page that
holds L (R writes into it). The SWA and full prefills of R's chunk [L, 1150) then run on the pool
and are compared with the fp64 oracle over R's whole logical sequence, whose keys come from the
seeded generator: positions < 950 from A's stream, the rest from R's own.
"""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import compare, kv_rows, q_rows

pytestmark = pytest.mark.gpu

SEED, W, HQ, HKV, D = 4401, 128, 8, 2, 128
SHARED, N_R = 950, 1150  # R shares tokens [0, 950) with A; R has 1150 tokens


def _path_kv(layer, lo, hi):
    """K/V of R's logical positions [lo, hi): A's stream before SHARED, R's own from there."""
    parts = []
    if lo < min(hi, SHARED):
        parts.append(kv_rows(SEED, layer, 0, lo, min(hi, SHARED) - lo, HKV, D))
    if max(lo, SHARED) < hi:
        parts.append(kv_rows(SEED, layer, 1, max(lo, SHARED), hi - max(lo, SHARED), HKV, D))
    return torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])


def _path_q(layer, lo, hi):
    parts = []
    if lo < min(hi, SHARED):
        parts.append(q_rows(SEED, layer, 0, lo, min(hi, SHARED) - lo, HQ, D))
    if max(lo, SHARED) < hi:
        parts.append(q_rows(SEED, layer, 1, max(lo, SHARED), hi - max(lo, SHARED), HQ, D))
    return torch.cat(parts)


def test_resume_from_prefix_tree_match_on_the_pool():
    dev = "cuda"
    tokens_a = np.arange(1, 1201, dtype=np.int32)
    A, A2 = tokens_a[:1000], tokens_a[:900]
    R = np.concatenate([tokens_a[:SHARED], np.arange(100001, 100001 + N_R - SHARED, dtype=np.int32)])

    tree = hs.PrefixTree(W)
    tree.insert(A, 0)
    tree.insert(A2, 1)
    evict = 930
    assert tree.evict_swa(A, evict, evict + 1) == 1
    m, L, owners = tree.match_slots(R)
    ops = [("insert", A, 0), ("insert", A2, 1), ("evict", A, evict, evict + 1), ("match_slots", R)]
    m2, L2, sets = oracle.prefix_cache_replay(W, ops)[0]
    assert (m, L) == (m2, L2) == (SHARED, evict)
    for s in range(W):
        assert (int(owners[s]) in sets[s]) if sets[s] else owners[s] == -1

    n_pages_phys = 64
    pool = hs.kv_pool_create(hs.PoolDesc(1, 1, W, HKV, D, 3, n_pages_phys))
    pool.data.fill_(0xFF)  # every slot and page row NaN until written
    # cached state: rings of A (row 0) and A2 (row 1), A's pages on the full layer
    pt_a = torch.arange(16, dtype=torch.int32).flip(0).view(1, 16).contiguous().to(dev)  # 1024 positions
    for row, n in ((0, 1000), (1, 900)):
        k, v = kv_rows(SEED, 0, 0, n - W, W, HKV, D, device=dev)
        hs.kv_pool_append(pool, 0, k[None], v[None], torch.tensor([n - W], device=dev),
                          seq_ids=torch.tensor([row], dtype=torch.int32, device=dev))
    k, v = kv_rows(SEED, 1, 0, 0, 1000, HKV, D, device=dev)
    hs.kv_pool_append(pool, 1, k[None], v[None], torch.tensor([0], device=dev), page_table=pt_a)
    # the eviction: A's ring slot of position 930 no longer holds valid KV
    pool.ring[:, 0, 0, :, evict % W].fill_(float("nan"))

    # resume R at L: its ring (row 2) from the rings that hold [L - W, L)
    hs.kv_pool_gather_ring(pool, 0, 2, torch.from_numpy(owners).to(dev))
    # R's pages: A's pages below the page that holds L, a private copy of that page, fresh ones after
    lp = L // 64
    fresh = torch.arange(32, 32 + (N_R + 63) // 64 - lp, dtype=torch.int32)
    pt_r = torch.cat([pt_a[0, :lp].cpu(), fresh]).view(1, -1).contiguous().to(dev)
    pool.pages[:, 0, int(fresh[0])].copy_(pool.pages[:, 0, int(pt_a[0, lp])])

    start = torch.tensor([L], device=dev)
    sid = torch.tensor([2], dtype=torch.int32, device=dev)
    # sliding-window layer: chunk [L, N_R) against the gathered ring
    kc, vc = _path_kv(0, L, N_R)
    qc = _path_q(0, L, N_R)
    o_swa = hs.swa_prefill_fwd(pool, 0, qc[None].to(dev), kc[None].to(dev), vc[None].to(dev), start_pos=start,
                               seq_ids=sid)
    # full layer: append the chunk through R's pages, then attend all of [0, N_R)
    kf, vf = _path_kv(1, L, N_R)
    hs.kv_pool_append(pool, 1, kf[None].to(dev), vf[None].to(dev), start, page_table=pt_r)
    qf = _path_q(1, L, N_R)
    o_full = hs.full_prefill_fwd(pool, 1, qf[None].to(dev), pt_r, start_pos=start)
    assert hs.hswa_pool_check_error(pool) == 0

    pos = L + np.arange(N_R - L)
    ks, vs = _path_kv(0, L - W + 1, N_R)
    compare(o_swa[0], oracle.attention(qc, pos, ks, vs, W, key_base=L - W + 1), "resumed SWA layer")
    ka, va = _path_kv(1, 0, N_R)
    compare(o_full[0], oracle.attention(qf, pos, ka, va, 0), "resumed full layer")
    # A's cached pages are untouched by R's writes
    ka_pages = pool.pages[0, 0, pt_a[0].long()].permute(0, 2, 1, 3).reshape(-1, HKV, D)[:1000]
    assert torch.equal(ka_pages.cpu(), kv_rows(SEED, 1, 0, 0, 1000, HKV, D)[0])
    tree.close()


def test_gather_ring_rejects_bad_arguments_and_records_bad_rows():
    pool = hs.kv_pool_create(hs.PoolDesc(1, 1, 64, 1, 64, 2, 2))
    pool.data.zero_()
    src = torch.full((64,), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(hs.HswaError):
        hs.kv_pool_gather_ring(pool, 1, 0, src)   # layer 1 is a full layer
    with pytest.raises(hs.HswaError):
        hs.kv_pool_gather_ring(pool, 0, 2, src)   # ring rows are 0 and 1
    src[5] = 7                                    # a source row the pool does not have
    hs.kv_pool_gather_ring(pool, 0, 0, src)
    assert hs.hswa_pool_check_error(pool) == hs.HSWA_ERR_DEVICE_BOUNDS
