"""CPU: the SWA-aware prefix cache (token trie with per-position sliding-window retention and the
window-safe match, "MiMo v2.5 inference optimisation", section "KV cache redesign").

The brute-force model in the oracle is pinned to the window_safe_len closed form (one cached
sequence whose ring slots are valid or not reduces to exactly that case) and to a worked example;
the library's hswa_tree_* calls are then checked against the model on random operation streams
with shared prefixes, releases and evictions. All results are exact integers.
"""
import numpy as np
import pytest

import oracle
import hybrid_sliding_window_swa_b200 as hs


def _single_sequence_case(C, m, W, valid_bits):
    """Tree-model ops for one cached sequence of length C whose ring slot s is valid iff bit s of
    valid_bits is set, queried with a request that matches min(m, C) tokens."""
    seq = list(range(1, C + 1))
    ops = [("insert", seq)]
    for p in range(max(0, C - W), C):
        if not (valid_bits >> (p % W)) & 1:
            ops.append(("evict", seq, p, p + 1))
    k = min(m, C)
    query = seq[:k] + [-(i + 1) for i in range(m - k)]  # tokens the tree does not hold
    ops.append(("match", query))
    return ops


@pytest.mark.parametrize("W", [1, 3, 8])
def test_model_reduces_to_window_safe_len(W):
    rng = np.random.default_rng(11 + W)
    rows = []
    for C in range(0, 3 * W + 3):
        for m in range(0, C + 3):
            for _ in range(3):
                bits = int(rng.integers(0, 1 << W))
                if rng.random() < 0.4:
                    bits = (1 << W) - 1
                rows.append((C, m, bits))
    got = [oracle.prefix_cache_replay(W, _single_sequence_case(C, m, W, bits))[0][1] for C, m, bits in rows]
    words = (W + 31) // 32
    mask = np.zeros((len(rows), words), dtype=np.uint32)
    for r, (_, _, bits) in enumerate(rows):
        mask[r, 0] = bits
    ref = oracle.window_safe_len(np.array([m for _, m, _ in rows], dtype=np.int64),
                                 np.array([C for C, _, _ in rows], dtype=np.int64), mask, W)
    assert np.array_equal(np.asarray(got, dtype=np.int64), np.asarray(ref, dtype=np.int64))


def test_worked_example():
    # W = 4. A = tokens 1..10 (positions 0..9); its window holds positions 6..9.
    # B = 1,2,3,4,5,20,21 shares positions 0..4 with A; its window holds positions 3..6, i.e.
    # positions 3 and 4 of the shared path and B's own positions 5 and 6.
    W = 4
    A = list(range(1, 11))
    B = [1, 2, 3, 4, 5, 20, 21]
    ops = [("insert", A), ("insert", B),
           ("match", A),            # m = 10; [6, 10) held (A's window)               -> L = 10
           ("match", A[:8]),        # m = 8; every L in 1..8 needs a position among 0..2 or
                                    # A's position 5 (token 6), none of them held     -> L = 0
           ("match", B),            # m = 7; [3, 7) held (B's window)                 -> L = 7
           ("match", B[:5] + [99]), # m = 5; [1, 5) needs positions 1, 2              -> L = 0
           ("release", B),          # B's window no longer counts
           ("match", B),            # m = 7; [3, 7) not held any more                 -> L = 0
           ("match", A)]            # A's window untouched                            -> L = 10
    assert oracle.prefix_cache_replay(W, ops) == [(10, 10), (8, 0), (7, 7), (5, 0), (7, 0), (10, 10)]
    assert _replay_library(W, ops) == [(10, 10), (8, 0), (7, 7), (5, 0), (7, 0), (10, 10)]


def _random_ops(rng, W, n_ops, alpha, owners=False):
    base = [list(rng.integers(0, alpha, size=int(rng.integers(0, 30)))) for _ in range(3)]
    cached = []
    ops = []
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.3:
            b = base[int(rng.integers(0, 3))]
            seq = b[:int(rng.integers(0, len(b) + 1))] + list(rng.integers(0, alpha, size=int(rng.integers(0, 12))))
            own = int(rng.integers(0, 4)) if owners else -1
            ops.append(("insert", seq, own))
            cached.append((seq, own))
        elif r < 0.4 and cached:
            seq, own = cached.pop(int(rng.integers(0, len(cached))))
            ops.append(("release", seq, own))
        elif r < 0.55 and cached:
            seq = cached[int(rng.integers(0, len(cached)))][0]
            lo = int(rng.integers(0, len(seq) + 2))
            ops.append(("evict", seq, lo, lo + int(rng.integers(0, 6))))
        else:
            if cached and rng.random() < 0.7:
                src = cached[int(rng.integers(0, len(cached)))][0]
                q = src[:int(rng.integers(0, len(src) + 1))] + list(rng.integers(0, alpha, size=int(rng.integers(0, 4))))
            else:
                q = list(rng.integers(0, alpha, size=int(rng.integers(0, 20))))
            ops.append(("match_slots" if owners else "match", q))
    return ops


def _replay_library(W, ops):
    t = hs.PrefixTree(W)
    out = []
    for op in ops:
        if op[0] == "insert":
            t.insert(op[1], *op[2:])
        elif op[0] == "release":
            t.release(op[1], *op[2:])
        elif op[0] == "evict":
            t.evict_swa(op[1], op[2], op[3])
        elif op[0] == "match_slots":
            out.append(t.match_slots(op[1]))
        else:
            out.append(t.match(op[1]))
    t.close()
    return out


@pytest.mark.parametrize("W,alpha,seed", [(1, 3, 1), (3, 3, 2), (4, 2, 3), (8, 5, 4), (16, 4, 5)])
def test_library_matches_model(W, alpha, seed):
    rng = np.random.default_rng(seed)
    for _ in range(20):
        ops = _random_ops(rng, W, 60, alpha)
        assert _replay_library(W, ops) == oracle.prefix_cache_replay(W, ops)


@pytest.mark.parametrize("W,alpha,seed", [(1, 3, 11), (3, 3, 12), (4, 2, 13), (8, 5, 14)])
def test_library_slot_owners_match_model(W, alpha, seed):
    # with owners (ring rows): every slot of the resumed window names one of the model's holders of
    # the position it keeps, and the other slots are -1
    rng = np.random.default_rng(seed)
    for _ in range(20):
        ops = _random_ops(rng, W, 60, alpha, owners=True)
        got = _replay_library(W, ops)
        want = oracle.prefix_cache_replay(W, ops)
        assert len(got) == len(want)
        for (m, L, slots), (m2, L2, sets) in zip(got, want):
            assert (m, L) == (m2, L2)
            for s in range(W):
                if sets[s]:
                    assert int(slots[s]) in sets[s], (s, slots, sets)
                else:
                    assert slots[s] == -1


def test_owner_released_after_eviction_and_reinsert():
    # A's window covers position 5; it is evicted, then B (same path) is inserted and holds it
    # afresh; releasing A must not take B's copy away
    W = 4
    A = [1, 2, 3, 4, 5, 6]
    B = A + [7]
    ops = [("insert", A, 0), ("evict", A, 5, 6), ("insert", B, 1), ("release", A, 0), ("match_slots", B)]
    want = oracle.prefix_cache_replay(W, ops)
    assert want[0][:2] == (7, 7) and want[0][2][5 % W] == {1}
    got = _replay_library(W, ops)
    assert got[0][:2] == (7, 7) and list(got[0][2]) == [1, 1, 1, 1]


def test_batch_equals_single_and_stats():
    rng = np.random.default_rng(7)
    t = hs.PrefixTree(8)
    seqs = [list(rng.integers(0, 4, size=int(rng.integers(1, 60)))) for _ in range(40)]
    for s in seqs:
        t.insert(s)
    queries = [s[:int(rng.integers(0, len(s) + 1))] + [9] for s in seqs] + [[]]
    m, L = t.match_batch(queries)
    single = [t.match(q) for q in queries]
    assert [(int(a), int(b)) for a, b in zip(m, L)] == single
    n_pos, n_held = t.stats()
    assert n_pos == len({tuple(s[:p + 1]) for s in seqs for p in range(len(s))})
    assert 0 < n_held <= n_pos
    assert all(b <= a for a, b in zip(m, L))


def test_errors():
    with pytest.raises(hs.HswaError) as e:
        hs.PrefixTree(0)
    assert e.value.code == hs.HSWA_ERR_INVALID_ARG
    t = hs.PrefixTree(4)
    t.insert([1, 2, 3])
    with pytest.raises(hs.HswaError) as e:
        t.release([1, 2, 9])  # not cached
    assert e.value.code == hs.HSWA_ERR_INVALID_ARG
    assert t.match([]) == (0, 0)
    assert t.evict_swa([5, 6], 0, 10) == 0  # nothing cached on that path


def test_release_needs_an_insert_of_exactly_those_tokens():
    # A release undoes one insert of the same tokens. Releasing a cached prefix that was never
    # inserted on its own, or releasing one insert twice, would take window counts that belong
    # to other cached sequences; both are rejected and leave the state unchanged.
    W = 4
    A = list(range(1, 11))
    t = hs.PrefixTree(W)
    t.insert(A)
    t.insert(A[:6])
    for bad in (A[:8], A[:3], A + [99]):
        with pytest.raises(hs.HswaError) as e:
            t.release(bad)
        assert e.value.code == hs.HSWA_ERR_INVALID_ARG
        with pytest.raises(ValueError):
            oracle.prefix_cache_replay(W, [("insert", A), ("insert", A[:6]), ("release", bad)])
    # the rejected releases changed nothing: both windows still count
    assert t.match(A) == (10, 10)
    assert t.match(A[:6]) == (6, 6)
    with pytest.raises(hs.HswaError):
        t.release(A[:6], 3)  # inserted by owner -1, not by owner 3
    t.release(A[:6])
    with pytest.raises(hs.HswaError):
        t.release(A[:6])  # its one insert is already undone
    with pytest.raises(ValueError):
        oracle.prefix_cache_replay(W, [("insert", A), ("insert", A[:6]), ("release", A[:6]),
                                       ("release", A[:6])])
    assert t.match(A[:6]) == (6, 0)
    assert t.match(A) == (10, 10)
    # two inserts of the same tokens take two releases
    t.insert(A)
    t.release(A)
    assert t.match(A) == (10, 10)
    t.release(A)
    assert t.match(A) == (10, 0)
    t.release([])  # the empty sequence: nothing to undo, accepted
    ops = [("insert", A), ("insert", A[:6]), ("insert", A), ("release", A[:6]), ("release", A),
           ("match", A), ("release", A), ("match", A), ("match", A[:6]), ("release", [])]
    assert oracle.prefix_cache_replay(W, ops) == [(10, 10), (10, 0), (6, 0)]
    t.close()
