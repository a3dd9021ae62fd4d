"""Multi-rank plumbing of bench.py on CPU with the gloo backend (world size 2): the step time is the
max over ranks, throughput is weak-scaling (per-rank units x ranks / slowest time), and the
reference arm prints from rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, ws, port, q):
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        ms = [12.5, 20.0][rank]
        bench.barrier(ws)
        m = bench.max_over_ranks(ms, ws)
        v = bench.weak_scaling_value(1e12, ws, m, 1e9)
        q.put((rank, m, v))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, m, v in got:
        assert m == 20.0                       # slowest rank
        assert abs(v - 2 * 1e12 / 20.0 / 1e9) < 1e-9  # both ranks' units over the slowest time


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""
    env["RANK"] = "0"
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600)
    assert out.returncode == 0
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # the same workload description, metric and unit as the GPU arm's line (what the two arms'
    # ratio is computed over)
    sys.path.insert(0, ROOT)
    import bench
    assert line["config"] == bench.SwaPrefill16k.config(2)  # WORLD_SIZE = 2 in this run
    assert line["metric"] == json.load(open(os.path.join(ROOT, "BASELINE.json")))["metric"]
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True


# ---------------------------------------------------------------- the multi-GPU partition

def _shard_worker(rank, ws, port, out_q):
    """One rank: the KV-head shard of a prefill and the sequence shard of a decode step, computed
    with the fp64 oracle on the CPU, gathered over gloo and put back together."""
    import numpy as np
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import hybrid_sliding_window_swa_b200 as hs
    import oracle
    from hswa_testlib import kv_rows, q_rows
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # prefill, split by KV head: Hq = 8, Hkv = 4, G = 2, W = 9
        n, hq, hkv, d, W = 40, 8, 4, 32, 9
        G = hq // hkv
        g0, g1 = hs.hswa_shard_kv_heads(hkv, ws, rank)
        qa = q_rows(91, 0, 0, 0, n, hq, d)
        k, v = kv_rows(91, 0, 0, 0, n, hkv, d)
        mine = oracle.attention(qa[:, g0 * G:g1 * G].contiguous(), np.arange(n), k[:, g0:g1].contiguous(),
                                v[:, g0:g1].contiguous(), W)
        parts = [torch.empty((n, (g1 - g0) * G, d), dtype=torch.float64) for _ in range(ws)]
        torch.distributed.all_gather(parts, torch.from_numpy(mine))
        o_prefill = torch.cat(parts, dim=1).numpy()  # rank-major head slices = head order
        # decode, split by sequence
        lens = np.array([3000, 17, 70000, 900, 264000, 5, 65536, 65535, 12000, 262144, 1], dtype=np.int64)
        ranks, loads = hs.hswa_shard_sequences(lens, ws)
        res = {}
        for b in np.nonzero(ranks == rank)[0]:
            L = int(lens[b])
            lo = max(0, L - 200)  # a 200-token window keeps the oracle quick
            kk, vv = kv_rows(92, 0, int(b), lo, L + 4 - lo, hkv, d)
            qq = q_rows(92, 0, int(b), L, 4, hq, d)
            res[int(b)] = oracle.attention(qq, L + np.arange(4), kk, vv, 200, key_base=lo)
        gathered = [None] * ws
        torch.distributed.all_gather_object(gathered, res)
        merged = {}
        for r in gathered:
            assert not (set(r) & set(merged))  # a sequence lives on one rank
            merged.update(r)
        out_q.put((rank, o_prefill, merged, ranks, loads))
    finally:
        torch.distributed.destroy_process_group()


def test_kv_head_and_sequence_shards_reassemble_the_single_rank_result():
    import numpy as np
    import oracle
    import hybrid_sliding_window_swa_b200 as hs
    from hswa_testlib import kv_rows, q_rows
    hs.load_library()
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = 29700 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, out_q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [out_q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    n, hq, hkv, d, W = 40, 8, 4, 32, 9
    want = oracle.attention(q_rows(91, 0, 0, 0, n, hq, d), np.arange(n), *kv_rows(91, 0, 0, 0, n, hkv, d), W)
    lens = [3000, 17, 70000, 900, 264000, 5, 65536, 65535, 12000, 262144, 1]
    for rank, o_prefill, merged, ranks, loads in got:
        assert np.array_equal(o_prefill, want)  # every head computed once, in place
        assert sorted(merged) == list(range(len(lens)))
        for b, L in enumerate(lens):
            lo = max(0, L - 200)
            kk, vv = kv_rows(92, 0, b, lo, L + 4 - lo, hkv, d)
            ref = oracle.attention(q_rows(92, 0, b, L, 4, hq, d), L + np.arange(4), kk, vv, 200, key_base=lo)
            assert np.array_equal(merged[b], ref)
        assert int(loads.sum()) == sum(lens)


def test_sequence_split_is_longest_first_and_within_the_greedy_bound():
    # Longest-first greedy onto the least-loaded rank keeps the largest rank load within
    # (4/3 - 1/(3m)) of the best split (Graham's bound); checked against brute force on small cases.
    import itertools
    import numpy as np
    import hybrid_sliding_window_swa_b200 as hs
    rng = np.random.default_rng(3)
    for trial in range(60):
        m = int(rng.integers(2, 4))
        n = int(rng.integers(1, 9))
        lens = np.exp(rng.uniform(np.log(1024), np.log(1 << 20), n)).astype(np.int64)
        ranks, loads = hs.hswa_shard_sequences(lens, m)
        assert ((ranks >= 0) & (ranks < m)).all()
        assert np.array_equal(np.bincount(ranks, weights=lens, minlength=m).astype(np.int64), loads)
        best = min(max(sum(int(lens[i]) for i in range(n) if a[i] == r) for r in range(m))
                   for a in itertools.product(range(m), repeat=n))
        assert loads.max() <= (4 / 3 - 1 / (3 * m)) * best + 1e-9
    # the same lengths in another order give the same loads; ties go to the lowest rank
    lens = np.array([5, 5, 5, 5], dtype=np.int64)
    ranks, loads = hs.hswa_shard_sequences(lens, 2)
    assert list(ranks) == [0, 1, 0, 1] and list(loads) == [10, 10]


def test_kv_head_ranges_cover_every_head_once():
    import hybrid_sliding_window_swa_b200 as hs
    for hkv, m in [(8, 1), (8, 2), (8, 4), (8, 8), (6, 3)]:
        ranges = [hs.hswa_shard_kv_heads(hkv, m, r) for r in range(m)]
        assert ranges[0][0] == 0 and ranges[-1][1] == hkv
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        assert len({e - b for b, e in ranges}) == 1
    with pytest.raises(hs.HswaError):
        hs.hswa_shard_kv_heads(8, 3, 0)  # 8 heads do not split over 3 ranks


def test_partition_edge_cases():
    """No sequences; more ranks than sequences (one per rank, longest on rank 0, the rest empty);
    zero-length contexts; and the arguments the calls refuse."""
    import numpy as np
    import hybrid_sliding_window_swa_b200 as hs
    ranks, loads = hs.hswa_shard_sequences(np.zeros(0, dtype=np.int64), 4)
    assert ranks.size == 0 and list(loads) == [0, 0, 0, 0]
    lens = np.array([70000, 300000, 1024, 65536], dtype=np.int64)  # three length buckets
    ranks, loads = hs.hswa_shard_sequences(lens, 6)
    assert list(ranks) == [1, 0, 3, 2]  # placed longest first, each onto the next empty rank
    assert list(loads) == [300000, 70000, 65536, 1024, 0, 0]
    ranks, loads = hs.hswa_shard_sequences(np.array([0, 0, 7], dtype=np.int64), 2)
    assert list(ranks) == [1, 1, 0] and list(loads) == [7, 0]  # the 7 first; the empty ones join the least loaded
    with pytest.raises(hs.HswaError):
        hs.hswa_shard_sequences(np.array([5, -1], dtype=np.int64), 2)
    with pytest.raises(hs.HswaError):
        hs.hswa_shard_sequences(np.array([5], dtype=np.int64), 0)
    for hkv, m, r in [(8, 2, 2), (8, 2, -1), (8, 0, 0), (0, 1, 0)]:
        with pytest.raises(hs.HswaError):
            hs.hswa_shard_kv_heads(hkv, m, r)
