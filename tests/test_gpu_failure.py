"""GPU: a bounded wait that runs out is reported, not hung: the library's wait gives up after its
limit, records HSWA_ERR_TIMEOUT in the pool's error word, and the context keeps working.
Nothing here faults, traps or hangs the GPU (the wait is limited to 50 ms)."""
import numpy as np
import pytest
import torch

import oracle
import hybrid_sliding_window_swa_b200 as hs
from hswa_testlib import compare, kv_rows, q_rows

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_context_survives():
    desc = hs.PoolDesc(n_swa_layers=1, n_full_layers=0, window=64, n_kv_heads=1, head_dim=64, max_seqs=1,
                       pages_per_full_layer=0)
    pool = hs.kv_pool_create(desc)
    assert hs.hswa_pool_check_error(pool) == 0
    hs.hswa_selftest_wait_timeout(pool, 50_000_000)
    assert hs.hswa_pool_check_error(pool) == hs.HSWA_ERR_TIMEOUT
    assert hs.hswa_pool_check_error(pool) == 0  # read and cleared
    # a pending error makes compute calls on the pool skip their work ...
    hs.hswa_selftest_wait_timeout(pool, 1_000_000)
    q = q_rows(5, 0, 0, 0, 200, 2, 64)
    k, v = kv_rows(5, 0, 0, 0, 200, 1, 64)
    o = torch.zeros(1, 200, 2, 64, dtype=torch.bfloat16, device="cuda")
    hs.swa_prefill_fwd(pool, 0, q[None].cuda(), k[None].cuda(), v[None].cuda(), o=o)
    assert hs.hswa_pool_check_error(pool) == hs.HSWA_ERR_TIMEOUT
    assert float(o.float().abs().sum()) == 0.0
    # ... and once it is cleared the same context computes correctly
    hs.swa_prefill_fwd(pool, 0, q[None].cuda(), k[None].cuda(), v[None].cuda(), o=o)
    assert hs.hswa_pool_check_error(pool) == 0
    compare(o[0], oracle.attention(q, np.arange(200), k, v, 64), "after timeout")


def test_selftest_limit_is_validated_on_the_host():
    desc = hs.PoolDesc(1, 0, 64, 1, 64, 1, 0)
    lib = hs.load_library()
    assert lib.hswa_selftest_wait_timeout(None, 50_000_000, None) == hs.HSWA_ERR_INVALID_ARG
