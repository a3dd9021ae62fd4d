"""Pins for the fp64 oracle: values the pages print, closed forms, library routines
(torch's scaled_dot_product_attention in float64), special cases and invariants.

None of these re-types the oracle's loop: each compares it with something the
pages or the mathematics fix independently.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _bf16(shape, seed, tag, sigma=1.0):
    n = int(np.prod(shape))
    return synth.normal_bf16(seed, synth.stream_id(tag), 0, n, sigma).view(*shape)


def _f64(x):
    return x.to(torch.float64)


# ---------------------------------------------------------------- page values

def test_mask_counts_match_page(page_values):
    assert oracle.mask_count(32, 0) == int(page_values["full_causal_nonzeros_n32"])
    assert oracle.mask_count(32, 32) == 528 == 32 * 33 // 2
    c = oracle.mask_count(32, 8)
    assert c <= int(page_values["swa_nonzeros_upper_bound_n32_w8"])
    # closed form: the first w rows hold 1..w keys, every later row exactly w
    assert c == 8 * 9 // 2 + (32 - 8) * 8 == 228


@pytest.mark.parametrize("n,w", [(1, 1), (5, 1), (7, 3), (16, 16), (16, 40), (33, 8), (64, 17)])
def test_mask_count_closed_form(n, w):
    expect = n * (n + 1) // 2 if w >= n else w * (w + 1) // 2 + (n - w) * w
    assert oracle.mask_count(n, w) == expect


def test_ring_trace_matches_page(page_values):
    s5 = [int(x) for x in page_values["ring_w4_after_step5"].split(",")]
    s7 = [int(x) for x in page_values["ring_w4_after_step7"].split(",")]
    assert list(oracle.ring_trace(6, 4)) == s5
    assert list(oracle.ring_trace(8, 4)) == s7
    # memory stays w slots; the slots hold exactly the last w positions
    for t in range(0, 40):
        held = sorted(p for p in oracle.ring_trace(t, 5) if p >= 0)
        assert held == list(range(max(0, t - 5), t))


def test_kv_bytes_match_page(page_values):
    assert oracle.kv_bytes(1, 32, 32768, 128) == int(page_values["kv_bytes_full_mha_layer"])
    assert oracle.kv_bytes(1, 8, 4096, 128) == int(page_values["kv_bytes_swa_gqa_layer"])
    mib = 1 << 20
    assert oracle.kv_bytes(32, 8, 4096, 128) // mib == int(page_values["kv_mb_swa_gqa_32_layers"])
    assert oracle.kv_bytes(32, 32, 32768, 128) // mib == int(page_values["kv_mb_full_mha_32_layers_n32768"])
    assert oracle.kv_bytes(32, 32, 131072, 128) // mib == int(page_values["kv_mb_full_mha_32_layers_n131072"])


def test_hybrid_ratio_tends_to_one_seventh(page_values):
    n_swa, n_full, w = (int(x) for x in page_values["hybrid_layers"].split(","))
    limit = float(page_values["hybrid_ratio_asymptote"])
    prev = 2.0
    for logn in range(8, 31):
        r = oracle.hybrid_kv_ratio(n_swa, n_full, w, 1 << logn)
        assert r < prev and r > limit
        prev = r
    assert abs(oracle.hybrid_kv_ratio(n_swa, n_full, w, 1 << 30) - limit) < 1e-6
    # N = W: every layer keeps N slots, ratio 1
    assert oracle.hybrid_kv_ratio(n_swa, n_full, w, w) == 1.0
    # the 1M-token figure the pages quote as "about 7.0x"
    assert round(1.0 / oracle.hybrid_kv_ratio(n_swa, n_full, w, 1 << 20), 1) == 7.0


def test_pool_bytes_dual_pool_footprint():
    # 60 SWA layers with a 128-slot ring + 10 full layers holding 2^20 tokens,
    # Hkv = 8, d = 128, bf16: 30 MiB + 40 GiB
    swa, full = oracle.pool_bytes(60, 10, 128, 8, 128, 64, 1, (1 << 20) // 64)
    assert swa == 31_457_280 and full == 42_949_672_960
    # the SWA pool does not depend on N
    swa2, _ = oracle.pool_bytes(60, 10, 128, 8, 128, 64, 1, 1)
    assert swa2 == swa


# ---------------------------------------------------------------- attention vs library

def _sdpa_rows(q, k, v, rows, window):
    """Per-row torch SDPA (float64, no mask) over the slice of keys in the window."""
    n, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    kr = _f64(k).repeat_interleave(g, dim=1)  # [n, hq, d]
    vr = _f64(v).repeat_interleave(g, dim=1)
    out = torch.empty(len(rows), hq, d, dtype=torch.float64)
    for r, i in enumerate(rows):
        lo = 0 if window == 0 else max(0, i - window + 1)
        qq = _f64(q[i]).unsqueeze(1)                 # [hq, 1, d]
        kk = kr[lo:i + 1].transpose(0, 1)            # [hq, cnt, d]
        vv = vr[lo:i + 1].transpose(0, 1)
        out[r] = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0, :]
    return out


@pytest.mark.parametrize("n,hq,hkv,d,window", [
    (37, 4, 2, 16, 0), (37, 4, 1, 16, 5), (50, 8, 2, 32, 1), (29, 3, 3, 8, 29), (64, 4, 4, 64, 13)])
def test_attention_matches_sdpa(n, hq, hkv, d, window):
    q = _bf16((n, hq, d), 11, synth.TAG_Q)
    k = _bf16((n, hkv, d), 11, synth.TAG_K)
    v = _bf16((n, hkv, d), 11, synth.TAG_V)
    got = oracle.attention(q, np.arange(n), k, v, window)
    ref = _sdpa_rows(q, k, v, list(range(n)), window).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_full_causal_matches_sdpa_is_causal():
    n, h, d = 45, 4, 32
    q = _bf16((n, h, d), 5, synth.TAG_Q)
    k = _bf16((n, h, d), 5, synth.TAG_K)
    v = _bf16((n, h, d), 5, synth.TAG_V)
    got = oracle.attention(q, np.arange(n), k, v, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        _f64(q).transpose(0, 1), _f64(k).transpose(0, 1), _f64(v).transpose(0, 1), is_causal=True)
    np.testing.assert_allclose(got, ref.transpose(0, 1).numpy(), rtol=0, atol=1e-12)


def test_window_at_least_n_is_full_causal():
    n, h, d = 40, 2, 16
    q, k, v = (_bf16((n, h, d), 9, t) for t in (synth.TAG_Q, synth.TAG_K, synth.TAG_V))
    full = oracle.attention(q, np.arange(n), k, v, 0)
    for w in (n, n + 1, 4 * n):
        assert np.array_equal(oracle.attention(q, np.arange(n), k, v, w), full)
    assert not np.allclose(oracle.attention(q, np.arange(n), k, v, n - 1), full)


def test_window_one_returns_own_value():
    n, hq, hkv, d = 33, 4, 2, 16
    q = _bf16((n, hq, d), 3, synth.TAG_Q)
    k = _bf16((n, hkv, d), 3, synth.TAG_K)
    v = _bf16((n, hkv, d), 3, synth.TAG_V)
    got = oracle.attention(q, np.arange(n), k, v, 1)
    expect = _f64(v).repeat_interleave(hq // hkv, dim=1).numpy()
    assert np.array_equal(got, expect)


@pytest.mark.parametrize("window", [1, 4, 9, 0])
def test_zero_query_gives_window_mean(window):
    n, h, d = 30, 2, 8
    q = torch.zeros(n, h, d, dtype=torch.bfloat16)
    k = _bf16((n, h, d), 4, synth.TAG_K)
    v = _bf16((n, h, d), 4, synth.TAG_V)
    got = oracle.attention(q, np.arange(n), k, v, window)
    vf = _f64(v).numpy()
    for i in range(n):
        lo = 0 if window == 0 else max(0, i - window + 1)
        np.testing.assert_allclose(got[i], vf[lo:i + 1].mean(axis=0), rtol=0, atol=1e-14)


def test_equal_keys_give_uniform_weights():
    n, h, d = 20, 1, 8
    q = _bf16((n, h, d), 6, synth.TAG_Q)
    k = _bf16((1, h, d), 6, synth.TAG_K).expand(n, h, d).contiguous()
    v = _bf16((n, h, d), 6, synth.TAG_V)
    got = oracle.attention(q, np.arange(n), k, v, 6)
    vf = _f64(v).numpy()
    for i in range(n):
        np.testing.assert_allclose(got[i], vf[max(0, i - 5):i + 1].mean(axis=0), atol=1e-13)


def test_constant_values_pass_through():
    n, h, d = 25, 2, 16
    q = _bf16((n, h, d), 7, synth.TAG_Q)
    k = _bf16((n, h, d), 7, synth.TAG_K)
    v = torch.full((n, h, d), 0.375, dtype=torch.bfloat16)
    got = oracle.attention(q, np.arange(n), k, v, 7)
    np.testing.assert_allclose(got, 0.375, rtol=0, atol=1e-15)


def test_gqa_equals_mha_with_repeated_heads():
    n, hq, hkv, d = 31, 8, 2, 16
    q = _bf16((n, hq, d), 8, synth.TAG_Q)
    k = _bf16((n, hkv, d), 8, synth.TAG_K)
    v = _bf16((n, hkv, d), 8, synth.TAG_V)
    a = oracle.attention(q, np.arange(n), k, v, 6)
    b = oracle.attention(q, np.arange(n), k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), 6)
    assert np.array_equal(a, b)
    # and a different head grouping (interleaved) would give another answer
    c = oracle.attention(q, np.arange(n), k.repeat(1, 4, 1), v.repeat(1, 4, 1), 6)
    assert not np.allclose(a, c)


def test_key_base_slice_is_equivalent():
    n, h, d, w = 60, 2, 16, 8
    q = _bf16((n, h, d), 12, synth.TAG_Q)
    k = _bf16((n, h, d), 12, synth.TAG_K)
    v = _bf16((n, h, d), 12, synth.TAG_V)
    rows = np.arange(40, 60)
    full = oracle.attention(q[40:], rows, k, v, w)
    base = 40 - w + 1
    part = oracle.attention(q[40:], rows, k[base:], v[base:], w, key_base=base)
    assert np.array_equal(full, part)
    with pytest.raises(ValueError):
        oracle.attention(q[40:], rows, k[base + 1:], v[base + 1:], w, key_base=base + 1)


def test_softmax_weights_shift_invariance():
    # adding a constant to every score of a row (q . k_j + c) leaves the output unchanged:
    # give every key an extra coordinate with value 1 and the query a constant there.
    n, d = 24, 16
    q = _bf16((n, 1, d), 13, synth.TAG_Q).float()
    k = _bf16((n, 1, d), 13, synth.TAG_K).float()
    v = _bf16((n, 1, d), 13, synth.TAG_V)
    q0 = q.clone(); q0[..., -1] = 0
    k1 = k.clone(); k1[..., -1] = 1
    q1 = q0.clone(); q1[..., -1] = 2.0
    a = oracle.attention(q0.bfloat16(), np.arange(n), k1.bfloat16(), v, 5)
    b = oracle.attention(q1.bfloat16(), np.arange(n), k1.bfloat16(), v, 5)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- window_safe_len

def _closed_form_wsl(m, c, bits, w):
    """Closed form derived from the definition: with the ring holding [max(0, c - w), c), a cached
    length above w is resumable only in full (every slot valid and m >= c), otherwise the answer is
    min(m, c, first invalid slot)."""
    if c > w:
        return c if (m >= c and all(bits)) else 0
    first_bad = next((s for s in range(w) if not bits[s]), w)
    return min(m, c, first_bad)


def _pack(bits_rows, w):
    words = (w + 31) // 32
    out = np.zeros((len(bits_rows), words), dtype=np.uint32)
    for r, bits in enumerate(bits_rows):
        for s, b in enumerate(bits):
            if b:
                out[r, s // 32] |= np.uint32(1 << (s % 32))
    return out


@pytest.mark.parametrize("w", [1, 2, 3, 4, 5])
def test_window_safe_len_closed_form_exhaustive(w):
    ms, cs, bs = [], [], []
    for mask in range(1 << w):
        bits = [(mask >> s) & 1 for s in range(w)]
        for c in range(0, 3 * w + 2):
            for m in range(0, 3 * w + 3):
                ms.append(m); cs.append(c); bs.append(bits)
    got = oracle.window_safe_len(ms, cs, _pack(bs, w), w)
    expect = [_closed_form_wsl(m, c, b, w) for m, c, b in zip(ms, cs, bs)]
    assert list(got) == expect


def test_window_safe_len_invariants_random():
    rng = np.random.default_rng(0)
    for w in (8, 33, 128):
        n = 400
        c = rng.integers(0, 4 * w, n)
        m = np.where(rng.random(n) < 0.5, c, rng.integers(0, 4 * w, n))
        bits = (rng.random((n, w)) > 0.02).astype(int)
        bits[: n // 3] = 1
        got = oracle.window_safe_len(m, c, _pack(bits.tolist(), w), w)
        for r in range(n):
            L = int(got[r])
            assert 0 <= L <= m[r] and L <= c[r]
            ring_lo = max(0, c[r] - w)
            for p in range(max(0, L - w), L):  # every admitted tail position is resident
                assert ring_lo <= p < c[r] and bits[r][p % w]
            assert L == _closed_form_wsl(int(m[r]), int(c[r]), bits[r].tolist(), w)


def test_window_safe_len_reading_literal_w_tail():
    # the slot of position C - W is the one whose eviction separates the readings:
    # with the literal tail of W tokens the match must drop to 0.
    w, c = 8, 20
    bits = [1] * w
    bits[c % w] = 0
    assert oracle.window_safe_len([c], [c], _pack([bits], w), w)[0] == 0
    bits = [1] * w
    assert oracle.window_safe_len([c], [c], _pack([bits], w), w)[0] == c
    assert oracle.window_safe_len([c + 5], [c], _pack([bits], w), w)[0] == c
    assert oracle.window_safe_len([c - 1], [c], _pack([bits], w), w)[0] == 0
