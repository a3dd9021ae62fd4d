"""Shared helpers for the tests: seeded logical K/V/Q, pool filling, oracle comparison.

Keys and values are generated per (layer, sequence) as one logical stream indexed by
absolute position, so the oracle can regenerate any window without reading the pool.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

ATOL_MAX = 2e-2   # max-abs error bound vs fp64 (bf16 inputs, bf16 output)
ATOL_MEAN = 2e-3  # mean-abs error bound


def kv_rows(seed, layer, seq, pos0, n, hkv, d, sigma=1.0, device="cpu"):
    """K and V rows for positions pos0 .. pos0+n-1 of (layer, seq): two [n, hkv, d] bf16 tensors."""
    k = synth.normal_bf16_rows(seed, synth.stream_id(synth.TAG_K, layer, seq), pos0, n, hkv * d, sigma, device)
    v = synth.normal_bf16_rows(seed, synth.stream_id(synth.TAG_V, layer, seq), pos0, n, hkv * d, sigma, device)
    return k.view(n, hkv, d), v.view(n, hkv, d)


def q_rows(seed, layer, seq, pos0, n, hq, d, sigma=1.0, device="cpu"):
    q = synth.normal_bf16_rows(seed, synth.stream_id(synth.TAG_Q, layer, seq), pos0, n, hq * d, sigma, device)
    return q.view(n, hq, d)


def compare(got: torch.Tensor, ref: np.ndarray, what: str = ""):
    """Element-wise check of a bf16 GPU result against fp64 oracle values."""
    g = got.detach().float().cpu().double().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def page_table_for(seed, n_seqs, pages_per_seq, total_pages, stream_tag=0):
    """Row b: a seeded random choice of distinct physical pages (no sharing across rows)."""
    perm = synth.permutation(seed, synth.stream_id(synth.TAG_MISC, 77, stream_tag), total_pages)
    need = n_seqs * pages_per_seq
    assert need <= total_pages
    return perm[:need].view(n_seqs, pages_per_seq).to(torch.int32).contiguous()
