"""The seeded generator: deterministic, row-addressable, and N(0, sigma^2) shaped."""
import numpy as np
import torch

import synth


def test_rows_regenerate_independently():
    s = synth.stream_id(synth.TAG_K, 3, 7)
    whole = synth.normal_bf16(42, s, 0, 10_000)
    part = synth.normal_bf16(42, s, 1234, 777)
    assert torch.equal(whole[1234:2011].view(torch.int16), part.view(torch.int16))
    rows = synth.normal_bf16_rows(42, s, 5, 3, 100)
    assert torch.equal(rows.reshape(-1).view(torch.int16), whole[500:800].view(torch.int16))


def test_streams_and_seeds_differ():
    a = synth.normal_bf16(1, synth.stream_id(synth.TAG_Q), 0, 4096)
    b = synth.normal_bf16(2, synth.stream_id(synth.TAG_Q), 0, 4096)
    c = synth.normal_bf16(1, synth.stream_id(synth.TAG_K), 0, 4096)
    assert not torch.equal(a, b) and not torch.equal(a, c)


def test_normal_moments_and_bins():
    for sigma in (1.0, 2 ** -0.5):
        x = synth.normal_bf16(7, synth.stream_id(synth.TAG_V), 0, 1 << 21, sigma).double().numpy()
        assert abs(x.mean()) < 3e-3
        assert abs(x.std() / sigma - 1) < 3e-3
        # mass within one and two sigma of a normal law
        assert abs(np.mean(np.abs(x) < sigma) - 0.682689) < 2e-3
        assert abs(np.mean(np.abs(x) < 2 * sigma) - 0.954500) < 1e-3


def test_values_are_bf16_round_to_nearest_of_the_table_bins():
    thr, val = synth.normal_table(1.0)
    assert torch.all(thr[1:] > thr[:-1])
    v = val.view(torch.bfloat16).double()
    assert torch.all(v[1:] > v[:-1])
    assert len(val) == len(thr) + 1


def test_uniform_int_range_and_permutation():
    u = synth.uniform_int(3, synth.stream_id(synth.TAG_MISC), 10000, 5, 17)
    assert int(u.min()) == 5 and int(u.max()) == 17
    p = synth.permutation(3, synth.stream_id(synth.TAG_MISC, 1), 1000)
    assert sorted(p.tolist()) == list(range(1000))


def test_c_and_torch_generators_agree_bitwise():
    s = synth.stream_id(synth.TAG_K, 1, 2)
    for sigma in (1.0, 2 ** -0.5):
        a = synth.normal_bf16(5, s, 1000, 300_000, sigma, use_c=False)
        b = synth.normal_bf16(5, s, 1000, 300_000, sigma, use_c=True)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
