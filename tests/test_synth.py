"""The seeded input generator: published constants, rounding, distribution, slicing, host/device agreement."""
import numpy as np
import pytest

import synth


def test_splitmix64_reference_output():
    # splitmix64 seeded with state 0: its first output is mix(0 + golden gamma), a published value
    # (the reference C implementation by Vigna prints 0xe220a8397b1dcdaf first).
    x = synth._mix_np(np.array([0x9E3779B97F4A7C15], dtype=np.uint64))[0]
    assert int(x) == 0xE220A8397B1DCDAF


def test_bf16_rounding_matches_torch():
    import torch

    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38 / 4])])
    ours = synth.f64_to_bf16_bits(x)
    theirs = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)
    back = synth.bf16_bits_to_f64(ours)
    assert np.array_equal(back, torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy())


def test_normal_draws_look_standard():
    z = synth.bf16_bits_to_f64(synth.normal_bf16(7, synth.STREAM_Q, (1 << 20,)))
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    # quantiles of N(0,1): 2.5% -> -1.95996, 50% -> 0, 97.5% -> 1.95996
    qs = np.quantile(z, [0.025, 0.5, 0.975])
    np.testing.assert_allclose(qs, [-1.95996, 0.0, 1.95996], atol=0.02)


def test_streams_and_seeds_differ():
    a = synth.normal_bf16(1, 0, (64,))
    assert not np.array_equal(a, synth.normal_bf16(1, 1, (64,)))
    assert not np.array_equal(a, synth.normal_bf16(2, 0, (64,)))
    assert np.array_equal(a, synth.normal_bf16(1, 0, (64,)))


def test_slices_match_whole_tensor():
    shape = (2, 33, 3, 16)
    full = synth.normal_bf16(5, synth.STREAM_K, shape)
    idx = np.ravel_multi_index(np.meshgrid(np.array([1]), np.arange(4, 21), np.array([2]), np.arange(16),
                                           indexing="ij"), shape).reshape(-1)
    part = synth.normal_bf16_at(5, synth.STREAM_K, idx).reshape(17, 16)
    assert np.array_equal(part, full[1, 4:21, 2, :])


def test_torch_drawing_matches_numpy():
    import torch

    shape = (3, 37, 2, 32)
    host = synth.normal_bf16(11, synth.STREAM_V, shape)
    dev = synth.normal_bf16_torch(11, synth.STREAM_V, shape, device="cpu", chunk=1000)
    assert np.array_equal(dev.view(torch.int16).numpy().view(np.uint16), host)


def test_kv_lengths_in_range():
    lens = synth.kv_lengths(1005, 4096, 1024, 131072)
    assert lens.min() >= 1024 and lens.max() <= 131072
    assert abs(lens.mean() - (1024 + 131072) / 2) < 3000
    assert np.array_equal(synth.DECODE.lengths(), synth.kv_lengths(1005, 8, 1024, 131072))


@pytest.mark.parametrize("w", synth.PREFILL_WORKLOADS, ids=lambda w: w.name)
def test_workload_flop_counts(w):
    f = 4.0 * w.B * w.Hq * w.Nq * w.Nkv * w.d
    assert w.flops == (f / 2 if w.causal else f)
