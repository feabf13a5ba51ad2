"""Prefill parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the same seeded
bf16 inputs, element by element over the whole output: small shapes drawn on the host, and every
full-size workload drawn on the device with the oracle fed the exact bits the kernel read."""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import (assert_parity, bf16_tensor_to_f64, device_bits, draw_prefill, oracle_whole_prefill,
                    to_torch_bf16)

pytestmark = pytest.mark.gpu


def _run_small(lib, seed, B, Hq, Hkv, Nq, Nkv, d, causal, scale=None):
    import torch

    qb, kb, vb = draw_prefill(seed, B, Hq, Hkv, Nq, Nkv, d)
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    o, lse = lib.attn_fwd(to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb), scale=sc, causal=causal)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention(synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(kb),
                                    synth.bf16_bits_to_f64(vb), sc, causal)
    what = f"B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nkv{Nkv} d{d} causal={causal}"
    lse_g = lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1)
    assert_parity(bf16_tensor_to_f64(o), lse_g, O_ref, L_ref.transpose(0, 2, 1), what)
    assert lib.attn_get_last_error() == lib.ATTN_OK


def test_tiny_workload(lib):
    w = synth.TINY
    _run_small(lib, w.seed, w.B, w.Hq, w.Hkv, w.Nq, w.Nkv, w.d, w.causal)


@pytest.mark.parametrize("d", [32, 64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_every_head_dim_ragged_tiles(lib, d, causal):
    # 300 rows/keys: several 128-row tiles and a ragged tail; GQA group of 2
    _run_small(lib, 2000 + d, 2, 4, 2, 300, 300, d, causal)


@pytest.mark.parametrize("Nq,Nkv,causal", [
    (1, 777, False), (1, 777, True), (130, 513, True), (600, 200, True), (5, 5, False), (5, 5, True),
    (256, 1, False), (257, 129, False), (64, 1000, True),
])
def test_edge_shapes(lib, Nq, Nkv, causal):
    _run_small(lib, 3000 + Nq + Nkv, 1, 2, 1, Nq, Nkv, 128, causal)


@pytest.mark.parametrize("d", [64, 256])
def test_edge_shapes_other_head_dims(lib, d):
    _run_small(lib, 3100 + d, 1, 2, 2, 1, 300, d, True)
    _run_small(lib, 3200 + d, 1, 2, 2, 200, 70, d, True)


def test_many_units_whose_first_tile_has_no_key(lib):
    # causal, Nq - Nkv = 400: per head, the 256-row block 0 sees no key, block 1's first 128 rows see
    # none (its second tile does) and block 2 sees all; 4 x 32 heads give 384 units on at most 148
    # CTAs, the light ones last, so CTAs take several keyless-first-tile units in a row
    _run_small(lib, 4600, 4, 32, 8, 600, 200, 128, True)


def test_gqa_group_of_eight_causal(lib):
    _run_small(lib, 4000, 1, 8, 1, 384, 384, 128, True)


def test_large_score_spread(lib):
    # scale far above 1/sqrt(d) makes the running max jump often, exercising the O rescale path
    _run_small(lib, 4100, 1, 2, 2, 512, 512, 128, False, scale=1.5)
    _run_small(lib, 4101, 1, 2, 2, 512, 512, 128, True, scale=1.5)
    _run_small(lib, 4102, 1, 2, 2, 384, 384, 256, True, scale=1.5)


def test_head_dim_256_cta_pairs(lib):
    # d = 256 runs on CTA pairs: 256 query rows per unit, 128 in each CTA, 128-key tiles split between
    # the two. 100 rows leave the second CTA without a valid row and 130 with two; 300 keys end in a
    # ragged tile whose two halves are partly and wholly past the end; 2 x 8 x 6 = 96 causal units on
    # at most 74 pairs give pairs several units, so the hand-off counters carry across units (twice
    # 1/sqrt(d) makes the running max move often; much larger scales make P nearly one-hot and O a
    # single V row, whose bf16 rounding alone can exceed the gate at every head dim).
    _run_small(lib, 4500, 1, 2, 1, 100, 300, 256, False)
    _run_small(lib, 4501, 1, 2, 2, 130, 130, 256, True)
    _run_small(lib, 4502, 1, 2, 2, 1, 193, 256, False)
    _run_small(lib, 4503, 2, 8, 4, 1300, 1300, 256, True, scale=0.125)
    # one key (the second CTA's half of the only K tile lies wholly past the end), one query row,
    # and a causal square smaller than a tile
    _run_small(lib, 4504, 1, 2, 2, 300, 1, 256, False)
    _run_small(lib, 4505, 1, 2, 1, 1, 1, 256, True)
    _run_small(lib, 4506, 2, 2, 2, 5, 5, 256, True)


@pytest.mark.parametrize("d", [32, 64])
def test_small_head_dims_rescale_and_units_per_cta(lib, d):
    # d <= 64 keeps P in buffers of its own; a large scale makes the running max jump (O rescales that
    # must wait for the previous PV), and 384 causal units on the persistent grid give every CTA
    # several units, so the S and P hand-off counters carry across units
    _run_small(lib, 4300 + d, 1, 2, 2, 512, 512, d, False, scale=1.5)
    _run_small(lib, 4310 + d, 4, 16, 4, 1300, 1300, d, True, scale=0.6)


DOMINANT_KEYS = (0, 63, 64, 100, 127, 128, 191, 255)  # first, middle and last of 64- and 128-key tiles


@pytest.mark.parametrize("d", [64, 128, 256])
def test_dominant_score_anywhere_in_a_tile(lib, d):
    # Row i's score for key DOMINANT_KEYS[i % 8] is ~500 log2 units above every other score of the
    # row, so every position of the key tiles holds some row's maximum. A row max that misses one
    # position would leave 2^(score - max) to overflow; O must come out as that key's V row.
    import torch

    N = 256
    qb, kb, vb = draw_prefill(4400 + d, 1, 1, 1, N, N, d)
    q = synth.bf16_bits_to_f64(qb) * 0.01
    k = synth.bf16_bits_to_f64(kb) * 0.01
    big = 64.0
    for m, key in enumerate(DOMINANT_KEYS):
        k[0, key, 0, :8] = 0.0
        k[0, key, 0, m] = big
    for i in range(N):
        q[0, i, 0, i % 8] = big
    qb2, kb2 = synth.f64_to_bf16_bits(q), synth.f64_to_bf16_bits(k)
    sc = 1.0 / math.sqrt(d)
    o, lse = lib.attn_fwd(to_torch_bf16(qb2), to_torch_bf16(kb2), to_torch_bf16(vb), scale=sc, causal=False)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention(synth.bf16_bits_to_f64(qb2), synth.bf16_bits_to_f64(kb2),
                                    synth.bf16_bits_to_f64(vb), sc, False)
    og = bf16_tensor_to_f64(o)
    lg = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg))
    assert_parity(og, lg.transpose(0, 2, 1), O_ref, L_ref.transpose(0, 2, 1), f"dominant keys d{d}")
    assert lib.attn_get_last_error() == lib.ATTN_OK


def test_repeat_calls_are_identical(lib):
    import torch

    qb, kb, vb = draw_prefill(4200, 1, 4, 4, 512, 512, 128)
    q, k, v = to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb)
    o1, l1 = lib.attn_fwd(q, k, v, causal=True)
    o1, l1 = o1.clone(), l1.clone()
    for _ in range(5):
        o2, l2 = lib.attn_fwd(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


FULL = [synth.CAUSAL_2K, synth.LONG_8K, synth.LONG_8K_CAUSAL, synth.LONG_8K_GQA, synth.LONG_8K_GQA_CAUSAL,
        *synth.SWEEP]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_workload_whole_output(lib, w):
    """Every full-size workload, compared element by element over the whole O and LSE. The inputs
    are drawn on the device (as the benchmark does), and the oracle is fed the exact bits the kernel
    read, copied back to the host, so the comparison does not rest on the two draws agreeing."""
    import torch

    dev = "cuda"
    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
    k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
    v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
    o, lse = lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    qb, kb, vb = device_bits(q), device_bits(k), device_bits(v)
    og, lg = bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1)
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    O_ref, L_ref = oracle_whole_prefill(qb, kb, vb, w.scale, w.causal)
    assert_parity(og, lg, O_ref, L_ref, w.name)
