"""Launch-level behaviour on the GPU: concurrent launches on different streams, many launches in a
row (the prefill's unit-claiming counters are recycled), extreme shapes, and decode tails that
straddle the shared-memory tiles."""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import assert_parity, bf16_tensor_to_f64, device_bits, draw_prefill, to_torch_bf16

pytestmark = pytest.mark.gpu


def _prefill_ref(qb, kb, vb, scale, causal):
    O, L = oracle.attention(synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(kb), synth.bf16_bits_to_f64(vb),
                            scale, causal)
    return O, L.transpose(0, 2, 1)


def test_concurrent_prefill_launches_on_two_streams(lib):
    """Two launches in flight at once claim units from different counters and both come out right."""
    import torch

    cases = [(5100, 2, 4, 2, 700, 700, 128, True), (5101, 1, 8, 8, 1300, 1300, 64, False)]
    ins = [draw_prefill(*c[:7]) for c in cases]
    tens = [tuple(to_torch_bf16(x) for x in t) for t in ins]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    torch.cuda.synchronize()
    for rep in range(3):
        for (c, (q, k, v), st) in zip(cases, tens, streams):
            with torch.cuda.stream(st):
                outs.append(lib.attn_fwd(q, k, v, scale=1 / math.sqrt(c[6]), causal=c[7], stream=st))
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    for i, (o, lse) in enumerate(outs):
        c = cases[i % 2]
        O_ref, L_ref = _prefill_ref(*ins[i % 2], 1 / math.sqrt(c[6]), c[7])
        assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_ref, L_ref,
                      f"concurrent launch {i}")


def test_many_launches_recycle_the_claim_counters(lib):
    """More launches than there are claim counters: every result stays identical."""
    import torch

    qb, kb, vb = draw_prefill(5200, 1, 2, 2, 384, 384, 128)
    q, k, v = to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb)
    o0, l0 = lib.attn_fwd(q, k, v, causal=True)
    o0, l0 = o0.clone(), l0.clone()
    o = torch.empty_like(o0)
    l = torch.empty_like(l0)
    bad = torch.zeros((), dtype=torch.int64, device="cuda")
    for _ in range(600):
        lib.attn_fwd(q, k, v, causal=True, out=o, lse=l)
        bad += (o != o0).sum() + (l != l0).sum()
    torch.cuda.synchronize()
    assert int(bad) == 0
    assert lib.attn_get_last_error() == lib.ATTN_OK


def test_one_query_row_against_128k_keys(lib):
    import torch

    Nkv, d = 131072, 128
    qb, kb, vb = draw_prefill(5300, 1, 2, 1, 1, Nkv, d)
    o, lse = lib.attn_fwd(to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb), causal=True)
    torch.cuda.synchronize()
    O_ref, L_ref = _prefill_ref(qb, kb, vb, 1 / math.sqrt(d), True)
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_ref, L_ref,
                  "Nq=1 Nkv=131072")


def test_many_heads_tiny_sequences(lib):
    import torch

    qb, kb, vb = draw_prefill(5400, 16, 32, 4, 17, 33, 64)
    o, lse = lib.attn_fwd(to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb), causal=True)
    torch.cuda.synchronize()
    O_ref, L_ref = _prefill_ref(qb, kb, vb, 1 / 8, True)
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_ref, L_ref,
                  "B16 Hq32 Hkv4 Nq17 Nkv33")


def _decode_case(lib, seed, B, Hq, Hkv, d, cap, lens, chunk):
    import torch

    qb = synth.normal_bf16(seed, synth.STREAM_Q, (B, Hq, d))
    kb = synth.normal_bf16(seed, synth.STREAM_K, (B, cap, Hkv, d))
    vb = synth.normal_bf16(seed, synth.STREAM_V, (B, cap, Hkv, d))
    # cache rows past each sequence's length hold NaN: they must never reach the result
    kc, vc = to_torch_bf16(kb), to_torch_bf16(vb)
    for b, L in enumerate(lens):
        kc[b, L:] = float("nan")
        vc[b, L:] = float("nan")
    sc = 1 / math.sqrt(d)
    o, lse = lib.attn_decode_splitkv(to_torch_bf16(qb), kc, vc, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                     scale=sc, chunk=chunk)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    O_ref, L_ref = oracle.decode(synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(kb), synth.bf16_bits_to_f64(vb),
                                 np.array(lens), sc)
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), O_ref, L_ref,
                  f"decode d{d} lens {lens} chunk {chunk}")


@pytest.mark.parametrize("d", [32, 64, 128, 256])
def test_decode_tails_straddling_tiles_with_nan_padding(lib, d):
    # lengths 1..130 around the 16- and 64-token tile edges; the unused cache rows are NaN
    _decode_case(lib, 5500 + d, 8, 8, 2, d, 192, [1, 15, 16, 17, 63, 65, 127, 130], 64)


def test_decode_all_lengths_zero(lib):
    import torch

    B, Hq, Hkv, d, cap = 3, 8, 2, 128, 128
    q = torch.ones((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.full((B, cap, Hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    o, lse = lib.attn_decode_splitkv(q, kc, kc, lens, chunk=64)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_decode_full_cache_every_sequence(lib):
    _decode_case(lib, 5600, 2, 16, 2, 128, 4096, [4096, 4096], 0)


def test_tensor_map_cache_same_pointer_many_shapes_two_streams(lib):
    """The library caches TMA descriptors per (pointer, shape). Views of the same three buffers with
    more distinct shapes than the cache holds, launched alternately on two streams and then again
    in the same order (after their entries were evicted), must each give the oracle's result."""
    import torch

    n = 1 << 20
    bufs = [synth.normal_bf16_torch(5700 + i, 0, (n,), "cuda") for i in range(3)]
    shapes = []
    for i in range(72):  # > 64 cache entries
        d = (32, 64, 128, 256)[i % 4]
        Hkv = 1 + (i // 4) % 2
        Hq = Hkv * (1 + (i // 8) % 2)
        N = 40 + 13 * i
        shapes.append((Hq, Hkv, N, d, bool(i % 3 == 0)))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    torch.cuda.synchronize()
    for rep in range(2):
        for i, (Hq, Hkv, N, d, causal) in enumerate(shapes):
            q = bufs[0][:N * Hq * d].view(1, N, Hq, d)
            k = bufs[1][:N * Hkv * d].view(1, N, Hkv, d)
            v = bufs[2][:N * Hkv * d].view(1, N, Hkv, d)
            st = streams[(i + rep) % 2]
            with torch.cuda.stream(st):
                outs.append(lib.attn_fwd(q, k, v, causal=causal, stream=st))
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    for j, (o, lse) in enumerate(outs):
        Hq, Hkv, N, d, causal = shapes[j % len(shapes)]
        qb = device_bits(bufs[0][:N * Hq * d]).reshape(1, N, Hq, d)
        kb = device_bits(bufs[1][:N * Hkv * d]).reshape(1, N, Hkv, d)
        vb = device_bits(bufs[2][:N * Hkv * d]).reshape(1, N, Hkv, d)
        O_ref, L_ref = _prefill_ref(qb, kb, vb, 1 / math.sqrt(d), causal)
        assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_ref,
                      L_ref, f"shape {shapes[j % len(shapes)]} pass {j // len(shapes)}")
