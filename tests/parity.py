"""Helpers shared by the GPU parity tests: seeded inputs on both sides, oracle rows, tolerances."""
from __future__ import annotations

import numpy as np

import oracle
import synth

# Tolerances of the exact-attention parity gate (bf16 in, fp32 accumulate, bf16 O, fp32 LSE).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def to_torch_bf16(bits: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch

    return synth.bf16_bits_to_f64(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def assert_parity(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray, what: str):
    """O within max-abs / mean-abs, LSE within abs; -inf LSE (and O = 0) exactly where the oracle has it.

    O is [..., d]; LSE is laid out like O without its last axis.
    """
    assert o_gpu.shape == o_ref.shape and lse_gpu.shape == lse_ref.shape == o_ref.shape[:-1], what
    o_err = np.abs(o_gpu - o_ref)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    assert o_err.max() <= O_MAX_ABS, f"{what}: O max-abs {o_err.max():.3e}"
    assert o_err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {o_err.mean():.3e}"
    ref_inf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ref_inf), f"{what}: -inf LSE pattern differs"
    assert np.all(o_gpu[ref_inf] == 0.0), f"{what}: rows without keys must be 0"
    if (~ref_inf).any():
        l_err = np.abs(lse_gpu[~ref_inf] - lse_ref[~ref_inf])
        assert l_err.max() <= LSE_ABS, f"{what}: LSE max-abs {l_err.max():.3e}"


def draw_prefill(seed, B, Hq, Hkv, Nq, Nkv, d):
    return (synth.normal_bf16(seed, synth.STREAM_Q, (B, Nq, Hq, d)),
            synth.normal_bf16(seed, synth.STREAM_K, (B, Nkv, Hkv, d)),
            synth.normal_bf16(seed, synth.STREAM_V, (B, Nkv, Hkv, d)))


def kv_slice_bits(seed, stream, shape, b, g, n):
    """bf16 bits of tensor[b, :n, g, :] of a [B, N, H, d] stream, drawn on its own."""
    _, N, H, d = shape
    t = np.arange(n, dtype=np.int64)[:, None]
    e = np.arange(d, dtype=np.int64)[None, :]
    flat = ((b * N + t) * H + g) * d + e
    return synth.normal_bf16_at(seed, stream, flat.reshape(-1)).reshape(n, d)


def q_row_bits(seed, shape, b, i, h):
    _, N, H, d = shape
    flat = ((b * N + i) * H + h) * d + np.arange(d, dtype=np.int64)
    return synth.normal_bf16_at(seed, synth.STREAM_Q, flat)


def sample_rows(rng, B, Nq, Hq, n, causal):
    """A fixed set of (b, i, h) triples: corners, tile edges, and random rows."""
    picks = {(0, 0, 0), (B - 1, Nq - 1, Hq - 1), (0, Nq - 1, 0), (B - 1, 0, Hq - 1)}
    for i in (127, 128, 255, 256, 383, 384, Nq // 2):
        if i < Nq:
            picks.add((int(rng.integers(B)), i, int(rng.integers(Hq))))
    while len(picks) < n:
        picks.add((int(rng.integers(B)), int(rng.integers(Nq)), int(rng.integers(Hq))))
    return sorted(picks)


def oracle_rows_prefill(w, picks):
    """Oracle O rows and LSE for the sampled (b, i, h) of a prefill workload drawn from its seed."""
    qshape = (w.B, w.Nq, w.Hq, w.d)
    kshape = (w.B, w.Nkv, w.Hkv, w.d)
    cache = {}
    outs = []
    for (b, i, h) in picks:
        g = oracle.kv_head(h, w.Hq, w.Hkv)
        if (b, g) not in cache:
            cache[(b, g)] = (synth.bf16_bits_to_f64(kv_slice_bits(w.seed, synth.STREAM_K, kshape, b, g, w.Nkv)),
                             synth.bf16_bits_to_f64(kv_slice_bits(w.seed, synth.STREAM_V, kshape, b, g, w.Nkv)))
        K, V = cache[(b, g)]
        keys = oracle.visible_keys(i, w.Nq, w.Nkv, w.causal)
        q = synth.bf16_bits_to_f64(q_row_bits(w.seed, qshape, b, i, h))
        outs.append(oracle.attention_row(q, K[keys], V[keys], w.scale))
    return np.array([o for o, _ in outs]), np.array([l for _, l in outs])
