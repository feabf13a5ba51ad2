"""Helpers shared by the GPU parity tests: seeded inputs on both sides, oracle rows, tolerances."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

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


def device_bits(t) -> np.ndarray:
    """The exact bf16 bit patterns of a device tensor, copied to the host (uint16, same shape)."""
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_whole_prefill(qbits, kbits, vbits, scale, causal, workers=None):
    """The oracle's O [B, Nq, Hq, d] and LSE [B, Nq, Hq] over the whole output, one (b, h) head per
    task: each task widens its head's bf16 bits and calls oracle.attention on that head alone. Tasks
    run on a thread pool (the BLAS products and numpy's elementwise passes release the GIL) with one
    BLAS thread each."""
    from threadpoolctl import threadpool_limits

    B, Nq, Hq, d = qbits.shape
    Hkv = kbits.shape[2]
    O = np.empty((B, Nq, Hq, d))
    L = np.empty((B, Nq, Hq))
    f = synth.bf16_bits_to_f64

    def head(bh):
        b, h = divmod(bh, Hq)
        g = oracle.kv_head(h, Hq, Hkv)
        o, lse = oracle.attention(f(qbits[b:b + 1, :, h:h + 1]), f(kbits[b:b + 1, :, g:g + 1]),
                                  f(vbits[b:b + 1, :, g:g + 1]), scale, causal)
        O[b, :, h] = o[0, :, 0]
        L[b, :, h] = lse[0, 0]

    n = workers or max(1, min(8, os.cpu_count() or 1))
    with threadpool_limits(limits=1, user_api="blas"), ThreadPoolExecutor(n) as ex:
        list(ex.map(head, range(B * Hq)))
    return O, L


def oracle_whole_prefill_values(q, k, v, scale, causal, workers=None):
    """oracle_whole_prefill for inputs given as values (any float array exactly widened to fp64)."""
    from threadpoolctl import threadpool_limits

    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    O = np.empty((B, Nq, Hq, d))
    L = np.empty((B, Nq, Hq))

    def head(bh):
        b, h = divmod(bh, Hq)
        g = oracle.kv_head(h, Hq, Hkv)
        o, lse = oracle.attention(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, g:g + 1], v[b:b + 1, :, g:g + 1], scale,
                                  causal)
        O[b, :, h] = o[0, :, 0]
        L[b, :, h] = lse[0, 0]

    n = workers or max(1, min(8, os.cpu_count() or 1))
    with threadpool_limits(limits=1, user_api="blas"), ThreadPoolExecutor(n) as ex:
        list(ex.map(head, range(B * Hq)))
    return O, L


# 8-bit path: P is rounded to e4m3 before the PV product. Rounding P_j (relative to the kernel's
# running max, so P_j >= its value relative to the true max) to nearest e4m3 changes it by at most
# 2^-4 P_j, or 2^-10 below 2^-6 (subnormal spacing 2^-9). Modelled as independent zero-mean errors,
# O[i, e] then deviates from the result on unrounded P by a sum with standard deviation at most
#   sigma[i, e] = sqrt(sum_j w_j^2 V[j, e]^2 / 3) / sum_j P_j,   w_j = max(2^-4 P_j, 2^-10 [P_j < 2^-6])
# (P relative to the true row max). Gates: the mean over elements of |err| <= 3 * mean(sigma) and
# every |err| <= 8 sigma, both plus the bf16 rounding of O (2^-8 |O|) and 1e-6.
FP8_MEAN_SIGMAS = 3.0
FP8_MAX_SIGMAS = 8.0


def fp8_sigma(q, k, v, scale, causal):
    """sigma[b, i, h, e] above, from the decoded inputs (fp64) per (b, h) head."""
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    sig = np.zeros((B, Nq, Hq, d))
    for b in range(B):
        for h in range(Hq):
            g = oracle.kv_head(h, Hq, Hkv)
            P = oracle.probabilities(q[b, :, h], k[b, :, g], scale, causal)     # rows sum to 1 (or 0)
            Pm = P / np.where(P.max(axis=1, keepdims=True) > 0, P.max(axis=1, keepdims=True), 1.0)
            w = np.maximum(Pm * 2.0 ** -4, np.where((Pm > 0) & (Pm < 2.0 ** -6), 2.0 ** -10, 0.0))
            z = Pm.sum(axis=1, keepdims=True)
            sig[b, :, h] = np.sqrt((w ** 2) @ (v[b, :, g] ** 2) / 3.0) / np.where(z > 0, z, 1.0)
    return sig


def assert_parity_fp8(o_gpu, lse_gpu, o_ref, lse_ref, sigma, what):
    """The 8-bit gate: O within the e4m3-rounding model above; LSE within LSE_ABS; empty rows exact."""
    assert o_gpu.shape == o_ref.shape == sigma.shape and lse_gpu.shape == lse_ref.shape, what
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    err = np.abs(o_gpu - o_ref)
    slack = 2.0 ** -8 * np.abs(o_ref) + 1e-6
    assert err.mean() <= FP8_MEAN_SIGMAS * sigma.mean() + slack.mean(), \
        f"{what}: O mean-abs {err.mean():.3e} > {FP8_MEAN_SIGMAS * sigma.mean() + slack.mean():.3e}"
    worst = (err - slack - FP8_MAX_SIGMAS * sigma).max()
    assert worst <= 0, f"{what}: an element exceeds 8 sigma by {worst:.3e} (max |err| {err.max():.3e})"
    ref_inf = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ref_inf), f"{what}: -inf LSE pattern differs"
    assert np.all(o_gpu[ref_inf] == 0.0), f"{what}: rows without keys must be 0"
    if (~ref_inf).any():
        l_err = np.abs(lse_gpu[~ref_inf] - lse_ref[~ref_inf])
        assert l_err.max() <= LSE_ABS, f"{what}: LSE max-abs {l_err.max():.3e}"


# Backward pass: each gradient element is a sum of products in which one factor (P for dV; dS for dQ
# and dK) was rounded to bf16 (relative 2^-9), D comes from the bf16 O, and the result is rounded to
# bf16 (2^-9). The error of a tensor is therefore a small multiple of 2^-9 of its own magnitude. Gate:
# RMS error <= 2^-7 x RMS of the reference, and every element within 2^-5 x max |reference|.
BWD_RMS_REL = 2.0 ** -7
BWD_MAX_REL = 2.0 ** -5


def assert_grad_parity(g_gpu, g_ref, what):
    assert g_gpu.shape == g_ref.shape, what
    assert np.all(np.isfinite(g_gpu)), f"{what}: non-finite"
    err = g_gpu - g_ref
    rms_ref = np.sqrt(np.mean(g_ref ** 2))
    rms_err = np.sqrt(np.mean(err ** 2))
    max_ref = np.abs(g_ref).max()
    assert rms_err <= BWD_RMS_REL * rms_ref + 1e-7, f"{what}: RMS error {rms_err:.3e} vs RMS {rms_ref:.3e}"
    assert np.abs(err).max() <= BWD_MAX_REL * max_ref + 1e-6, \
        f"{what}: max error {np.abs(err).max():.3e} vs max {max_ref:.3e} (RMS error {rms_err:.3e} / {rms_ref:.3e})"
