"""Backward pass through the C ABI against the fp64 oracle's gradients: dQ, dK, dV of sum(O * dO)
with O from attn_fwd on the same inputs, on small shapes (ragged tiles, causal with Nq != Nkv, GQA)
and on the causal N2048 workload, whole tensors."""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import assert_grad_parity, bf16_tensor_to_f64, device_bits, draw_prefill, to_torch_bf16

pytestmark = pytest.mark.gpu

STREAM_DO = 5  # generator stream of dO


def _grads_ref_per_head(q, k, v, do, scale, causal):
    """oracle.attention_backward one (b, kv head) at a time (thread pool), summed like the oracle."""
    from concurrent.futures import ThreadPoolExecutor
    import os

    from threadpoolctl import threadpool_limits

    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)

    def work(bg):
        b, g = divmod(bg, Hkv)
        hs = slice(g * G, (g + 1) * G)
        a, bk, c = oracle.attention_backward(q[b:b + 1, :, hs], k[b:b + 1, :, g:g + 1], v[b:b + 1, :, g:g + 1],
                                             do[b:b + 1, :, hs], scale, causal)
        dq[b, :, hs] = a[0]
        dk[b, :, g] = bk[0, :, 0]
        dv[b, :, g] = c[0, :, 0]

    with threadpool_limits(limits=1, user_api="blas"), ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        list(ex.map(work, range(B * Hkv)))
    return dq, dk, dv


def _run(lib, seed, B, Hq, Hkv, Nq, Nkv, causal, scale=None):
    import torch

    d = 128
    qb, kb, vb = draw_prefill(seed, B, Hq, Hkv, Nq, Nkv, d)
    dob = synth.normal_bf16(seed, STREAM_DO, (B, Nq, Hq, d))
    q, k, v, do = to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb), to_torch_bf16(dob)
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    o, lse = lib.attn_fwd(q, k, v, scale=sc, causal=causal)
    dq, dk, dv = lib.attn_bwd(q, k, v, o, lse, do, scale=sc, causal=causal)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    f = synth.bf16_bits_to_f64
    rq, rk, rv = _grads_ref_per_head(f(qb), f(kb), f(vb), f(dob), sc, causal)
    what = f"bwd B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nkv{Nkv} causal={causal}"
    assert_grad_parity(bf16_tensor_to_f64(dq), rq, what + " dQ")
    assert_grad_parity(bf16_tensor_to_f64(dk), rk, what + " dK")
    assert_grad_parity(bf16_tensor_to_f64(dv), rv, what + " dV")


@pytest.mark.parametrize("Nq,Nkv,causal", [(256, 256, False), (256, 256, True), (300, 300, False), (300, 300, True),
                                           (130, 513, True), (600, 200, True), (1, 300, False)])
def test_backward_against_the_oracle(lib, Nq, Nkv, causal):
    _run(lib, 8000 + Nq + Nkv, 2, 2, 2, Nq, Nkv, causal)


def test_backward_gqa_and_large_scale(lib):
    _run(lib, 8100, 1, 8, 2, 384, 384, True)
    _run(lib, 8101, 1, 4, 1, 256, 320, False, scale=0.5)


def test_backward_more_units_than_sms(lib):
    # 6 key blocks x 4 batches x 8 kv heads = 192 key-block CTAs, more than one wave on 148 SMs, with
    # causal units of 1 to 6 steps, key blocks that end ragged (700 keys), a non-causal GQA case, and
    # 100 queries against 700 keys (causal: one step per key block)
    _run(lib, 8200, 4, 8, 8, 700, 700, True)
    _run(lib, 8201, 4, 16, 8, 700, 700, False)
    _run(lib, 8202, 4, 8, 8, 100, 700, True)


def test_backward_causal_2k_workload_whole_tensors(lib):
    import torch

    w = synth.CAUSAL_2K
    dev = "cuda"
    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
    k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
    v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
    do = synth.normal_bf16_torch(w.seed, STREAM_DO, (w.B, w.Nq, w.Hq, w.d), dev)
    o, lse = lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal)
    dq, dk, dv = lib.attn_bwd(q, k, v, o, lse, do, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    f = synth.bf16_bits_to_f64
    rq, rk, rv = _grads_ref_per_head(f(device_bits(q)), f(device_bits(k)), f(device_bits(v)), f(device_bits(do)),
                                     w.scale, w.causal)
    assert_grad_parity(bf16_tensor_to_f64(dq), rq, "bwd " + w.name + " dQ")
    assert_grad_parity(bf16_tensor_to_f64(dk), rk, "bwd " + w.name + " dK")
    assert_grad_parity(bf16_tensor_to_f64(dv), rv, "bwd " + w.name + " dV")
