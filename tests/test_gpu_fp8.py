"""The 8-bit prefill path through the C ABI: incoherent processing and e4m3 quantization compared bit
for bit with the oracle's codes, then attention on the 8-bit operands against the fp64 oracle on the
decoded values, within the e4m3-rounding model of P (tests/parity.py), and the accuracy gain of the
rotation on inputs with outlier channels."""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import (assert_parity_fp8, bf16_tensor_to_f64, device_bits, draw_prefill, fp8_sigma,
                    oracle_whole_prefill, oracle_whole_prefill_values, to_torch_bf16)

pytestmark = pytest.mark.gpu


def _signs(seed, d=128):
    u = np.random.default_rng(seed).random(d)
    return np.where(u < 0.5, -1.0, 1.0).astype(np.float32)


def _quantize_all(lib, q, k, v, signs_t):
    q8, aq = lib.attn_fp8_quantize(q, signs_t)
    k8, ak = lib.attn_fp8_quantize(k, signs_t)
    vt8, av = lib.attn_fp8_quantize(v, None, transpose=True)
    return q8, aq, k8, ak, vt8, av


def _check_codes(q8, aq, k8, ak, vt8, av, qf, kf, vf, signs):
    """GPU codes and maxima equal the oracle's, bit for bit; returns the oracle's decoded values."""
    out = []
    for c_gpu, a_gpu, x, s, tr in ((q8, aq, qf, signs, False), (k8, ak, kf, signs, False), (vt8, av, vf, None, True)):
        codes, amax = oracle.fp8_quantize(x, s)
        cg = c_gpu.cpu().numpy()
        if tr:
            cg = cg.transpose(0, 3, 1, 2)  # [B, H, d, N] -> [B, N, H, d]
        assert np.array_equal(a_gpu.cpu().numpy().view(np.uint32), amax.view(np.uint32)), "amax differs"
        bad = np.count_nonzero(cg != codes)
        assert bad == 0, f"{bad} codes differ"
        out.append(oracle.fp8_dequantize(codes, amax))
    return out


def _run(lib, seed, B, Hq, Hkv, Nq, Nkv, causal, scale=None):
    import torch

    d = 128
    qb, kb, vb = draw_prefill(seed, B, Hq, Hkv, Nq, Nkv, d)
    q, k, v = to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb)
    s = _signs(seed)
    q8, aq, k8, ak, vt8, av = _quantize_all(lib, q, k, v, torch.from_numpy(s).cuda())
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    o, lse = lib.attn_fwd_fp8(q8, k8, vt8, aq, ak, av, scale=sc, causal=causal)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    f = synth.bf16_bits_to_f64
    qd, kd, vd = _check_codes(q8, aq, k8, ak, vt8, av, f(qb).astype(np.float32), f(kb).astype(np.float32),
                              f(vb).astype(np.float32), s)
    O_ref, L_ref = oracle.attention(qd, kd, vd, sc, causal)
    assert_parity_fp8(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_ref,
                      L_ref.transpose(0, 2, 1), fp8_sigma(qd, kd, vd, sc, causal),
                      f"fp8 B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nkv{Nkv} causal={causal}")


@pytest.mark.parametrize("Nq,Nkv,causal", [(300, 320, False), (300, 320, True), (256, 256, True), (1, 512, True),
                                           (130, 16, False), (600, 208, True)])
def test_fp8_attention_against_the_oracle_on_decoded_inputs(lib, Nq, Nkv, causal):
    _run(lib, 7000 + Nq + Nkv, 2, 4, 2, Nq, Nkv, causal)


def test_fp8_gqa_group_of_eight_and_large_scale(lib):
    _run(lib, 7100, 1, 8, 1, 384, 384, True)
    _run(lib, 7101, 1, 2, 2, 512, 512, False, scale=0.5)


def test_fp8_quantize_every_layout_and_ragged_rows(lib):
    import torch

    rng_seed = 7200
    for (B, N, H, signs, tr) in ((2, 300, 3, True, False), (1, 37, 2, False, False), (2, 336, 2, False, True),
                                 (1, 48, 1, True, True)):
        xb = synth.normal_bf16(rng_seed, 0, (B, N, H, 128))
        s = _signs(rng_seed) if signs else None
        x = to_torch_bf16(xb)
        codes, amax = lib.attn_fp8_quantize(x, None if s is None else torch.from_numpy(s).cuda(), transpose=tr)
        torch.cuda.synchronize()
        want_c, want_a = oracle.fp8_quantize(synth.bf16_bits_to_f64(xb).astype(np.float32), s)
        got = codes.cpu().numpy()
        if tr:
            got = got.transpose(0, 3, 1, 2)
        assert np.array_equal(got, want_c)
        assert np.array_equal(amax.cpu().numpy().view(np.uint32), want_a.view(np.uint32))
        rng_seed += 1


def test_fp8_long_workload_whole_output(lib):
    """The long non-causal B2 H16 N8192 d128 workload on the 8-bit path, whole output."""
    import torch

    w = synth.LONG_8K
    dev = "cuda"
    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
    k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
    v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
    s = _signs(w.seed)
    q8, aq, k8, ak, vt8, av = _quantize_all(lib, q, k, v, torch.from_numpy(s).cuda())
    o, lse = lib.attn_fwd_fp8(q8, k8, vt8, aq, ak, av, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    f = synth.bf16_bits_to_f64
    qd, kd, vd = _check_codes(q8, aq, k8, ak, vt8, av, f(device_bits(q)).astype(np.float32),
                              f(device_bits(k)).astype(np.float32), f(device_bits(v)).astype(np.float32), s)
    og, lg = bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1)
    del q, k, v, q8, k8, vt8, o, lse
    torch.cuda.empty_cache()
    O_ref, L_ref = oracle_whole_prefill_values(qd, kd, vd, w.scale, w.causal)
    # sigma on two heads (its P is the costly part), applied as the bound for every head
    sig = fp8_sigma(qd[:, :, :2], kd[:, :, :2], vd[:, :, :2], w.scale, w.causal)
    sig_all = np.broadcast_to(sig.max(axis=2, keepdims=True), og.shape)
    assert_parity_fp8(og, lg, O_ref, L_ref, sig_all, "fp8 " + w.name)


def test_rotation_lowers_the_error_of_outlier_channels(lib):
    """Q and K with two channels 40x larger: against the exact bf16 result, the 8-bit path is much
    closer with the rotation than without."""
    import torch

    B, N, H, d = 1, 512, 2, 128
    qb, kb, vb = draw_prefill(7300, B, H, H, N, N, d)
    q, k, v = (synth.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    for ch in (3, 77):
        q[..., ch] *= 40.0
        k[..., ch] *= 40.0
    qb, kb = synth.f64_to_bf16_bits(q), synth.f64_to_bf16_bits(k)
    sc = 1.0 / math.sqrt(d) / 40.0
    O, _ = oracle_whole_prefill(qb, kb, vb, sc, False)
    errs = {}
    for name, s in (("rotated", _signs(7300)), ("plain", None)):
        st = None if s is None else torch.from_numpy(s).cuda()
        q8, aq = lib.attn_fp8_quantize(to_torch_bf16(qb), st)
        k8, ak = lib.attn_fp8_quantize(to_torch_bf16(kb), st)
        vt8, av = lib.attn_fp8_quantize(to_torch_bf16(vb), None, transpose=True)
        o, _ = lib.attn_fwd_fp8(q8, k8, vt8, aq, ak, av, scale=sc)
        torch.cuda.synchronize()
        errs[name] = np.abs(bf16_tensor_to_f64(o) - O).mean()
    assert errs["rotated"] < 0.5 * errs["plain"], errs
