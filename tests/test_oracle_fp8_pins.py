"""Pins for the oracle's 8-bit path: e4m3 decoding and rounding, the Hadamard rotation, the per-head
quantization and the effect the rotation exists for. Each check fixes the oracle against the format's
definition, an independent library routine (torch's float8_e4m3fn on the CPU), a closed form or an
invariant, never against a retyping of the same code."""
import math

import numpy as np
import pytest

import oracle


def _decode_by_format(code: int) -> float:
    """e4m3 by its bit fields, in plain Python: s eeee mmm, bias 7, no infinities, S.1111.111 = NaN."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def test_e4m3_decode_every_code():
    import torch

    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    want = np.array([_decode_by_format(int(c)) for c in codes])
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for ref in (want, lib):
        same = (got == ref) | (np.isnan(got) & np.isnan(ref))
        assert same.all(), np.nonzero(~same)
    assert oracle.e4m3_decode(np.array([0x7E], dtype=np.uint8))[0] == 448.0  # largest finite
    assert oracle.e4m3_decode(np.array([0x01], dtype=np.uint8))[0] == 2.0 ** -9  # smallest subnormal


def test_e4m3_round_matches_torch_including_every_tie():
    import torch

    finite = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))  # +0 .. 448
    mids = (finite[:-1] + finite[1:]) / 2                              # exact ties (representable in fp32)
    rng = np.random.default_rng(40)
    xs = np.concatenate([finite, mids, np.nextafter(mids, 0), np.nextafter(mids, 1000),
                         rng.uniform(0, 448, 200000), rng.uniform(0, 2.0 ** -6, 20000),
                         np.exp2(rng.uniform(-12, 8.8, 20000))])
    xs = np.concatenate([xs, -xs]).astype(np.float32)
    xs = xs[np.abs(xs) <= 448]
    got = oracle.e4m3_round(xs)
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want), np.nonzero(got != want)[0][:10]
    # ties go to the even code: 1 + 1/16 lies between codes 0x38 (1.0) and 0x39 (1.125)
    assert oracle.e4m3_round(np.float32([1.0625]))[0] == 0x38
    assert oracle.e4m3_round(np.float32([1.1875]))[0] == 0x3A  # between 1.125 (0x39) and 1.25 (0x3A)


def test_e4m3_round_saturates_and_keeps_the_sign_of_zero():
    big = np.float32([448.0, 460.0, 464.0, 1000.0, 3.0e38, -449.0, -1.0e30])
    assert oracle.e4m3_round(big).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    tiny = np.float32([0.0, -0.0, 2.0 ** -11, -(2.0 ** -11), 2.0 ** -10, 3 * 2.0 ** -11])
    # 2^-10 is the tie between 0 and the smallest subnormal 2^-9: even code 0; 3*2^-11 rounds up
    assert oracle.e4m3_round(tiny).tolist() == [0x00, 0x80, 0x00, 0x80, 0x00, 0x01]


def _hadamard(d):
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


@pytest.mark.parametrize("d", [2, 8, 128])
def test_rotation_is_the_scaled_hadamard_product(d):
    rng = np.random.default_rng(41 + d)
    x = rng.standard_normal((5, 3, d)).astype(np.float32)
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
    got = oracle.hadamard_rotate_f32(x, s).astype(np.float64)
    # row vector convention: y = (x * s) H / sqrt(d), H symmetric
    want = (x.astype(np.float64) * s) @ _hadamard(d) / math.sqrt(d)
    assert np.max(np.abs(got - want)) <= 2e-6 * max(1.0, np.abs(want).max())


def test_rotation_is_orthogonal_and_keeps_inner_products():
    d = 128
    rng = np.random.default_rng(42)
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
    basis = oracle.hadamard_rotate_f32(np.eye(d, dtype=np.float32), s).astype(np.float64)
    np.testing.assert_allclose(basis @ basis.T, np.eye(d), atol=1e-6)
    q = rng.standard_normal((64, d)).astype(np.float32)
    k = rng.standard_normal((64, d)).astype(np.float32)
    qr, kr = oracle.hadamard_rotate_f32(q, s), oracle.hadamard_rotate_f32(k, s)
    np.testing.assert_allclose(qr.astype(np.float64) @ kr.T.astype(np.float64),
                               q.astype(np.float64) @ k.T.astype(np.float64), atol=2e-4)
    # d = 2, signs (+1, -1), x = (3, 5): (3, -5) -> butterfly (-2, 8) -> times fp32(1/sqrt 2)
    y = oracle.hadamard_rotate_f32(np.float32([[3.0, 5.0]]), np.float32([1.0, -1.0]))
    r = np.float32(1 / math.sqrt(2))
    assert y.tolist() == [[float(np.float32(-2.0) * r), float(np.float32(8.0) * r)]]


def test_quantize_maps_each_head_max_to_448_and_rounds_the_rest():
    rng = np.random.default_rng(43)
    B, N, H, d = 2, 37, 3, 128
    x = rng.standard_normal((B, N, H, d)).astype(np.float32)
    x[1, 5, 2, 7] = -20.0  # a head whose max is negative
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
    for signs in (s, None):
        codes, amax = oracle.fp8_quantize(x, signs)
        y = oracle.hadamard_rotate_f32(x, signs) if signs is not None else x
        np.testing.assert_array_equal(amax, np.abs(y).max(axis=(1, 3)))
        for b in range(B):
            for h in range(H):
                yh = y[b, :, h, :]
                arg = np.unravel_index(np.abs(yh).argmax(), yh.shape)
                assert codes[b, arg[0], h, arg[1]] in (0x7E, 0xFE)
        # every code is within half an e4m3 step of y * 448 / amax (relative 2^-4, or 2^-10 below 2^-6)
        t = y.astype(np.float64) * (448.0 / amax.astype(np.float64))[:, None, :, None]
        v = oracle.e4m3_decode(codes)
        assert np.all(np.abs(v - t) <= np.maximum(np.abs(t) * 2.0 ** -4, 2.0 ** -10) + 1e-6)
        deq = oracle.fp8_dequantize(codes, amax)
        assert np.all(np.abs(deq - y) <= np.maximum(np.abs(y) * 2.0 ** -4, amax.max() / 448 * 2.0 ** -10) + 1e-6)
    zero_codes, zero_amax = oracle.fp8_quantize(np.zeros((1, 4, 1, d), np.float32))
    assert np.all(zero_codes == 0) and np.all(zero_amax == 0)


def test_rotation_lowers_the_quantization_error_of_outlier_channels():
    """The point of incoherent processing: with a few large channels in Q and K, attention on the
    8-bit values is much closer to the exact result when Q and K are rotated first."""
    rng = np.random.default_rng(44)
    B, N, H, d = 1, 256, 2, 128
    q = rng.standard_normal((B, N, H, d)).astype(np.float32)
    k = rng.standard_normal((B, N, H, d)).astype(np.float32)
    v = rng.standard_normal((B, N, H, d)).astype(np.float32)
    for ch in (3, 77):
        q[..., ch] *= 40.0
        k[..., ch] *= 40.0
    sc = 1 / math.sqrt(d) / 40.0
    O, _ = oracle.attention(q, k, v, sc, False)
    s = np.where(rng.random(d) < 0.5, -1.0, 1.0).astype(np.float32)
    errs = {}
    for name, signs in (("rotated", s), ("plain", None)):
        qc, qa = oracle.fp8_quantize(q, signs)
        kc, ka = oracle.fp8_quantize(k, signs)
        vc, va = oracle.fp8_quantize(v)
        O8, _ = oracle.attention(oracle.fp8_dequantize(qc, qa), oracle.fp8_dequantize(kc, ka),
                                 oracle.fp8_dequantize(vc, va), sc, False)
        errs[name] = np.abs(O8 - O).mean()
    assert errs["rotated"] < 0.5 * errs["plain"], errs
