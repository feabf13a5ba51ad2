"""Pins for the oracle's backward pass: central finite differences of the forward oracle, GQA as
MHA with repeated K/V heads summed per group, and closed forms (one key, the causal first row)."""
import math

import numpy as np
import pytest

import oracle


def _loss(q, k, v, do, sc, causal):
    O, _ = oracle.attention(q, k, v, sc, causal)
    return float((O * do).sum())


@pytest.mark.parametrize("Hq,Hkv,Nq,Nkv,causal", [(2, 2, 5, 7, False), (2, 1, 6, 6, True), (4, 2, 7, 4, True)])
def test_gradients_match_central_differences(Hq, Hkv, Nq, Nkv, causal):
    rng = np.random.default_rng(50 + Nq * Nkv)
    d = 4
    q = rng.standard_normal((1, Nq, Hq, d))
    k = rng.standard_normal((1, Nkv, Hkv, d))
    v = rng.standard_normal((1, Nkv, Hkv, d))
    do = rng.standard_normal((1, Nq, Hq, d))
    sc = 0.7
    dq, dk, dv = oracle.attention_backward(q, k, v, do, sc, causal)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, sc, causal)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, sc, causal)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=1e-7, err_msg=name)


def test_gqa_gradients_are_group_sums_of_repeated_heads():
    rng = np.random.default_rng(60)
    q = rng.standard_normal((2, 5, 4, 3))
    k = rng.standard_normal((2, 6, 2, 3))
    v = rng.standard_normal((2, 6, 2, 3))
    do = rng.standard_normal((2, 5, 4, 3))
    for causal in (False, True):
        dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, causal)
        dq2, dk2, dv2 = oracle.attention_backward(q, np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2), do, 0.5, causal)
        np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(dk, dk2.reshape(2, 6, 2, 2, 3).sum(axis=3), rtol=0, atol=1e-13)
        np.testing.assert_allclose(dv, dv2.reshape(2, 6, 2, 2, 3).sum(axis=3), rtol=0, atol=1e-13)


def test_single_key_and_causal_first_row():
    rng = np.random.default_rng(61)
    q = rng.standard_normal((1, 4, 1, 5))
    k = rng.standard_normal((1, 1, 1, 5))
    v = rng.standard_normal((1, 1, 1, 5))
    do = rng.standard_normal((1, 4, 1, 5))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.9, False)
    # one key: P = 1 whatever the scores, so the scores get no gradient and dV sums dO
    assert np.all(dq == 0) and np.all(dk == 0)
    np.testing.assert_allclose(dv[0, 0, 0], do[0, :, 0].sum(axis=0), rtol=0, atol=1e-14)
    q = rng.standard_normal((1, 6, 1, 5))
    k = rng.standard_normal((1, 6, 1, 5))
    v = rng.standard_normal((1, 6, 1, 5))
    do = rng.standard_normal((1, 6, 1, 5))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.9, True)
    # causal: row 0 sees key 0 alone (no gradient into q_0); the last key is seen only by the last row
    assert np.all(dq[0, 0] == 0)
    O, _ = oracle.attention(q, k, v, 0.9, True)
    P_last = math.exp(0.9 * q[0, 5, 0] @ k[0, 5, 0] - oracle.attention(q, k, v, 0.9, True)[1][0, 0, 5])
    np.testing.assert_allclose(dv[0, 5, 0], P_last * do[0, 5, 0], rtol=0, atol=1e-13)
