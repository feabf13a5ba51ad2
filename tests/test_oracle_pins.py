"""Pins for the CPU oracle: each check fixes the oracle against something other than itself.

The pages print no worked example, so the pins are closed forms derived by hand (golden file),
invariants the definition implies, special cases that reduce to a library routine, and brute force
in plain Python on tiny inputs. Each is chosen so that a plausible slip in the oracle (a dropped
scale, a wrong sign, a transposed operand, a wrong mask offset, a wrong GQA head map) fails one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _case(rng, B=1, Hq=2, Hkv=2, Nq=7, Nkv=9, d=5):
    return _rand(rng, B, Nq, Hq, d), _rand(rng, B, Nkv, Hkv, d), _rand(rng, B, Nkv, Hkv, d)


# -------------------------------------------------------------------------------------------
# golden closed forms (derived by hand; the derivation is stored beside each case)
# -------------------------------------------------------------------------------------------

def test_golden_closed_forms():
    with open(os.path.join(HERE, "golden", "closed_form.json")) as f:
        cases = json.load(f)["cases"]
    assert len(cases) >= 5
    for c in cases:
        q = np.array(c["q"], dtype=np.float64)[None, :, None, :]
        k = np.array(c["k"], dtype=np.float64)[None, :, None, :]
        v = np.array(c["v"], dtype=np.float64)[None, :, None, :]
        O, L = oracle.attention(q, k, v, c["scale"], c["causal"])
        exp_O = np.array(c["O"], dtype=np.float64)
        exp_L = np.array([float(x) for x in c["LSE"]], dtype=np.float64)
        np.testing.assert_allclose(O[0, :, 0, :], exp_O, rtol=0, atol=1e-12, err_msg=c["name"])
        np.testing.assert_allclose(L[0, 0, :], exp_L, rtol=0, atol=1e-12, err_msg=c["name"])


def test_golden_probabilities():
    """oracle.probabilities against the hand-derived P of each golden case (a dropped or inverted
    scale, or negated scores, change these values; a per-row constant does not, hence the LSE pins)."""
    with open(os.path.join(HERE, "golden", "closed_form.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        P = oracle.probabilities(np.array(c["q"], dtype=np.float64), np.array(c["k"], dtype=np.float64),
                                 c["scale"], c["causal"])
        np.testing.assert_allclose(P, np.array(c["P"], dtype=np.float64), rtol=0, atol=1e-12, err_msg=c["name"])


# -------------------------------------------------------------------------------------------
# invariants and special cases
# -------------------------------------------------------------------------------------------

@pytest.mark.parametrize("causal,Nq,Nkv", [(False, 6, 9), (True, 6, 9), (True, 9, 9), (True, 9, 4)])
def test_probability_rows_sum_to_one(causal, Nq, Nkv):
    rng = np.random.default_rng(1)
    q, k = _rand(rng, Nq, 8), _rand(rng, Nkv, 8)
    P = oracle.probabilities(q, k, 0.3, causal)
    vis = oracle.visibility_mask(Nq, Nkv, causal)
    assert np.all(P[~vis] == 0.0)
    rows = vis.any(axis=1)
    np.testing.assert_allclose(P[rows].sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(P[~rows] == 0.0)
    assert np.all(P >= 0.0)


@pytest.mark.parametrize("causal,Nq,Nkv", [(False, 5, 8), (True, 8, 8), (True, 5, 8), (True, 8, 5)])
def test_equal_scores_give_column_mean(causal, Nq, Nkv):
    """Q = 0 makes all scores equal: O[i] = mean of V over Vis(i), LSE[i] = ln |Vis(i)|."""
    rng = np.random.default_rng(2)
    d = 6
    q = np.zeros((1, Nq, 2, d))
    k, v = _rand(rng, 1, Nkv, 2, d), _rand(rng, 1, Nkv, 2, d)
    O, L = oracle.attention(q, k, v, 0.7, causal)
    for h, i in itertools.product(range(2), range(Nq)):
        n = i + Nkv - Nq + 1 if causal else Nkv
        n = max(0, min(Nkv, n))
        if n == 0:
            assert np.all(O[0, i, h] == 0) and L[0, h, i] == -np.inf
            continue
        np.testing.assert_allclose(O[0, i, h], v[0, :n, h].mean(axis=0), rtol=0, atol=1e-12)
        assert abs(L[0, h, i] - math.log(n)) < 1e-12


def test_one_hot_dominant_key():
    """A key aligned with q and 40+ nats above the rest returns its own V row and score."""
    rng = np.random.default_rng(3)
    d, N, jstar = 16, 12, 7
    scale = 1 / math.sqrt(d)
    q = _rand(rng, d)
    k = 1e-3 * _rand(rng, N, d)
    k[jstar] = 64.0 * q / np.linalg.norm(q) * math.sqrt(d)
    v = _rand(rng, N, d)
    s_star = scale * q @ k[jstar]
    assert s_star - max(scale * q @ k[j] for j in range(N) if j != jstar) > 40
    O, L = oracle.attention(q[None, None, None, :], k[None, :, None, :], v[None, :, None, :], scale, False)
    np.testing.assert_allclose(O[0, 0, 0], v[jstar], rtol=0, atol=math.exp(-40) * np.abs(v).max() * N)
    assert abs(L[0, 0, 0] - s_star) < 1e-12


def test_causal_first_row_is_first_value():
    rng = np.random.default_rng(4)
    q, k, v = _case(rng, Nq=10, Nkv=10)
    O, L = oracle.attention(q, k, v, 0.45, True)
    for h in range(2):
        assert np.array_equal(O[0, 0, h], v[0, 0, h])
        assert abs(L[0, h, 0] - 0.45 * q[0, 0, h] @ k[0, 0, h]) < 1e-15


def test_single_key_closed_form():
    rng = np.random.default_rng(5)
    q, k, v = _case(rng, Nq=3, Nkv=1)
    O, L = oracle.attention(q, k, v, 1.3, False)
    for h, i in itertools.product(range(2), range(3)):
        assert np.array_equal(O[0, i, h], v[0, 0, h])
        assert abs(L[0, h, i] - 1.3 * q[0, i, h] @ k[0, 0, h]) < 1e-12


def test_two_keys_is_a_sigmoid():
    rng = np.random.default_rng(6)
    q, k, v = _case(rng, Nq=4, Nkv=2, d=3)
    sc = 0.9
    O, L = oracle.attention(q, k, v, sc, False)
    for h, i in itertools.product(range(2), range(4)):
        s0, s1 = sc * q[0, i, h] @ k[0, 0, h], sc * q[0, i, h] @ k[0, 1, h]
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))
        np.testing.assert_allclose(O[0, i, h], (1 - w1) * v[0, 0, h] + w1 * v[0, 1, h], rtol=0, atol=1e-12)
        assert abs(L[0, h, i] - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) < 1e-12


def test_causal_rows_with_no_visible_key():
    rng = np.random.default_rng(7)
    q, k, v = _case(rng, Nq=9, Nkv=4)
    O, L = oracle.attention(q, k, v, 0.5, True)
    assert np.all(O[0, :5] == 0) and np.all(L[0, :, :5] == -np.inf)
    assert np.all(np.isfinite(L[0, :, 5:]))


# -------------------------------------------------------------------------------------------
# brute force in plain Python (no numpy in the arithmetic)
# -------------------------------------------------------------------------------------------

def _brute(q, k, v, scale, causal):
    B, Nq, Hq, d = q.shape
    Nkv, Hkv = k.shape[1], k.shape[2]
    O = [[[[0.0] * d for _ in range(Hq)] for _ in range(Nq)] for _ in range(B)]
    L = [[[-math.inf] * Nq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h * Hkv // Hq
            for i in range(Nq):
                keys = [j for j in range(Nkv) if (not causal) or j - (Nkv - Nq) <= i]
                if not keys:
                    continue
                s = {j: scale * sum(float(q[b, i, h, t]) * float(k[b, j, g, t]) for t in range(d)) for j in keys}
                m = max(s.values())
                z = sum(math.exp(x - m) for x in s.values())
                for t in range(d):
                    O[b][i][h][t] = sum(math.exp(s[j] - m) / z * float(v[b, j, g, t]) for j in keys)
                L[b][h][i] = m + math.log(z)
    return np.array(O), np.array(L)


@pytest.mark.parametrize("Hq,Hkv,Nq,Nkv,causal", [
    (2, 2, 5, 5, False), (2, 2, 5, 5, True), (4, 2, 3, 7, True), (4, 1, 7, 3, True), (3, 3, 6, 2, False),
])
def test_brute_force_tiny(Hq, Hkv, Nq, Nkv, causal):
    rng = np.random.default_rng(8 + Nq)
    q, k, v = _case(rng, B=2, Hq=Hq, Hkv=Hkv, Nq=Nq, Nkv=Nkv, d=4)
    O, L = oracle.attention(q, k, v, 0.6, causal)
    Ob, Lb = _brute(q, k, v, 0.6, causal)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(L), np.isinf(Lb))
    np.testing.assert_allclose(L[np.isfinite(L)], Lb[np.isfinite(Lb)], rtol=0, atol=1e-12)


@pytest.mark.parametrize("Nq,Nkv,causal,qscale", [
    (5, 7, False, 2.0), (7, 7, True, 2.0), (3, 6, True, 2.0), (6, 3, True, 2.0),
    (5, 7, False, 600.0), (7, 7, True, 600.0),  # scores in the hundreds: exp overflows without a max shift
])
def test_probabilities_brute_force(Nq, Nkv, causal, qscale):
    """P entry by entry in plain Python: exp(s_ij - m_i) / sum over visible j of exp(s_ij - m_i),
    with m_i the row's largest visible score (the same ratio as exp(s_ij) / sum exp(s_ij))."""
    rng = np.random.default_rng(30 + Nq + Nkv)
    q, k = qscale * _rand(rng, Nq, 4), _rand(rng, Nkv, 4)
    P = oracle.probabilities(q, k, 0.7, causal)
    assert np.all(np.isfinite(P))
    for i in range(Nq):
        keys = [j for j in range(Nkv) if (not causal) or j <= i + Nkv - Nq]
        s = {j: 0.7 * sum(float(q[i, t]) * float(k[j, t]) for t in range(4)) for j in keys}
        if not s:  # a row that sees no key is all zero
            assert np.all(P[i] == 0.0)
            continue
        m = max(s.values())
        z = sum(math.exp(x - m) for x in s.values())
        for j in range(Nkv):
            want = math.exp(s[j] - m) / z if j in s else 0.0
            assert abs(P[i, j] - want) < 1e-12, (i, j)


# -------------------------------------------------------------------------------------------
# an independent library routine
# -------------------------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_fp64_on_tiny_workload(causal):
    """torch's softmax / logsumexp / sdpa in fp64 on the CPU agree with the oracle (Nq = Nkv)."""
    import torch

    rng = np.random.default_rng(9)
    q, k, v = _case(rng, B=1, Hq=2, Hkv=2, Nq=64, Nkv=64, d=16)
    sc = 1 / 4
    O, L = oracle.attention(q, k, v, sc, causal)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    S = sc * tq @ tk.transpose(-1, -2)
    if causal:
        S = S.masked_fill(torch.ones(64, 64, dtype=torch.bool).triu(1), float("-inf"))
    ref_O = (torch.softmax(S, dim=-1) @ tv).permute(0, 2, 1, 3).numpy()
    ref_L = torch.logsumexp(S, dim=-1).numpy()
    np.testing.assert_allclose(O, ref_O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, ref_L, rtol=0, atol=1e-12)
    sdpa = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=sc)
    np.testing.assert_allclose(O, sdpa.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


# -------------------------------------------------------------------------------------------
# structure: GQA, linearity, equivariance
# -------------------------------------------------------------------------------------------

def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(10)
    q, k, v = _case(rng, B=2, Hq=8, Hkv=2, Nq=6, Nkv=6, d=4)
    for causal in (False, True):
        O1, L1 = oracle.attention(q, k, v, 0.5, causal)
        O2, L2 = oracle.attention(q, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2), 0.5, causal)
        assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_linear_in_v_and_key_permutation_invariant():
    rng = np.random.default_rng(11)
    q, k, v = _case(rng, Nq=5, Nkv=11)
    O, L = oracle.attention(q, k, v, 0.8, False)
    O2, L2 = oracle.attention(q, k, -2.5 * v, 0.8, False)
    np.testing.assert_allclose(O2, -2.5 * O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L, rtol=0, atol=0)
    perm = rng.permutation(11)
    O3, L3 = oracle.attention(q, k[:, perm], v[:, perm], 0.8, False)
    np.testing.assert_allclose(O3, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L3, L, rtol=0, atol=1e-12)
    # shifting every score of row i by the same amount a_i moves LSE[i] by a_i and leaves O alone:
    # append a coordinate a_i / scale to q_i and 1 to every key
    a = rng.uniform(-3.0, 3.0, size=(1, 5, 2))
    q5 = np.concatenate([q, (a / 0.8)[..., None]], axis=-1)
    k5 = np.concatenate([k, np.ones(k.shape[:-1] + (1,))], axis=-1)
    v5 = np.concatenate([v, np.zeros(v.shape[:-1] + (1,))], axis=-1)
    O4, L4 = oracle.attention(q5, k5, v5, 0.8, False)
    np.testing.assert_allclose(O4[..., :-1], O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L4, L + a.transpose(0, 2, 1), rtol=0, atol=1e-12)


def test_scale_enters_as_a_factor_on_scores():
    rng = np.random.default_rng(12)
    q, k, v = _case(rng, Nq=4, Nkv=6)
    O1, L1 = oracle.attention(q, k, v, 0.5, False)
    O2, L2 = oracle.attention(2 * q, k, v, 0.25, False)
    np.testing.assert_allclose(O1, O2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L1, L2, rtol=0, atol=1e-12)


# -------------------------------------------------------------------------------------------
# exactness: the tiled online-softmax route equals the materialised one
# -------------------------------------------------------------------------------------------

def _random_tiles(rng, n):
    tiles = []
    while sum(tiles) < n:
        tiles.append(int(min(n - sum(tiles), rng.integers(1, 12))))
    return tiles


@pytest.mark.parametrize("Nq,Nkv,d,causal", [
    (17, 17, 4, False), (17, 17, 8, True), (9, 33, 16, True), (33, 9, 32, True), (40, 64, 64, False),
    (1, 50, 128, False), (64, 64, 256, True),
])
def test_tiled_online_softmax_is_exact(Nq, Nkv, d, causal):
    rng = np.random.default_rng(Nq * 100 + Nkv)
    q, k, v = _rand(rng, Nq, d), _rand(rng, Nkv, d), _rand(rng, Nkv, d)
    # large score spread exercises the running-max rescale
    q *= 3.0
    sc = 1 / math.sqrt(d)
    O, L = oracle.attention(q[None, :, None], k[None, :, None], v[None, :, None], sc, causal)
    for q_tile in (1, 5, 16):
        for tiles in ([1] * Nkv, _random_tiles(rng, Nkv), [Nkv]):
            Ot, Lt = oracle.tiled_online_softmax(q, k, v, sc, causal, q_tile, tiles)
            np.testing.assert_allclose(Ot, O[0, :, 0], rtol=1e-12, atol=1e-12)
            fin = np.isfinite(L[0, 0])
            np.testing.assert_array_equal(np.isfinite(Lt), fin)
            np.testing.assert_allclose(Lt[fin], L[0, 0][fin], rtol=1e-12, atol=1e-12)


# -------------------------------------------------------------------------------------------
# decode: split-combine identity and reduction to the prefill definition
# -------------------------------------------------------------------------------------------

def test_split_combine_identity():
    rng = np.random.default_rng(13)
    n, d = 257, 32
    q, k, v = _rand(rng, d), _rand(rng, n, d), _rand(rng, n, d)
    whole = oracle.attention_row(q, k, v, 0.2)
    for _ in range(20):
        cuts = sorted(set(rng.integers(0, n + 1, size=int(rng.integers(1, 9))).tolist()) | {0, n})
        bounds = list(zip(cuts[:-1], cuts[1:])) + [(n, n)]  # includes an empty partition
        o, lse = oracle.merge_partials(oracle.split_partials(q, k, v, 0.2, bounds))
        np.testing.assert_allclose(o, whole[0], rtol=0, atol=1e-12)
        assert abs(lse - whole[1]) < 1e-12


def test_decode_is_prefill_with_one_query_row():
    rng = np.random.default_rng(14)
    B, Hq, Hkv, cap, d = 3, 8, 2, 40, 16
    q = _rand(rng, B, Hq, d)
    kc, vc = _rand(rng, B, cap, Hkv, d), _rand(rng, B, cap, Hkv, d)
    lens = np.array([40, 1, 17])
    O, L = oracle.decode(q, kc, vc, lens, 0.25)
    for b in range(B):
        Op, Lp = oracle.attention(q[b][None, None], kc[b:b + 1, :lens[b]], vc[b:b + 1, :lens[b]], 0.25, False)
        np.testing.assert_allclose(O[b], Op[0, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(L[b], Lp[0, :, 0], rtol=0, atol=1e-12)
    O0, L0 = oracle.decode(q, kc, vc, np.array([0, 3, 5]), 0.25)
    assert np.all(O0[0] == 0) and np.all(L0[0] == -np.inf)


def test_attention_row_agrees_with_full_oracle_causal():
    rng = np.random.default_rng(15)
    q, k, v = _case(rng, B=1, Hq=4, Hkv=2, Nq=12, Nkv=20, d=8)
    O, L = oracle.attention(q, k, v, 0.4, True)
    for i, h in [(0, 0), (5, 3), (11, 1)]:
        g = oracle.kv_head(h, 4, 2)
        keys = oracle.visible_keys(i, 12, 20, True)
        o, lse = oracle.attention_row(q[0, i, h], k[0, keys, g], v[0, keys, g], 0.4)
        np.testing.assert_allclose(o, O[0, i, h], rtol=0, atol=1e-12)
        assert abs(lse - L[0, h, i]) < 1e-12
