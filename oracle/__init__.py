"""CPU fp64 oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The library's product path (the CUDA kernels behind the C ABI
and their Python binding) never calls it, and this package imports nothing from the library.

What it computes, and from which passage of the pages:

* The function itself: every FlashAttention version computes the same dense attention,
  O = softmax(Q K^T) V  -- "FlashAttention evolution" article (sandeep007734.github.io), section 1
  "The Invariant and the Moving Bottleneck". The overview page "Flash Attention"
  (vladislavkruglikov.com), opening paragraph, calls it *scaled* dot-product attention with scores S,
  probabilities P and output O; its equation block was lost in extraction, so the scale is read as a
  caller-supplied factor on Q K^T (the workloads use 1/sqrt(d)).
* Exactness: tiling "changes the order and location of the computation, not the attention function"
  -- "Flash Attention" overview, section "The IO problem". Hence the parity oracle is the plain
  definition with S and P materialised (:func:`attention`), and the tiled online-softmax recurrence
  (:func:`tiled_online_softmax`) is a second, independent route used only to pin the first.
* Per-row metadata written beside O -- same section; read as the natural-log log-sum-exp of the
  scaled scores, LSE[i] = log sum_j exp(s_ij).
* Delayed normalisation (divide the accumulator once, at the end) -- evolution article, section 3
  "FlashAttention-2".
* Flash-Decoding: partial maxima, normalisation sums and weighted outputs over KV partitions,
  merged with the same online-softmax identity -- evolution article, section 6 "Flash-Decoding:
  A Different Parallel Shape" (:func:`split_partials`, :func:`merge_partials`).

Readings where the pages are silent (each is listed with its reason in the design notes):
softmax is row-wise over keys; the causal mask is bottom-right aligned (key j visible to query i
iff j <= i + Nkv - Nq); GQA groups are contiguous (kv head = hq // (Hq // Hkv)); a row with no
visible key has O = 0 and LSE = -inf; layouts are token-major, Q/O [B, Nq, Hq, d],
K/V [B, Nkv, Hkv, d], LSE [B, Hq, Nq].

All arithmetic is fp64. Inputs are the bf16 values the GPU receives, widened exactly.
Every function here is pinned by a check that does not restate it (tests/test_oracle_pins.py).
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def kv_head(hq: int, Hq: int, Hkv: int) -> int:
    """GQA reading: query head hq reads kv head hq // (Hq / Hkv) (contiguous groups)."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def visible_keys(i: int, Nq: int, Nkv: int, causal: bool) -> np.ndarray:
    """Indices of the keys query row i attends to (bottom-right aligned causal mask)."""
    if not causal:
        return np.arange(Nkv)
    last = i + Nkv - Nq
    return np.arange(max(0, min(Nkv, last + 1)))


def visibility_mask(Nq: int, Nkv: int, causal: bool) -> np.ndarray:
    """Boolean [Nq, Nkv]: True where key j is visible to query i."""
    if not causal:
        return np.ones((Nq, Nkv), dtype=bool)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nkv)[None, :]
    return j <= i + (Nkv - Nq)


def probabilities(q_bh: np.ndarray, k_bg: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """P = softmax(scale * Q K^T) row-wise over visible keys, materialised, [Nq, Nkv] fp64.

    Rows with no visible key are all zero.
    """
    Nq, Nkv = q_bh.shape[0], k_bg.shape[0]
    S = scale * (q_bh @ k_bg.T)
    vis = visibility_mask(Nq, Nkv, causal)
    S = np.where(vis, S, NEG_INF)
    has = vis.any(axis=1)
    M = np.where(has, S.max(axis=1, initial=NEG_INF), 0.0)
    E = np.where(vis, np.exp(S - M[:, None]), 0.0)
    Z = E.sum(axis=1)
    return np.where(has[:, None], E / np.where(has, Z, 1.0)[:, None], 0.0)


def _one_head(q_bh, k_bg, v_bg, scale, causal):
    """O and LSE for one (batch, query head): S, then P, then O = P V, all materialised."""
    Nq, Nkv = q_bh.shape[0], k_bg.shape[0]
    vis = visibility_mask(Nq, Nkv, causal)
    has = vis.any(axis=1)
    S = scale * (q_bh @ k_bg.T)
    S[~vis] = NEG_INF
    M = S.max(axis=1, initial=NEG_INF)
    M[~has] = 0.0
    S -= M[:, None]
    np.exp(S, out=S)                      # exp(-inf) = 0 on masked entries
    Z = S.sum(axis=1)
    Zs = np.where(has, Z, 1.0)
    S /= Zs[:, None]                      # S now holds P
    O = S @ v_bg
    O[~has] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.where(has, M + np.log(Zs), NEG_INF)
    return O, lse


def attention(q, k, v, scale: float, causal: bool):
    """Exact attention, plain definition.

    q: [B, Nq, Hq, d], k and v: [B, Nkv, Hkv, d] (fp64 or anything numpy widens exactly).
    Returns O [B, Nq, Hq, d] fp64 and LSE [B, Hq, Nq] fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, Hq, d = q.shape
    _, Nkv, Hkv, _ = k.shape
    O = np.zeros((B, Nq, Hq, d))
    LSE = np.full((B, Hq, Nq), NEG_INF)
    for b in range(B):
        for hq in range(Hq):
            g = kv_head(hq, Hq, Hkv)
            O[b, :, hq, :], LSE[b, hq, :] = _one_head(
                np.ascontiguousarray(q[b, :, hq, :]), np.ascontiguousarray(k[b, :, g, :]),
                np.ascontiguousarray(v[b, :, g, :]), scale, causal)
    return O, LSE


def attention_row(q_row, k_vis, v_vis, scale: float):
    """One output row from the keys it sees: (o [d], lse). Used for sampled full-size checks."""
    q_row = np.asarray(q_row, dtype=np.float64)
    k_vis = np.asarray(k_vis, dtype=np.float64)
    v_vis = np.asarray(v_vis, dtype=np.float64)
    if k_vis.shape[0] == 0:
        return np.zeros(q_row.shape[0]), NEG_INF
    s = scale * (k_vis @ q_row)
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    return (e / z) @ v_vis, m + np.log(z)


def decode(q, k_cache, v_cache, kv_lens, scale: float):
    """Single-query decode: row (b, hq) attends to keys [0, kv_lens[b]) of kv head hq // group.

    q: [B, Hq, d]; caches: [B, Nkv_cap, Hkv, d]. Returns O [B, Hq, d] and LSE [B, Hq].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = k_cache.shape[2]
    O = np.zeros((B, Hq, d))
    LSE = np.full((B, Hq), NEG_INF)
    for b in range(B):
        L = int(kv_lens[b])
        for hq in range(Hq):
            g = kv_head(hq, Hq, Hkv)
            O[b, hq], LSE[b, hq] = attention_row(q[b, hq], k_cache[b, :L, g, :], v_cache[b, :L, g, :], scale)
    return O, LSE


# ------------------------------------------------------------------------------------------------
# The tiled route. Used only to pin the plain definition above (exactness), never for parity.
# ------------------------------------------------------------------------------------------------

def tiled_online_softmax(q_bh, k_bg, v_bg, scale: float, causal: bool, q_tile: int, k_tiles):
    """FlashAttention's tiled forward for one head, following the pages' steps.

    Query rows are taken a block at a time (query-block parallelism, evolution article section 3).
    For each block, key/value tiles of the given sizes are visited in order; each score tile is
    produced, folded into the running state (row max m, row sum l, unnormalised accumulator acc) and
    discarded (section 1). The accumulator is divided by l once after the last tile (delayed
    normalisation, section 3). ``k_tiles`` is a list of tile widths that sums to Nkv.
    """
    q_bh = np.asarray(q_bh, dtype=np.float64)
    Nq, d = q_bh.shape
    Nkv = k_bg.shape[0]
    assert sum(k_tiles) == Nkv
    O = np.zeros((Nq, d))
    LSE = np.full(Nq, NEG_INF)
    for r0 in range(0, Nq, q_tile):
        rows = np.arange(r0, min(Nq, r0 + q_tile))
        m = np.full(len(rows), NEG_INF)
        l = np.zeros(len(rows))
        acc = np.zeros((len(rows), d))
        c0 = 0
        for w in k_tiles:
            cols = np.arange(c0, c0 + w)
            c0 += w
            s = scale * (q_bh[rows] @ k_bg[cols].T)
            if causal:
                s = np.where(cols[None, :] <= rows[:, None] + (Nkv - Nq), s, NEG_INF)
            m_new = np.maximum(m, s.max(axis=1))
            live = m_new > NEG_INF
            ref = np.where(live, m_new, 0.0)
            alpha = np.where(live, np.exp(np.where(live, m - ref, 0.0)), 1.0)
            alpha = np.where(m == NEG_INF, 0.0, alpha)
            p = np.exp(s - ref[:, None])
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ v_bg[cols]
            m = m_new
        done = l > 0
        O[rows] = np.where(done[:, None], acc / np.where(done, l, 1.0)[:, None], 0.0)
        with np.errstate(divide="ignore"):
            LSE[rows] = np.where(done, m + np.log(np.where(done, l, 1.0)), NEG_INF)
    return O, LSE


def split_partials(q_row, k_vis, v_vis, scale: float, bounds):
    """Flash-Decoding partitions: for each KV range [a, b) the partial (max, sum, weighted output).

    Evolution article, section 6: each partition independently computes a partial maximum, a
    normalisation sum and a weighted output. Returned per partition as (lse_s, o_s) with o_s
    normalised by its own sum; an empty partition gives (-inf, 0).
    """
    parts = []
    for a, b in bounds:
        parts.append(attention_row(q_row, k_vis[a:b], v_vis[a:b], scale))
    return parts


def merge_partials(parts):
    """Merge partition states with the online-softmax identity (evolution article, section 6).

    LSE = log sum_s exp(lse_s); O = sum_s exp(lse_s - LSE) o_s.
    """
    lses = np.array([p[1] for p in parts], dtype=np.float64)
    if np.all(lses == NEG_INF):
        return np.zeros_like(parts[0][0]), NEG_INF
    mx = lses.max()
    w = np.exp(lses - mx)
    z = w.sum()
    o = sum(wi * p[0] for wi, p in zip(w, parts)) / z
    return o, mx + np.log(z)


# ------------------------------------------------------------------------------------------------
# 8-bit path: incoherent processing and e4m3 quantization, then attention on the decoded values.
# FP8 with incoherent processing is named by the "Flash Attention" overview (FA-3 paragraph) and the
# FlashAttention generation comparison record (FA-3 "Workarounds"); the pages give no recipe, so the
# steps below are this library's reading: rotate Q and K by diag(s) H / sqrt(d) (H the Sylvester
# Hadamard matrix, s a sign vector), scale each (batch, head) so its largest |value| maps to 448,
# round to e4m3 (nearest even, saturating). Q K^T is unchanged by the rotation in exact arithmetic.
# The codes are an encoding, so the oracle follows the same fp32 steps in the same order (the
# butterfly stages of the fast Walsh-Hadamard transform, then the fp32 products); the attention on
# the decoded values is the plain definition above, in fp64.
# ------------------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 code (uint8): sign bit 7, exponent bits 6-3 (bias 7), mantissa bits 2-0;
    exponent 0 is subnormal (m/8 * 2^-6); 0x7F / 0xFF are NaN (no infinities)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


_E4M3_GRID = None


def e4m3_round(x) -> np.ndarray:
    """Codes of fp32 values rounded to the nearest e4m3 value (ties to the even code), saturating
    at +-448; x must be finite."""
    global _E4M3_GRID
    if _E4M3_GRID is None:
        pos = np.arange(0, 0x7F, dtype=np.uint8)            # 0 .. 0x7E: +0 .. 448, increasing
        _E4M3_GRID = (pos, e4m3_decode(pos))
    pos, grid = _E4M3_GRID
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(grid, a, side="left")               # first grid value >= a
    hi = np.minimum(hi, len(grid) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (pos[hi] % 2 == 0))
    idx = np.where(a == grid[hi], hi, np.where(pick_hi, hi, lo))
    code = pos[idx].astype(np.uint8)
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)  # the sign survives rounding to 0


def hadamard_rotate_f32(x, signs) -> np.ndarray:
    """Rows of x (last axis d, a power of two) times diag(signs) H / sqrt(d), in fp32: sign flip,
    butterflies (a, b) -> (a + b, a - b) for h = 1, 2, ..., d/2 on pairs (j, j + h) inside blocks of
    2h, then one fp32 product with fp32(1/sqrt(d))."""
    y = np.asarray(x, dtype=np.float32) * np.asarray(signs, dtype=np.float32)
    d = y.shape[-1]
    lead = y.shape[:-1]
    h = 1
    while h < d:
        z = y.reshape(lead + (d // (2 * h), 2, h))
        a, b = z[..., 0, :], z[..., 1, :]
        y = np.stack((a + b, a - b), axis=-2).reshape(lead + (d,)).astype(np.float32)
        h *= 2
    return (y * np.float32(1.0 / np.sqrt(d))).astype(np.float32)


def fp8_quantize(x, signs=None):
    """Codes and per-head maxima of x [B, N, H, d] (values exactly representable in fp32, e.g. bf16).

    Returns (codes uint8 [B, N, H, d], amax fp32 [B, H]); code = e4m3(fp32(y * fp32(448 / amax)))
    with y the rotated rows (or x itself without signs) and amax = max |y| over the head (scale 1
    when amax = 0)."""
    y = np.asarray(x, dtype=np.float32)
    if signs is not None:
        y = hadamard_rotate_f32(y, signs)
    amax = np.abs(y).max(axis=(1, 3)).astype(np.float32)                      # [B, H]
    scale = np.where(amax > 0, np.float32(E4M3_MAX) / np.where(amax > 0, amax, 1), 1).astype(np.float32)
    codes = e4m3_round((y * scale[:, None, :, None]).astype(np.float32))
    return codes, amax


def fp8_dequantize(codes, amax) -> np.ndarray:
    """Values the codes stand for: code value * amax / 448 per (batch, head), fp64; [B, N, H, d]."""
    return e4m3_decode(codes) * (np.asarray(amax, dtype=np.float64) / E4M3_MAX)[:, None, :, None]


# ------------------------------------------------------------------------------------------------
# Backward pass. The FlashAttention generation comparison record ("Workarounds", FA-1) recomputes S
# in the backward pass instead of storing it; what the pass computes is the gradient of the exact
# forward above. With L a scalar loss and dO = dL/dO, per (batch, query head), materialised in fp64:
#   P = softmax(scale * Q K^T) (visible keys),  dV = P^T dO,  dP = dO V^T,
#   D_i = sum_j P_ij dP_ij,  dS = P * (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q,
# and dK, dV of a kv head are the sums over the query heads that read it (GQA).
# ------------------------------------------------------------------------------------------------

def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Gradients (dQ [B, Nq, Hq, d], dK, dV [B, Nkv, Hkv, d]) of sum(O * dO) for O = attention(...)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, Nq, Hq, d = q.shape
    _, Nkv, Hkv, _ = k.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for hq in range(Hq):
            g = kv_head(hq, Hq, Hkv)
            P = probabilities(q[b, :, hq], k[b, :, g], scale, causal)
            dO = do[b, :, hq]
            dv[b, :, g] += P.T @ dO
            dP = dO @ v[b, :, g].T
            Dd = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - Dd)
            dq[b, :, hq] = scale * (dS @ k[b, :, g])
            dk[b, :, g] += scale * (dS.T @ q[b, :, hq])
    return dq, dk, dv
