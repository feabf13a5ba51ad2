"""Seeded synthetic inputs for the attention workloads (test and benchmark infrastructure).

This module holds no attention arithmetic. It only draws the bf16 Q, K, V tensors and the decode
KV lengths that both the CPU oracle and the CUDA library are fed, so that the two sides see the
same bits while sharing no code.

The generator is counter based: element ``i`` of stream ``t`` under seed ``s`` is a pure function
of ``(s, t, i)``. Any slice can therefore be drawn on its own (the oracle draws only the rows it
checks), and the host (numpy) and device (torch) implementations give the same values.

Recipe
------
* ``mix(x)`` is the splitmix64 finaliser (Steele, Lea and Flood, "Fast splittable pseudorandom
  number generators", OOPSLA 2014)::

      x ^= x >> 30;  x *= 0xBF58476D1CE4E5B9
      x ^= x >> 27;  x *= 0x94D049BB133111EB
      x ^= x >> 31                                   (all mod 2**64)

* stream base ``b = mix(16 * seed + t)``; counter ``c`` yields ``mix(b + (c + 1) * 0x9E3779B97F4A7C15)``.
* a uniform in [0, 1) is the top 53 bits of that word times 2**-53.
* N(0, 1) values come from Box-Muller (1958) on counter pairs ``(2p, 2p + 1)``:
  ``r = sqrt(-2 ln(1 - u_2p))``, ``theta = 2 pi u_(2p+1)``; element ``2p`` is ``r cos theta`` and
  element ``2p + 1`` is ``r sin theta``, in fp64.
* bf16 rounding: fp64 -> fp32 (round to nearest even), then fp32 -> bf16 (round to nearest even on
  the bit pattern).
* Stream ids: 0 = Q, 1 = K, 2 = V, 3 = decode KV lengths. A decode length is
  ``lo + floor(u_c * (hi - lo + 1))`` for ``c = 0 .. B-1``.

Tensor layouts are token-major: Q and O ``[B, Nq, Hq, d]``, K and V ``[B, Nkv, Hkv, d]``; the decode
query is ``[B, Hq, d]`` and the KV cache ``[B, Nkv_cap, Hkv, d]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

STREAM_Q, STREAM_K, STREAM_V, STREAM_LENS = 0, 1, 2, 3

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 24  # elements drawn per numpy pass (bounds host temporaries to a few hundred MB)


def _mix_np(x: np.ndarray) -> np.ndarray:
    x = x.copy()
    x ^= x >> np.uint64(30)
    x *= _M1
    x ^= x >> np.uint64(27)
    x *= _M2
    x ^= x >> np.uint64(31)
    return x


def _stream_base(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        return _mix_np(np.array([16 * int(seed) + int(stream)], dtype=np.uint64))[0]


def _uniform_np(seed: int, stream: int, counters: np.ndarray) -> np.ndarray:
    base = _stream_base(seed, stream)
    with np.errstate(over="ignore"):
        w = _mix_np(base + (counters.astype(np.uint64) + np.uint64(1)) * _GOLDEN)
    return (w >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _normal_f64_at(seed: int, stream: int, flat: np.ndarray) -> np.ndarray:
    flat = np.asarray(flat, dtype=np.int64)
    pair = flat >> 1
    u1 = _uniform_np(seed, stream, 2 * pair)
    u2 = _uniform_np(seed, stream, 2 * pair + 1)
    r = np.sqrt(-2.0 * np.log(1.0 - u1))
    theta = 2.0 * math.pi * u2
    return np.where((flat & 1) == 0, r * np.cos(theta), r * np.sin(theta))


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE) bit patterns as uint16 (finite inputs)."""
    b = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16_at(seed: int, stream: int, flat: np.ndarray) -> np.ndarray:
    """bf16 bits of the N(0,1) draws at the given flat element indices of a stream."""
    return f64_to_bf16_bits(_normal_f64_at(seed, stream, flat))


def normal_bf16(seed: int, stream: int, shape) -> np.ndarray:
    """A whole tensor of bf16 bits (uint16), element i of the row-major flattening = draw i."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = normal_bf16_at(seed, stream, np.arange(lo, hi, dtype=np.int64))
    return out.reshape(shape)


def kv_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """Per-sequence decode KV lengths, uniform on the integers [lo, hi]."""
    u = _uniform_np(seed, STREAM_LENS, np.arange(batch, dtype=np.int64))
    return (lo + np.floor(u * (hi - lo + 1))).astype(np.int32)


# ----------------------------------------------------------------------------------------------
# device-side drawing (torch, same recipe, for tensors too large to draw on the host)
# ----------------------------------------------------------------------------------------------

def _i64(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


def _mix_torch(x):
    import torch

    def lsr(v, k):
        return (v >> k) & ((1 << (64 - k)) - 1)

    x = x ^ lsr(x, 30)
    x = x * _i64(0xBF58476D1CE4E5B9)
    x = x ^ lsr(x, 27)
    x = x * _i64(0x94D049BB133111EB)
    x = x ^ lsr(x, 31)
    return x


def normal_bf16_torch(seed: int, stream: int, shape, device="cuda", chunk: int = 1 << 26):
    """The same draws as :func:`normal_bf16`, made with torch ops on ``device`` (bf16 tensor)."""
    import torch

    n = int(np.prod(shape))
    base = _i64(int(_stream_base(seed, stream)))
    gold = _i64(0x9E3779B97F4A7C15)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        pair = torch.arange(lo >> 1, (hi + 1) >> 1, dtype=torch.int64, device=device)
        c1 = 2 * pair
        w1 = _mix_torch(base + (c1 + 1) * gold)
        w2 = _mix_torch(base + (c1 + 2) * gold)
        u1 = ((w1 >> 11) & ((1 << 53) - 1)).to(torch.float64) * (2.0 ** -53)
        u2 = ((w2 >> 11) & ((1 << 53) - 1)).to(torch.float64) * (2.0 ** -53)
        r = torch.sqrt(-2.0 * torch.log(1.0 - u1))
        th = 2.0 * math.pi * u2
        z = torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).reshape(-1)
        z = z[(lo & 1):(lo & 1) + (hi - lo)]
        out[lo:hi] = z.to(torch.float32).to(torch.bfloat16)
    return out.reshape(shape)


# ----------------------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class Prefill:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    d: int
    causal: bool

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """Attention forward FLOPs, 4*B*Hq*Nq*Nkv*d, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nkv * self.d
        return f / 2 if self.causal else f

    def draw(self):
        """Host bf16 bits for q [B,Nq,Hq,d], k and v [B,Nkv,Hkv,d]."""
        return (normal_bf16(self.seed, STREAM_Q, (self.B, self.Nq, self.Hq, self.d)),
                normal_bf16(self.seed, STREAM_K, (self.B, self.Nkv, self.Hkv, self.d)),
                normal_bf16(self.seed, STREAM_V, (self.B, self.Nkv, self.Hkv, self.d)))


@dataclass(frozen=True)
class Decode:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    len_lo: int
    len_hi: int
    Nkv_cap: int = field(default=0)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def cap(self) -> int:
        return self.Nkv_cap or self.len_hi

    def lengths(self) -> np.ndarray:
        return kv_lengths(self.seed, self.B, self.len_lo, self.len_hi)

    def algorithmic_bytes(self) -> int:
        """K and V rows actually attended plus q, O and LSE."""
        toks = int(self.lengths().astype(np.int64).sum())
        kv = toks * self.Hkv * self.d * 2 * 2
        return kv + self.B * self.Hq * self.d * 2 * 2 + self.B * self.Hq * 4


TINY = Prefill("tiny non-causal B1 H2 N256 d64", 1001, 1, 2, 2, 256, 256, 64, False)
CAUSAL_2K = Prefill("causal prefill B4 H16 N2048 d128", 1002, 4, 16, 16, 2048, 2048, 128, True)
LONG_8K = Prefill("long non-causal B2 H16 N8192 d128", 1003, 2, 16, 16, 8192, 8192, 128, False)
LONG_8K_CAUSAL = Prefill("long causal B2 H16 N8192 d128", 1003, 2, 16, 16, 8192, 8192, 128, True)
LONG_8K_GQA = Prefill("long GQA non-causal B2 Hq32 Hkv8 N8192 d128", 1003, 2, 32, 8, 8192, 8192, 128, False)
LONG_8K_GQA_CAUSAL = Prefill("long GQA causal B2 Hq32 Hkv8 N8192 d128", 1003, 2, 32, 8, 8192, 8192, 128, True)
SWEEP = tuple(Prefill(f"head-dim sweep B4 H16 N4096 d{d}", 1004, 4, 16, 16, 4096, 4096, d, False)
              for d in (32, 64, 128, 256))
DECODE = Decode("split-KV decode B8 Hq32 Hkv8 d128 L~U[1024,131072]", 1005, 8, 32, 8, 128, 1024, 131072)

PREFILL_WORKLOADS = (TINY, CAUSAL_2K, LONG_8K, LONG_8K_CAUSAL, LONG_8K_GQA, LONG_8K_GQA_CAUSAL) + SWEEP
