"""Prefill with part of its exponentials on the FMA pipe (Cody-Waite range reduction and a
polynomial; the "emulated exponentials" the FlashAttention generation comparison record lists for
FA-4), against the fp64 oracle.

The product library evaluates every exponential on the exp unit: the emulated split was measured
slower on B200 at every head dim. The same sources built with the split switched on (half of the
columns of each tile at d = 32 and 64, a quarter at d = 128 and 256, in tiles without masked keys)
are the test variant ``libattn_b200_emu.so``; it is called here through the same C ABI.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import synth
from parity import assert_parity, bf16_tensor_to_f64, draw_prefill, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def emu():
    from exact_io_aware_41_b200 import SIGNATURES, build

    path = build.build_emu_variant()
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _run(emu, lib, seed, B, Hq, Hkv, Nq, Nkv, d, causal, scale=None):
    import torch

    qb, kb, vb = draw_prefill(seed, B, Hq, Hkv, Nq, Nkv, d)
    q, k, v = to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb)
    sc = scale if scale is not None else 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = emu.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nkv,
                        d, sc, int(causal), st)
    assert code == 0
    torch.cuda.synchronize()
    assert emu.attn_get_last_error() == 0
    O_ref, L_ref = oracle.attention(synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(kb),
                                    synth.bf16_bits_to_f64(vb), sc, causal)
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_ref,
                  L_ref.transpose(0, 2, 1), f"emulated exp2 B{B} Hq{Hq} Hkv{Hkv} Nq{Nq} Nkv{Nkv} d{d} causal={causal}")
    # the emulated columns really ran: the product library (exp unit only) rounds some P entries
    # differently, so the two outputs are close but not bit-identical
    o_ref, _ = lib.attn_fwd(q, k, v, scale=sc, causal=causal)
    torch.cuda.synchronize()
    return bool((o != o_ref).any())


@pytest.mark.parametrize("d", [32, 64, 128, 256])
def test_emulated_exponentials_match_the_oracle(emu, lib, d):
    # several full key tiles (emulated) and a ragged tail (masked: exp unit), causal and not, GQA,
    # a large scale so the running max moves and O is rescaled
    differs = _run(emu, lib, 6000 + d, 2, 4, 2, 700, 700, d, False)
    differs |= _run(emu, lib, 6100 + d, 1, 4, 1, 650, 650, d, True)
    differs |= _run(emu, lib, 6200 + d, 1, 2, 2, 512, 512, d, False, scale=1.5)
    assert differs, "the emulated variant gave bit-identical results: its polynomial path did not run"
