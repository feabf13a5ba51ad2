"""The decode entry point that allocates nothing (attn_decode_splitkv_static).

Some callers cannot hand the library a workspace: a plugin inside a host runtime that owns all
device memory, or a serving loop that must not call cudaMalloc. For them the library keeps the
split partials in one fixed device array. These checks call that entry point through the C ABI and
compare it with the workspace entry point and with the fp64 oracle on the same inputs, twice in a
row with different inputs (the array keeps the previous call's partials, which must not leak into
the next result). The file is named so pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import synth
from parity import assert_parity, bf16_tensor_to_f64, device_bits

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Hq, Hkv, d, cap):
    dev = "cuda"
    q = synth.normal_bf16_torch(seed, synth.STREAM_Q, (B, Hq, d), dev)
    kc = synth.normal_bf16_torch(seed, synth.STREAM_K, (B, cap, Hkv, d), dev)
    vc = synth.normal_bf16_torch(seed, synth.STREAM_V, (B, cap, Hkv, d), dev)
    return q, kc, vc


def test_static_scratch_decode_matches_workspace_decode_twice(lib):
    import torch

    B, Hq, Hkv, d, cap = 4, 32, 8, 128, 20000
    # first call: long sequences fill many splits; second call: short ones leave stale partials behind
    for call, (seed, lens) in enumerate([(61, [20000, 19999, 12345, 7000]), (62, [1, 700, 0, 4097])]):
        q, kc, vc = _inputs(seed, B, Hq, Hkv, d, cap)
        lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
        o_ref, l_ref = lib.attn_decode_splitkv(q, kc, vc, lens_t, chunk=128)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        stream = torch.cuda.current_stream()
        code = lib.lib_handle().attn_decode_splitkv_static(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), lens_t.data_ptr(),
                                                   cap, o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, d,
                                                   1.0 / math.sqrt(d), 128, ctypes.c_void_p(stream.cuda_stream))
        assert code == lib.ATTN_OK, lib.status_string(code)
        torch.cuda.synchronize()
        assert lib.attn_get_last_error() == lib.ATTN_OK
        assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64),
                      bf16_tensor_to_f64(o_ref), l_ref.cpu().numpy().astype(np.float64), f"static decode call {call}")
        # and against the fp64 oracle on the exact inputs
        O_or, L_or = oracle.decode(synth.bf16_bits_to_f64(device_bits(q)), synth.bf16_bits_to_f64(device_bits(kc)),
                                   synth.bf16_bits_to_f64(device_bits(vc)), np.array(lens), 1.0 / math.sqrt(d))
        assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), O_or, L_or,
                      f"static decode call {call} vs oracle")


def test_static_scratch_decode_binding_and_size_limit(lib):
    import torch

    q, kc, vc = _inputs(63, 2, 8, 2, 64, 300)
    lens_t = torch.tensor([300, 5], dtype=torch.int32, device="cuda")
    o1, l1 = lib.attn_decode_splitkv_static(q, kc, vc, lens_t, chunk=64)
    o2, l2 = lib.attn_decode_splitkv(q, kc, vc, lens_t, chunk=64)
    torch.cuda.synchronize()
    assert_parity(bf16_tensor_to_f64(o1), l1.cpu().numpy().astype(np.float64), bf16_tensor_to_f64(o2),
                  l2.cpu().numpy().astype(np.float64), "static decode via binding")
    # partials larger than the fixed array are refused before anything is launched
    need = lib.attn_decode_workspace_bytes(64, 64, 8, 256, 1 << 20, 64)
    assert need > lib.DECODE_STATIC_SCRATCH_BYTES
    code = lib.lib_handle().attn_decode_splitkv_static(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), lens_t.data_ptr(),
                                               1 << 20, o1.data_ptr(), l1.data_ptr(), 64, 64, 8, 256, 0.0625, 64,
                                               None)
    assert code == lib.ATTN_ERR_WORKSPACE
