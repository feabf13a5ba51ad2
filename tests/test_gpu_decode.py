"""Split-KV decode parity: CUDA path (split kernel + combine, through the C ABI) against the fp64
oracle, on small shapes and on every row of the full decode workload."""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import assert_parity, bf16_tensor_to_f64, device_bits, to_torch_bf16

pytestmark = pytest.mark.gpu


def _decode_small(lib, seed, B, Hq, Hkv, d, cap, lens, chunk):
    import torch

    qb = synth.normal_bf16(seed, synth.STREAM_Q, (B, Hq, d))
    kb = synth.normal_bf16(seed, synth.STREAM_K, (B, cap, Hkv, d))
    vb = synth.normal_bf16(seed, synth.STREAM_V, (B, cap, Hkv, d))
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    sc = 1.0 / math.sqrt(d)
    o, lse = lib.attn_decode_splitkv(to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb), lens_t, scale=sc,
                                     chunk=chunk)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    O_ref, L_ref = oracle.decode(synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(kb),
                                 synth.bf16_bits_to_f64(vb), np.array(lens), sc)
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), O_ref, L_ref,
                  f"decode B{B} Hq{Hq} Hkv{Hkv} d{d} cap{cap} chunk{chunk}")


@pytest.mark.parametrize("d", [32, 64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_every_head_dim_and_group(lib, d, G):
    # lengths: full cache, one token, empty, and ragged values across several 64-token splits
    _decode_small(lib, 5000 + d + G, 5, 2 * G, 2, d, 700, [700, 1, 0, 333, 65], 64)


@pytest.mark.parametrize("chunk", [0, 64, 128, 512])
def test_decode_chunk_choice_does_not_change_the_result(lib, chunk):
    _decode_small(lib, 5100, 3, 32, 8, 128, 1500, [1500, 1023, 777], chunk)


def test_decode_length_out_of_range_is_clamped_and_flagged(lib):
    import torch

    B, Hq, Hkv, d, cap = 2, 8, 2, 128, 256
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, cap, Hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.ones((B, cap, Hkv, d), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([cap + 50, 10], dtype=torch.int32, device="cuda")
    o, lse = lib.attn_decode_splitkv(q, kc, vc, lens, chunk=64)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_ERR_INVALID_ARG
    # equal scores: O = mean of V rows = 1, LSE = ln(number of keys)
    assert torch.all(o.float() == 1.0)
    np.testing.assert_allclose(lse[0].cpu().numpy(), math.log(cap), atol=1e-5)
    np.testing.assert_allclose(lse[1].cpu().numpy(), math.log(10), atol=1e-5)
    assert lib.attn_get_last_error() == lib.ATTN_OK


def test_combine_entry_point_matches_the_merge_identity(lib):
    import torch

    rng = np.random.default_rng(7)
    rows, n_splits, d = 37, 9, 128
    po = rng.standard_normal((rows, n_splits, d)).astype(np.float32)
    pl = (rng.standard_normal((rows, n_splits)) * 4).astype(np.float32)
    pl[rng.random((rows, n_splits)) < 0.3] = -np.inf
    pl[5, :] = -np.inf
    o, lse = lib.attn_decode_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda())
    torch.cuda.synchronize()
    O_ref = np.zeros((rows, d))
    L_ref = np.zeros(rows)
    for r in range(rows):
        parts = [(po[r, s].astype(np.float64), float(pl[r, s])) for s in range(n_splits)]
        O_ref[r], L_ref[r] = oracle.merge_partials(parts)
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), O_ref, L_ref, "combine")


def test_full_decode_workload_every_row(lib):
    """The full decode workload (eight sequences of 1k-128k tokens, GQA 32/8), all 256 (b, hq) rows
    against oracle.decode, fed the exact bits the kernels read (copied back one sequence at a time)."""
    import torch

    w = synth.DECODE
    lens = w.lengths()
    cap = w.cap
    shape = (w.B, cap, w.Hkv, w.d)
    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Hq, w.d), "cuda")
    kc = synth.normal_bf16_torch(w.seed, synth.STREAM_K, shape, "cuda")
    vc = synth.normal_bf16_torch(w.seed, synth.STREAM_V, shape, "cuda")
    lens_t = torch.from_numpy(lens).cuda()
    o, lse = lib.attn_decode_splitkv(q, kc, vc, lens_t, scale=w.scale)
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    qh = synth.bf16_bits_to_f64(device_bits(q))
    O_ref = np.zeros((w.B, w.Hq, w.d))
    L_ref = np.zeros((w.B, w.Hq))
    for b in range(w.B):
        L = int(lens[b])
        kb = synth.bf16_bits_to_f64(device_bits(kc[b:b + 1, :L]))
        vb = synth.bf16_bits_to_f64(device_bits(vc[b:b + 1, :L]))
        O_ref[b:b + 1], L_ref[b:b + 1] = oracle.decode(qh[b:b + 1], kb, vb, np.array([L]), w.scale)
        del kb, vb
    assert_parity(bf16_tensor_to_f64(o), lse.cpu().numpy().astype(np.float64), O_ref, L_ref,
                  "full decode workload, all rows")


def test_refused_sizes_launch_nothing(lib):
    """More splits per row than the combine kernel takes: UNSUPPORTED, and the outputs keep their
    previous contents (nothing was launched). The buffers are sized for the requested shape, so even
    a launch would have stayed in bounds."""
    import ctypes

    import torch

    B, Hq, Hkv, d, chunk = 1, 1, 1, 32, 64
    cap = chunk * 25601
    kc = torch.zeros((B, cap, Hkv, d), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    o = torch.full((B, Hq, d), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq), 5.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.attn_decode_workspace_bytes(B, Hq, Hkv, d, cap, chunk), dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    h = lib.lib_handle()
    assert h.attn_decode_splitkv(q.data_ptr(), kc.data_ptr(), kc.data_ptr(), lens.data_ptr(), cap, o.data_ptr(),
                                 lse.data_ptr(), B, Hq, Hkv, d, 0.125, chunk, ws.data_ptr(), ws.numel(),
                                 st) == lib.ATTN_ERR_UNSUPPORTED
    assert h.attn_decode_splitkv_static(q.data_ptr(), kc.data_ptr(), kc.data_ptr(), lens.data_ptr(), cap,
                                        o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, d, 0.125, chunk,
                                        st) == lib.ATTN_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(o.float() == 3.0) and torch.all(lse == 5.0)
    assert lib.attn_get_last_error() == lib.ATTN_OK
