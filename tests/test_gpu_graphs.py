"""The kernels inside CUDA graphs: prefill (two-tile and CTA-pair kernels, causal and not) and split-KV
decode are captured once and replayed; every replay must reproduce the eager call bit for bit (each
output element is produced by one thread in a fixed order, whatever order the units run in), and the
eager call is itself checked against the oracle."""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import assert_parity, bf16_tensor_to_f64, draw_prefill, to_torch_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,causal", [(128, True), (128, False), (256, True), (64, True)])
def test_prefill_graph_replays_match_eager(lib, d, causal):
    import torch

    B, Hq, Hkv, N = 2, 4, 2, 700
    qb, kb, vb = draw_prefill(5000 + d + int(causal), B, Hq, Hkv, N, N, d)
    q, k, v = to_torch_bf16(qb), to_torch_bf16(kb), to_torch_bf16(vb)
    sc = 1.0 / math.sqrt(d)
    o_ref, l_ref = lib.attn_fwd(q, k, v, scale=sc, causal=causal)  # eager; also the warm-up
    torch.cuda.synchronize()
    O_or, L_or = oracle.attention(synth.bf16_bits_to_f64(qb), synth.bf16_bits_to_f64(kb),
                                  synth.bf16_bits_to_f64(vb), sc, causal)
    assert_parity(bf16_tensor_to_f64(o_ref), l_ref.cpu().numpy().astype(np.float64).transpose(0, 2, 1), O_or,
                  L_or.transpose(0, 2, 1), f"eager d{d} causal={causal}")

    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            lib.attn_fwd(q, k, v, scale=sc, causal=causal, out=o, lse=lse)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        o.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    assert lib.attn_get_last_error() == lib.ATTN_OK
    del g


def test_decode_graph_replays_match_eager(lib):
    import torch

    B, Hq, Hkv, d, cap = 3, 8, 2, 128, 5000
    rng = np.random.default_rng(5100)
    lens = np.array([1, 4097, 2500], dtype=np.int32)
    q = torch.randn((B, Hq, d), dtype=torch.bfloat16, device="cuda", generator=None)
    kc = torch.randn((B, cap, Hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.randn((B, cap, Hkv, d), dtype=torch.bfloat16, device="cuda")
    kv_lens = torch.from_numpy(lens).cuda()
    ws = torch.empty(lib.attn_decode_workspace_bytes(B, Hq, Hkv, d, cap, 512), dtype=torch.uint8, device="cuda")
    o_ref, l_ref = lib.attn_decode_splitkv(q, kc, vc, kv_lens, chunk=512, workspace=ws)
    torch.cuda.synchronize()
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            lib.attn_decode_splitkv(q, kc, vc, kv_lens, chunk=512, workspace=ws, out=o, lse=lse)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    # the eager result against the oracle, row by row
    qf, kf, vf = (t.float().cpu().numpy().astype(np.float64) for t in (q, kc, vc))
    og = o_ref.float().cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        O1, _ = oracle.attention(qf[b][None, None], kf[b][None, :L], vf[b][None, :L], 1.0 / math.sqrt(d), False)
        np.testing.assert_allclose(og[b], O1[0, 0], atol=2e-2)
    del g, rng
