"""The FMA-pipe exponential (Cody-Waite range reduction + degree-3 polynomial) that the prefill
kernels can use for part of their exponentials, checked on the GPU against the exact 2^x."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

FIT_MAX_REL_ERR = 7.5e-5  # of the polynomial on [-1/2, 1/2] (fit_exp2_poly.py)


def test_relative_error_over_the_range_softmax_uses(lib):
    import torch

    rng = np.random.default_rng(5150)
    # every argument the softmax can produce lies in [-125, 8] (P <= 2^tau, tau = 8); also cover the
    # rest of the valid range (x < 127.5, where 2^round(x) is still a normal float) and the
    # half-integer boundaries where the range reduction switches n
    grid = np.concatenate([
        np.linspace(-125.0, 127.0, 1_000_001),
        rng.uniform(-125.0, 8.0, 1_000_000),
        np.arange(-125, 127) + 0.5, np.arange(-124, 128) - 0.5, np.arange(-125, 128).astype(np.float64),
    ]).astype(np.float32)
    grid = grid[grid < 127.5]
    x = torch.from_numpy(grid).cuda()
    y = lib.attn_selftest_exp2_poly(x)
    torch.cuda.synchronize()
    exact = np.exp2(grid.astype(np.float64))
    rel = np.abs(y.cpu().numpy().astype(np.float64) / exact - 1.0)
    # the fit's error plus a few fp32 roundings of the Horner evaluation
    assert rel.max() <= FIT_MAX_REL_ERR + 1e-6, float(rel.max())


def test_arguments_below_the_clamp(lib):
    import torch

    x = torch.tensor([-126.0, -200.0, -1.0e30, float("-inf")], dtype=torch.float32, device="cuda")
    y = lib.attn_selftest_exp2_poly(x).cpu().numpy().astype(np.float64)
    # clamped to -125: 2^-125 times the polynomial at 0 (within the fit's error of 1)
    assert np.all(np.abs(y / 2.0 ** -125 - 1.0) <= FIT_MAX_REL_ERR + 1e-6)


def test_odd_length(lib):
    import torch

    x = torch.tensor([0.0, 1.0, 2.5], dtype=torch.float32, device="cuda")
    y = lib.attn_selftest_exp2_poly(x).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(y / np.exp2([0.0, 1.0, 2.5]) - 1.0) <= FIT_MAX_REL_ERR + 1e-6)
