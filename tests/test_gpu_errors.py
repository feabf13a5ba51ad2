"""Bounded waits and error reporting on the GPU, without faulting or hanging it."""
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports(lib):
    import torch

    assert lib.attn_get_last_error() == lib.ATTN_OK
    lib.attn_selftest_bounded_wait(2000)  # a 2 ms wait on a barrier nothing completes
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_ERR_TIMEOUT
    assert lib.attn_get_last_error() == lib.ATTN_OK  # reading clears the word
    # the context is still usable
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_cluster_pair_waits_complete_or_time_out(lib):
    import torch

    assert lib.attn_get_last_error() == lib.ATTN_OK
    lib.attn_selftest_pair_wait(2000000, True)  # each CTA arrives on the other's barrier: no timeout
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_OK
    lib.attn_selftest_pair_wait(2000, False)  # nothing arrives: both 2 ms waits run out
    torch.cuda.synchronize()
    assert lib.attn_get_last_error() == lib.ATTN_ERR_TIMEOUT
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_argument_errors_raise(lib):
    import torch

    q = torch.zeros((1, 16, 2, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError) as e:
        lib.attn_fwd(q, q, q)
    assert e.value.code == lib.ATTN_ERR_UNSUPPORTED
    q = torch.zeros((1, 16, 3, 64), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError) as e:
        lib.attn_fwd(q, k, k)
    assert e.value.code == lib.ATTN_ERR_INVALID_ARG


def test_kernel_is_native_sm100(lib):
    import torch

    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0)
