"""Failure detection without a GPU fault: a bounded device wait that runs out
(a barrier nothing arrives at) is reported through fp8_last_device_error, the
error word is cleared by reading it, and the context stays usable."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_cleanly():
    import fp8_delayed_scaling_quantize_b200 as fp8
    import gpu_util as g
    fp8.fp8_last_device_error()                     # start clean
    fp8.fp8_selftest_wait_timeout(2000)             # 2 ms limit
    with pytest.raises(fp8.Fp8Error) as e:
        fp8.fp8_last_device_error()
    assert e.value.status == fp8.FP8_ERR_DEVICE_TIMEOUT
    fp8.fp8_last_device_error()                     # reading cleared it
    # the context still computes correctly
    a8 = W.fp8_codes((128 * 128,), 0, 1)
    b8 = W.fp8_codes((128 * 128,), 0, 2)
    s = torch.ones(1, device="cuda")
    out = g.mm(a8.cuda(), 0, b8.cuda(), 0, s, s, fp8.FP8_NT, 128, 128, 128)
    y, sums = oracle.mm(a8.numpy(), 0, b8.numpy(), 0, 1.0, 1.0, oracle.NT, 128, 128, 128)
    got = out.float().cpu().numpy().reshape(1, 128, 128)
    assert np.all(np.abs(got - y) <= oracle.tolerance(y, sums))
    # a split-K call on the library's own scratch right after the timeout
    # gives what the caller-workspace call gives, bit for bit
    M, N, K = 2048, 1024, 4096
    a8 = W.fp8_codes((M * K,), 0, 3).cuda()
    b8 = W.fp8_codes((N * K,), 0, 4).cuda()
    args = (a8, 0, b8, 0, s, s, fp8.FP8_NT, M, N, K, 1, 0, 0, 0, None, None, 0)
    want = torch.empty(M * N, dtype=torch.bfloat16, device="cuda")
    fp8.fp8_mm_ws(*args, want, g.workspace(fp8.fp8_mm_workspace_size(M, N, K, 1, fp8.FP8_NT, 2)), 2)
    got = torch.empty_like(want)
    fp8.fp8_mm_splitk_static(*args, got, 2)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    fp8.fp8_last_device_error()


def test_selftest_argument_validation():
    import fp8_delayed_scaling_quantize_b200 as fp8
    assert fp8.raw_status("fp8_selftest_wait_timeout", 0, None) == fp8.FP8_ERR_INVALID_ARG
    assert fp8.raw_status("fp8_selftest_wait_timeout", 2_000_000, None) == fp8.FP8_ERR_INVALID_ARG
