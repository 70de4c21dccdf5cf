"""fp8_mm_splitk_static: the split-K GEMM on the library's own scratch.

The call takes no workspace and allocates nothing: the scratch is a static
device array of the library. On the GPU it must give exactly (bit for bit)
what fp8_mm_ws gives with a caller workspace and the same split, agree with
the oracle within the GEMM tolerance, stay reusable call after call (its
counters return to zero) and leave the device's free memory unchanged.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2, NN, NT, TN
import workloads as W

A = 0x7F0000000000
S = 0x7F0000100000


def test_static_split_validates_before_touching_the_device():
    import fp8_delayed_scaling_quantize_b200 as fp8
    for split_k in (-1, 0, 1, 5):
        st = fp8.raw_status("fp8_mm_splitk_static", A, 0, A, 0, S, S, 0, 2048, 1024, 4096, 1, 0, 0, 0, None, None,
                            0, A, split_k, None)
        assert st == fp8.FP8_ERR_INVALID_ARG
    # more partial-tile bytes than the 32 MiB scratch holds
    assert fp8.fp8_mm_workspace_size(4096, 2048, 8192, 1, fp8.FP8_NT, 4) > (32 << 20)
    st = fp8.raw_status("fp8_mm_splitk_static", A, 0, A, 0, S, S, 0, 4096, 2048, 8192, 1, 0, 0, 0, None, None,
                        0, A, 4, None)
    assert st == fp8.FP8_ERR_UNSUPPORTED


CASES = [
    # (layout, M, N, K, split_k, fa, fb, bias_kind)
    (NT, 2048, 1024, 4096, 2, E4M3, E4M3, 0),
    (NN, 2048, 1024, 3072, 3, E5M2, E4M3, 1),
    (TN, 1024, 1024, 2048, 4, E5M2, E4M3, 0),
    (NT, 1, 4096, 4096, 4, E4M3, E4M3, 1),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:5])))
def test_static_split_equals_the_workspace_split(case):
    import gpu_util as g
    import fp8_delayed_scaling_quantize_b200 as fp8
    layout, M, N, K, split_k, fa, fb, bias_kind = case
    a8 = W.fp8_codes((M * K,), fa, 700 + K)
    b8 = W.fp8_codes((N * K,), fb, 701 + K)
    bias = bias_dev = None
    if bias_kind:
        bb = W.bf16_normal((N,), 0.1, 702 + K)
        bias_dev = bb.cuda()
        bias = bb.view(torch.int16).numpy().view(np.uint16)
    ad, bd = a8.cuda(), b8.cuda()
    sa = torch.tensor([0.5], device="cuda")
    sb = torch.tensor([1.25], device="cuda")
    args = (ad, fa, bd, fb, sa, sb, layout, M, N, K, 1, M * K, N * K, M * N, bias_dev, None, 0)
    ws = g.workspace(fp8.fp8_mm_workspace_size(M, N, K, 1, layout, split_k))
    want = torch.empty(M * N, dtype=torch.bfloat16, device="cuda")
    fp8.fp8_mm_ws(*args, want, ws, split_k)
    got = torch.full((M * N,), float("nan"), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):  # reusable: the counters go back to zero every call
        got.fill_(float("nan"))
        fp8.fp8_mm_splitk_static(*args, got, split_k)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert torch.cuda.mem_get_info()[0] == free0
    y, s = oracle.mm(a8.numpy(), fa, b8.numpy(), fb, 0.5, 1.25, layout, M, N, K, bias=bias)
    g.assert_within(got.float().cpu().numpy().reshape(M, N), y, oracle.tolerance(y, s), f"static {case}")
    assert fp8.fp8_last_device_error() == fp8.FP8_OK
