"""fp8_mm_splitk_static: the split-K GEMM for callers that cannot allocate.

Some callers cannot call cudaMalloc (a memory pool that owns every device
byte, a callback run inside another framework's step, a real-time caller
that may not allocate after start-up), so they cannot hand fp8_mm_ws a
workspace. This entry point takes none and allocates nothing: its scratch is
a static device array of the library. On the GPU it must give exactly (bit
for bit) what fp8_mm_ws gives with a caller workspace and the same split,
agree with the oracle within the GEMM tolerance, give the same result on
consecutive calls (each call clears the array's counters) and leave the
device's free memory unchanged.

This file is collected last, so that a run stopping at its first failure has
already run every other test; it also passes alone in a fresh process.
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
# batches, one B broadcast to all of them (batch stride 0): more tiles, so the
# counters and partial tiles spread further through the fixed array
BATCHED = [(NT, 512, 768, 1024, 2, E4M3, E4M3, 1, 4), (NN, 384, 512, 1536, 3, E5M2, E4M3, 0, 3)]


def _run(case, batch=1, bcast_b=False):
    import gpu_util as g
    import fp8_delayed_scaling_quantize_b200 as fp8
    layout, M, N, K, split_k, fa, fb, bias_kind = case
    stride_a, stride_b, stride_c = M * K, 0 if bcast_b else N * K, M * N
    a8 = W.fp8_codes((batch * M * K,), fa, 700 + K + batch)
    b8 = W.fp8_codes(((1 if bcast_b else batch) * N * K,), fb, 701 + K + batch)
    bias = bias_dev = None
    if bias_kind:
        bb = W.bf16_normal((N,), 0.1, 702 + K)
        bias_dev = bb.cuda()
        bias = bb.view(torch.int16).numpy().view(np.uint16)
    ad, bd = a8.cuda(), b8.cuda()
    sa = torch.tensor([0.5], device="cuda")
    sb = torch.tensor([1.25], device="cuda")
    args = (ad, fa, bd, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias_dev, None, 0)
    need = fp8.fp8_mm_workspace_size(M, N, K, batch, layout, split_k)
    assert 0 < need <= (32 << 20)
    ws = g.workspace(need)
    want = torch.empty(batch * M * N, dtype=torch.bfloat16, device="cuda")
    # the caller-workspace call runs first; it also loads the GEMM module on
    # this device, so the free memory sampled below already counts the
    # library's static scratch
    fp8.fp8_mm_ws(*args, want, ws, split_k)
    got = torch.full((batch * M * N,), float("nan"), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):  # consecutive calls share the array and agree
        got.fill_(float("nan"))
        fp8.fp8_mm_splitk_static(*args, got, split_k)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    assert torch.cuda.mem_get_info()[0] == free0  # nothing allocated
    y, s = oracle.mm(a8.numpy(), fa, b8.numpy(), fb, 0.5, 1.25, layout, M, N, K, batch=batch, stride_a=stride_a,
                     stride_b=stride_b, bias=bias)
    g.assert_within(got.float().cpu().numpy().reshape(batch, M, N), y, oracle.tolerance(y, s), f"static {case}")
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:5])))
def test_static_split_equals_the_workspace_split(case):
    _run(case)


@pytest.mark.gpu
@pytest.mark.parametrize("case", BATCHED, ids=lambda c: "x".join(map(str, c[:5])) + f"b{c[8]}")
def test_static_split_batched_broadcast_b(case):
    _run(case[:8], batch=case[8], bcast_b=True)
