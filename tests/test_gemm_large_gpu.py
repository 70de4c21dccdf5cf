"""GPU parity of fp8_mm at the size limits: an operand of 2^31 bytes and an
output of more than 2^31 elements.

The operands repeat a seeded block along M (and N), so every output element
equals, bit for bit, the element at the same position of the first block
(each output is computed alone, with the same k-block order in every tile).
That property is checked over the whole output on the device; the first
block is held to the oracle's bar,
|gpu - oracle| <= ulp_bf16(oracle) + 2^-16 * sum_k |a b| / (sa sb).
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2, NN, NT
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gpu_util
    return gpu_util


def _scales():
    return (torch.tensor([0.75], dtype=torch.float32, device="cuda"),
            torch.tensor([1.5], dtype=torch.float32, device="cuda"))


def test_operand_of_2_to_31_bytes(g):
    """NT with A = 131072 x 16384 codes (2^31 bytes, byte offsets past
    2^31), N = 256: SM-pair tiles over 512 rounds of rows."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    R, M, N, K = 1024, 131072, 256, 16384
    block = W.fp8_codes((R, K), E4M3, 2100)
    b8 = W.fp8_codes((N * K,), E5M2, 2101)
    a = block.cuda().repeat(M // R, 1).reshape(-1)
    assert a.numel() == 1 << 31
    sa, sb = _scales()
    out = g.mm(a, E4M3, b8.cuda(), E5M2, sa, sb, NT, M, N, K)
    c = out.view(M // R, R, N).view(torch.int16)
    for r0 in range(0, M // R, 32):
        assert torch.equal(c[r0:r0 + 32], c[0:1].expand(min(32, M // R - r0), R, N)), f"row blocks {r0}.."
    y, s = oracle.mm(block.numpy().reshape(-1), E4M3, b8.numpy(), E5M2, 0.75, 1.5, NT, R, N, K)
    g.assert_within(out[:R * N].float().cpu().numpy().reshape(R, N), y, oracle.tolerance(y, s),
                    "NT 131072x256x16384, first rows")
    del a, out, c
    torch.cuda.empty_cache()
    assert fp8.fp8_last_device_error() == fp8.FP8_OK


@pytest.mark.parametrize("layout", [NT, NN], ids=["NT", "NN"])
def test_output_past_2_to_31_elements(g, layout):
    """M = N = 49152, K = 64 (one k-block, its tail zero-filled): 2.4 G
    outputs, 4.8 GB of bf16."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    R, M, N, K = 1024, 49152, 49152, 64
    ablock = W.fp8_codes((R, K), E4M3, 2200 + layout)
    bblock = W.fp8_codes((R, K) if layout == NT else (K, R), E4M3, 2300 + layout)
    a = ablock.cuda().repeat(M // R, 1).reshape(-1)
    b = (bblock.cuda().repeat(N // R, 1) if layout == NT else bblock.cuda().repeat(1, N // R)).reshape(-1)
    sa, sb = _scales()
    out = torch.empty(M * N, dtype=torch.bfloat16, device="cuda")
    g.mm(a, E4M3, b, E4M3, sa, sb, layout, M, N, K, out=out)
    assert out.numel() > 1 << 31
    c = out.view(M // R, R, N // R, R).view(torch.int16)
    first = c[0:1, :, 0:1, :]
    for r0 in range(M // R):
        assert torch.equal(c[r0:r0 + 1], first.expand(1, R, N // R, R)), f"row block {r0}"
    y, s = oracle.mm(ablock.numpy().reshape(-1), E4M3, bblock.numpy().reshape(-1), E4M3, 0.75, 1.5, layout, R, R, K)
    got = out.view(M, N)[:R, :R].float().cpu().numpy()
    g.assert_within(got, y, oracle.tolerance(y, s), f"{'NT' if layout == NT else 'NN'} {M}x{N}x{K}, first block")
    del a, b, out, c, first
    torch.cuda.empty_cache()
    assert fp8.fp8_last_device_error() == fp8.FP8_OK
