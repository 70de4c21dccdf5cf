"""Pins for the oracle's FP8 GEMM (CPU only).

Pinned against exact rational brute force on tiny shapes (operands decoded
by torch's float8 types, an independent library; the bf16 rounding by an
exhaustive nearest search), closed forms (identity operands, a single
non-zero k) and the tolerance's ulp at known points.
"""

import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2, NN, NT, TN
from workloads import fp8_codes
import workloads as W

TORCH_FP8 = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def _dec(codes, fmt):
    """Exact decode through torch's float8 dtype."""
    t = torch.as_tensor(np.asarray(codes, np.uint8)).view(TORCH_FP8[fmt])
    return [Fraction(v) for v in t.to(torch.float64).tolist()]


def _bf16_nearest(v: Fraction) -> Fraction:
    f = float(v)
    b = struct.unpack("<I", struct.pack("<f", np.float32(f)))[0] >> 16
    best = None
    for c in range(b - 2, b + 3):
        c &= 0xFFFF
        cv = Fraction(struct.unpack("<f", struct.pack("<I", c << 16))[0])
        d = abs(cv - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c, cv)
    return best[2]


def _brute(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b,
           bias_vals):
    A = _dec(a8, fa)
    B = _dec(b8, fb)
    inv = 1 / (Fraction(float(np.float32(sa))) * Fraction(float(np.float32(sb))))
    out = np.zeros((batch, M, N))
    for b in range(batch):
        for i in range(M):
            for j in range(N):
                acc = Fraction(0)
                for k in range(K):
                    if layout == NT:
                        av, bv = A[b * stride_a + i * K + k], B[b * stride_b + j * K + k]
                    elif layout == NN:
                        av, bv = A[b * stride_a + i * K + k], B[b * stride_b + k * N + j]
                    else:
                        av, bv = A[b * stride_a + k * M + i], B[b * stride_b + k * N + j]
                    acc += av * bv
                out[b, i, j] = float(_bf16_nearest(acc * inv + bias_vals[j]))
    return out


@pytest.mark.parametrize("layout", [NT, NN, TN])
@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 3, 4), (3, 5, 7), (4, 2, 9)])
@pytest.mark.parametrize("fmts", [(E4M3, E4M3), (E5M2, E4M3)])
def test_brute_force_tiny(layout, shape, fmts):
    M, N, K = shape
    fa, fb = fmts
    a8 = fp8_codes((M * K,), fa, 100 + M).numpy()
    b8 = fp8_codes((N * K,), fb, 200 + N).numpy()
    sa, sb = np.float32(0.75), np.float32(1.3)
    y, _ = oracle.mm(a8, fa, b8, fb, sa, sb, layout, M, N, K)
    want = _brute(a8, fa, b8, fb, sa, sb, layout, M, N, K, 1, M * K, N * K,
                  [Fraction(0)] * N)
    assert np.array_equal(y, want.astype(np.float32))


@pytest.mark.parametrize("layout", [NT, NN, TN])
def test_brute_force_batched_broadcast_and_bias(layout):
    M, N, K, batch = 3, 5, 6, 3
    a8 = fp8_codes((batch * M * K,), E4M3, 301).numpy()
    b8 = fp8_codes((N * K,), E4M3, 302).numpy()       # broadcast: stride 0
    bias_bits = torch.randn(N, generator=torch.Generator().manual_seed(3)).to(
        torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    bias_vals = [Fraction(v) for v in torch.from_numpy(bias_bits.view(np.int16)).view(
        torch.bfloat16).to(torch.float64).tolist()]
    sa, sb = np.float32(2.0), np.float32(0.625)
    y, _ = oracle.mm(a8, E4M3, b8, E4M3, sa, sb, layout, M, N, K, batch=batch,
                     stride_a=M * K, stride_b=0, bias=bias_bits)
    want = _brute(a8, E4M3, b8, E4M3, sa, sb, layout, M, N, K, batch, M * K, 0, bias_vals)
    assert np.array_equal(y, want.astype(np.float32))


def test_brute_force_fp8_bias():
    M, N, K = 2, 7, 5
    a8 = fp8_codes((M * K,), E4M3, 401).numpy()
    b8 = fp8_codes((N * K,), E4M3, 402).numpy()
    bias8 = fp8_codes((N,), E5M2, 403).numpy()
    bscale = np.float32(3.0)
    bias_vals = [v / Fraction(3) for v in _dec(bias8, E5M2)]
    y, _ = oracle.mm(a8, E4M3, b8, E4M3, 1.0, 1.0, NT, M, N, K, bias=bias8,
                     bias_scale=bscale, bias_fmt=E5M2)
    want = _brute(a8, E4M3, b8, E4M3, 1.0, 1.0, NT, M, N, K, 1, M * K, N * K, bias_vals)
    assert np.array_equal(y[0], want[0].astype(np.float32))


def test_identity_operand_reproduces_the_other():
    """A = I (code 0x38 = 1.0 on the diagonal): y = B^T exactly (fp8 values
    are bf16-representable)."""
    n = 48
    a8 = np.zeros((n, n), np.uint8)
    a8[np.arange(n), np.arange(n)] = 0x38
    b8 = fp8_codes((n * n,), E4M3, 501).numpy()
    y, _ = oracle.mm(a8.reshape(-1), E4M3, b8, E4M3, 1.0, 1.0, NT, n, n, n)
    bt = oracle.decode_table(E4M3)[b8.reshape(n, n)].T
    assert np.array_equal(y[0].astype(np.float64), bt)
    # NN with the same B stored as [K, N] gives B itself
    y2, _ = oracle.mm(a8.reshape(-1), E4M3, b8, E4M3, 1.0, 1.0, NN, n, n, n)
    assert np.array_equal(y2[0].astype(np.float64), bt.T)


def test_single_nonzero_k_is_one_exact_product():
    M, N, K, k0 = 9, 11, 13, 6
    a8 = np.zeros((M, K), np.uint8)
    a8[:, k0] = fp8_codes((M,), E5M2, 601).numpy()
    b8 = np.zeros((N, K), np.uint8)
    b8[:, k0] = fp8_codes((N,), E4M3, 602).numpy()
    y, s = oracle.mm(a8.reshape(-1), E5M2, b8.reshape(-1), E4M3, 1.0, 1.0, NT, M, N, K)
    av = oracle.decode_table(E5M2)[a8[:, k0]]
    bv = oracle.decode_table(E4M3)[b8[:, k0]]
    assert np.array_equal(y[0].astype(np.float64), np.outer(av, bv))
    assert np.array_equal(s[0], np.abs(np.outer(av, bv)))


def test_sampled_equals_full():
    M, N, K, batch = 37, 29, 64, 2
    a8 = fp8_codes((batch * K * M,), E4M3, 701).numpy()
    b8 = fp8_codes((K * N,), E5M2, 702).numpy()
    y, s = oracle.mm(a8, E4M3, b8, E5M2, 0.5, 4.0, TN, M, N, K, batch=batch,
                     stride_a=K * M, stride_b=0)
    rng = np.random.default_rng(0)
    idx = np.stack([rng.integers(0, batch, 200), rng.integers(0, M, 200),
                    rng.integers(0, N, 200)], axis=1)
    ys, ss = oracle.mm_sampled(a8, E4M3, b8, E5M2, 0.5, 4.0, TN, M, N, K, idx,
                               batch=batch, stride_a=K * M, stride_b=0)
    assert np.array_equal(ys, y[idx[:, 0], idx[:, 1], idx[:, 2]])
    assert np.allclose(ss, s[idx[:, 0], idx[:, 1], idx[:, 2]], rtol=1e-12)


def test_tolerance_ulp_points():
    t = oracle.tolerance(np.array([1.0, 1.5, -3.0, 2.0 ** -130, 0.0, 256.0]), np.zeros(6))
    assert list(t) == [2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -133, 2.0 ** -133, 2.0]
    assert oracle.tolerance(np.array([0.0]), np.array([2.0 ** 16]))[0] == 1.0 + 2.0 ** -133


def test_mm_out8_identity_and_composition():
    """An identity A passes B's values through exactly (scale 1, no bias), so
    the FP8 output reproduces B's codes for every finite non-negative-zero
    code of the same format; with a scale and a bias the codes are the quantize
    of fp32(y); the amax is max |fp32(y)|."""
    M = N = K = 32
    for fmt in (E4M3, E5M2):
        one = int(np.nonzero(oracle.decode_table(fmt) == 1.0)[0][0])
        a = np.zeros((M, K), np.uint8)
        a[np.arange(M), np.arange(K)] = one
        b = W.fp8_codes((K * N,), fmt, 41 + fmt).numpy()
        b[b == 0x80] = 0  # -0 sums to +0
        q, y64, s, amax = oracle.mm_out8(a.reshape(-1), fmt, b, fmt, 1.0, 1.0, NN, M, N, K, fmt, 1.0)
        assert np.array_equal(q[0].reshape(-1), b)
        assert amax == np.max(np.abs(oracle.decode_table(fmt)[b]))
    # composition with a scale and a bf16 bias
    a8 = W.fp8_codes((64 * 96,), E4M3, 51).numpy()
    b8 = W.fp8_codes((80 * 96,), E4M3, 52).numpy()
    bias = W.bf16_normal((80,), 0.5, 53).view(torch.int16).numpy().view(np.uint16)
    q, y64, s, amax = oracle.mm_out8(a8, E4M3, b8, E4M3, 0.75, 2.0, NT, 64, 80, 96, E5M2, 3.5, bias=bias)
    y32 = y64.astype(np.float32)
    assert np.array_equal(q.reshape(-1), oracle.quantize_with_scale(y32.reshape(-1), np.float32(3.5), E5M2))
    assert amax == np.max(np.abs(y32))
    yb, _ = oracle.mm(a8, E4M3, b8, E4M3, 0.75, 2.0, NT, 64, 80, 96, bias=bias)
    assert np.array_equal(yb, oracle.bf16_round_from_f64(y64).astype(np.float32))


def test_fp8_ulp_points():
    assert oracle.fp8_ulp(448.0, E4M3) == 32.0          # 1.75 * 2^8: spacing 2^(8-3)
    assert oracle.fp8_ulp(1.0, E4M3) == 0.125
    assert oracle.fp8_ulp(2.0 ** -10, E4M3) == 2.0 ** -9  # subnormal spacing
    assert oracle.fp8_ulp(0.0, E5M2) == 2.0 ** -16
    assert oracle.fp8_ulp(57344.0, E5M2) == 2.0 ** 13   # 1.75 * 2^15
