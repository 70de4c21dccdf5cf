"""Pins for the oracle's linear-layer composition and bias gradient (CPU)."""

from fractions import Fraction

import numpy as np
import oracle
from workloads import bf16_normal


def _nearest_bf16(v: Fraction) -> float:
    """Exhaustive nearest-even bf16 to an exact rational."""
    import struct
    b = struct.unpack("<I", struct.pack("<f", np.float32(float(v))))[0] >> 16
    best = None
    for c in range(b - 2, b + 3):
        c &= 0xFFFF
        cv = Fraction(struct.unpack("<f", struct.pack("<I", c << 16))[0])
        d = abs(cv - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c, float(cv))
    return best[2]


def test_bias_grad_exact_brute_force():
    g = bf16_normal((37, 10), 0.5, 1).float().numpy()
    got = oracle.bias_grad(g)
    for j in range(10):
        exact = sum(Fraction(float(v)) for v in g[:, j])
        assert got[j] == _nearest_bf16(exact), j


def test_bias_grad_closed_forms():
    ones = np.ones((2048, 6), np.float32)
    assert np.all(oracle.bias_grad(ones) == 2048.0)
    alt = np.tile(np.array([[1.5], [-1.5]], np.float32), (100, 4))
    assert np.all(oracle.bias_grad(alt) == 0.0)


def test_linear_ref_matches_the_direct_definition():
    """Forward y is within the GEMM tolerance of x W^T computed from the
    dequantized codes, and the backward uses the forward's W scale."""
    x = bf16_normal((64, 96), 0.02, 3).float().numpy()
    w = bf16_normal((48, 96), 0.02, 4).float().numpy()
    g = bf16_normal((64, 48), 1e-3, 5).float().numpy()
    lin = oracle.Fp8LinearRef()
    y, s, saved = lin.forward(x, w)
    qx, qw, sx, sw, T, N, K = saved
    dx4 = oracle.decode_table(0)[qx].reshape(T, K) / float(sx)
    dw4 = oracle.decode_table(0)[qw].reshape(N, K) / float(sw)
    direct = dx4 @ dw4.T
    assert np.all(np.abs(y - direct) <= oracle.tolerance(direct, s))
    dx, _, dw, _ = lin.backward(g, saved)
    # against the unquantized products: FP8 noise only (direction preserved)
    true_dx = g.astype(np.float64) @ w.astype(np.float64)
    cos = (dx * true_dx).sum() / np.linalg.norm(dx) / np.linalg.norm(true_dx)
    assert cos > 0.99
    true_dw = g.astype(np.float64).T @ x.astype(np.float64)
    cos = (dw * true_dw).sum() / np.linalg.norm(dw) / np.linalg.norm(true_dw)
    assert cos > 0.99
