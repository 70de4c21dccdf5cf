"""A linear layer's FP8 training step, composed from the oracle's pieces.

Test infrastructure only (see the package docstring).

What the AstrAI commit logs fix (``astrai/extension/fp8.py`` @4dc5e923 and
@f4c44ebf): the forward quantizes x and W (E4M3) with one delayed ring each
and computes y = x W^T (+ bias); the backward quantizes g (E5M2) with its own
ring and computes dX = g W and dW = g^T x with the scales the forward used
(bullet on carrying the forward's scale to backward); the gradients come out
in bf16; the bias gradient is the column sum of g over the flattened leading
dimensions, computed only when the bias needs it, from the bf16 g.

Readings: the bias gradient is summed in fp64 and rounded once to bf16.
Tolerance of the GPU's fp32 sum: ulp_bf16 + 2^-14 * sum|g| (at most 1024
sequential fp32 additions per partial, each off by at most 2^-24 of the
running sum, then a tree of 8).
"""

import numpy as np

from .codec import bf16_round_from_f64
from .gemm import NN, NT, TN, mm
from .quantize import DelayedRing


def bias_grad(g):
    """bf16(sum over rows of g) for g [rows, cols] holding bf16 values."""
    g = np.asarray(g, dtype=np.float64)
    return bf16_round_from_f64(g.sum(axis=0))


def bias_grad_tolerance(out, g):
    out = np.abs(np.asarray(out, dtype=np.float64))
    _, ex = np.frexp(np.where(out > 0, out, 1.0))
    e = np.where(out > 0, np.maximum(ex - 1, -126), -126)
    return np.ldexp(1.0, e - 7) + 2.0 ** -14 * np.abs(np.asarray(g, dtype=np.float64)).sum(axis=0)


class Fp8LinearRef:
    """The FP8 linear layer: three delayed rings (x, W, g)."""

    def __init__(self):
        self.rx, self.rw, self.rg = DelayedRing(), DelayedRing(), DelayedRing()

    def forward(self, x, w, bias_bits=None):
        """x [T, K], w [N, K] (bf16 values). Returns (y, saved) with y the
        bf16 output [T, N] and the oracle's abs-sum for the tolerance."""
        T, K = x.shape
        N = w.shape[0]
        qx, _, sx = self.rx.step(x.reshape(-1), 0)
        qw, _, sw = self.rw.step(w.reshape(-1), 0)
        y, s = mm(qx, 0, qw, 0, sx, sw, NT, T, N, K, bias=bias_bits)
        return y[0], s[0], (qx, qw, sx, sw, T, N, K)

    def backward(self, g, saved):
        """g [T, N] (bf16 values) -> (dx, dx_abs, dw, dw_abs)."""
        qx, qw, sx, sw, T, N, K = saved
        qg, _, sg = self.rg.step(g.reshape(-1), 1)
        dx, sdx = mm(qg, 1, qw, 0, sg, sw, NN, T, K, N)
        dw, sdw = mm(qg, 1, qx, 0, sg, sx, TN, N, K, T)
        return dx[0], sdx[0], dw[0], sdw[0]
