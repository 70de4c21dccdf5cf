"""Per-tensor-scaled FP8 GEMM with fused bias and bf16 output, in fp64.

Test infrastructure only (see the package docstring).

What the AstrAI commit logs fix:

* the three layouts a linear layer needs: forward y = x W^T, dX = g W,
  dW = g^T x (``tests/extension/test_fp8_mma.py @cebdd45d``, bullet on
  routing dX/dW; ``csrc/kernels/fp8/gemm.cuh @5e76fbd1``, bullet on the
  RowMajor/ColMajor operand tags).
* the bias joins in fp32 before the single bf16 rounding; a null bias scale
  means a bf16 bias, a non-null one an fp8 bias dequantized after the
  operand scaling (``astrai/extension/fp8.py @f4c44ebf``, bullet on the
  fused bias; ``tests/extension/test_fp8_mma.py @cebdd45d``, bullet on the
  bias_scale slot).
* 3-D operands: batches are sliced by strides and a stride of 0 broadcasts
  one matrix to every batch (``astrai/extension/fp8.py @f4c44ebf``, bullet
  on 3-D mm_fp8 operands).
* the output is always bf16 (``astrai/extension/fp8.py @f4c44ebf``, bullet
  dropping the fp8 output parameter); the FP8-in / FP8-out op that an earlier
  page adds (``tests/extension/test_fp8_mma.py @cebdd45d``, bullet on
  fp8_mm_prequant_fp8) is ``mm_out8``: the same y, rounded once to fp32, then
  quantized with the output scale as a quantize call would.

Definition written out (all matrices row-major, codes decoded exactly):

    NT: A [M,K], B [N,K]:  d[i,j] = sum_k A[i,k] B[j,k]
    NN: A [M,K], B [K,N]:  d[i,j] = sum_k A[i,k] B[k,j]
    TN: A [K,M], B [K,N]:  d[i,j] = sum_k A[k,i] B[k,j]
    y[i,j] = bf16( d[i,j] / (sa * sb) + bias[j] )

with d accumulated in fp64 (a library matmul: each product of two FP8
values is exact in fp64 and the sum's error, about K * 2^-53 * sum|ab|, is
far below the tolerance) and ONE rounding from fp64 to bf16.

Tolerance (the stated GEMM bound):
    |gpu - y| <= ulp_bf16(y) + 2^-16 * sum_k |A B| / (sa * sb)
with ulp_bf16(o) = 2^(max(floor(log2|o|), -126) - 7), 2^-133 for o = 0.
"""

import numpy as np

from .codec import bf16_bits_to_f32, bf16_round_from_f64, decode_table

NT = 0
NN = 1
TN = 2


def _decoded(codes, fmt):
    return decode_table(fmt)[np.asarray(codes, dtype=np.uint8)]


def _op_a(a8, fa, layout, M, K, b, stride_a):
    """op(A) of batch b as a float64 [M, K] matrix."""
    base = b * stride_a
    flat = np.asarray(a8, dtype=np.uint8).reshape(-1)[base: base + M * K]
    if layout in (NT, NN):
        return _decoded(flat, fa).reshape(M, K)
    if layout == TN:
        return _decoded(flat, fa).reshape(K, M).T
    raise ValueError(f"unknown layout {layout}")


def _op_b(b8, fb, layout, N, K, b, stride_b):
    """op(B) of batch b as a float64 [K, N] matrix."""
    base = b * stride_b
    flat = np.asarray(b8, dtype=np.uint8).reshape(-1)[base: base + N * K]
    if layout == NT:
        return _decoded(flat, fb).reshape(N, K).T
    if layout in (NN, TN):
        return _decoded(flat, fb).reshape(K, N)
    raise ValueError(f"unknown layout {layout}")


def _bias64(bias, bias_scale, bias_fmt, N):
    """Bias as float64 [N]: bf16 bits (uint16) or fp8 codes / bias_scale."""
    if bias is None:
        return np.zeros(N, dtype=np.float64)
    bias = np.asarray(bias).reshape(-1)[:N]
    if bias_scale is None:
        return bf16_bits_to_f32(bias.astype(np.uint16)).astype(np.float64)
    return _decoded(bias.astype(np.uint8), bias_fmt) / np.float64(np.float32(bias_scale))


def mm_exact(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch=1, stride_a=None,
             stride_b=None, bias=None, bias_scale=None, bias_fmt=0):
    """The GEMM before any output rounding. Returns (y [batch,M,N] =
    d / (sa sb) + bias in fp64, abs_sum [batch,M,N] = sum_k |A B| / (sa sb))."""
    stride_a = M * K if stride_a is None else stride_a
    stride_b = N * K if stride_b is None else stride_b
    inv = 1.0 / (np.float64(np.float32(sa)) * np.float64(np.float32(sb)))
    bias64 = _bias64(bias, bias_scale, bias_fmt, N)
    y = np.empty((batch, M, N), dtype=np.float64)
    s = np.empty((batch, M, N), dtype=np.float64)
    for b in range(batch):
        A = _op_a(a8, fa, layout, M, K, b, stride_a)
        B = _op_b(b8, fb, layout, N, K, b, stride_b)
        y[b] = (A @ B) * inv + bias64[None, :]
        s[b] = (np.abs(A) @ np.abs(B)) * inv
    return y, s


def mm(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch=1, stride_a=None,
       stride_b=None, bias=None, bias_scale=None, bias_fmt=0):
    """Full GEMM. Returns (y [batch,M,N] bf16 values as fp32,
    abs_sum [batch,M,N] = sum_k |A B| / (sa sb) as fp64)."""
    y64, s = mm_exact(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, bias, bias_scale,
                      bias_fmt)
    return bf16_round_from_f64(y64).astype(np.float32), s


def mm_out8(a8, fa, b8, fb, sa, sb, layout, M, N, K, out_fmt, out_scale, batch=1, stride_a=None,
            stride_b=None, bias=None, bias_scale=None, bias_fmt=0):
    """FP8-output GEMM: y as in ``mm`` rounded once to fp32, then
    q = sat_rne(fp32(y * out_scale)) (``quantize_with_scale``). Returns
    (codes [batch,M,N] uint8, y64 [batch,M,N], abs_sum [batch,M,N],
    amax = max |fp32(y)|)."""
    from .quantize import amax, quantize_with_scale
    y64, s = mm_exact(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, bias, bias_scale,
                      bias_fmt)
    y32 = y64.astype(np.float32)
    q = quantize_with_scale(y32.reshape(-1), np.float32(out_scale), out_fmt).reshape(y32.shape)
    return q, y64, s, amax(y32.reshape(-1))


def fp8_ulp(v, fmt):
    """Spacing of the FP8 values of ``fmt`` at magnitude |v| (the subnormal
    spacing below the smallest normal): 2^(max(e, emin) - mantissa bits)."""
    mbits, emin = (3, -6) if fmt == 0 else (2, -14)
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.where(a > 0, np.maximum(ex - 1, emin), emin)
    return np.ldexp(1.0, e - mbits)


def out8_tolerance(y64, abs_sum, out_scale, fmt):
    """Allowed |dec(q_gpu) - clamp(y64 * s)| for an FP8-output GEMM: one FP8
    spacing at the clamped target plus the GEMM's own error bound (2^-16 of
    the scaled absolute sum, and one fp32 rounding of y), scaled by s."""
    fmax = 448.0 if fmt == 0 else 57344.0
    s = np.float64(np.float32(out_scale))
    t = np.clip(np.asarray(y64, np.float64) * s, -fmax, fmax)
    err = (2.0 ** -16 * np.asarray(abs_sum, np.float64) + 2.0 ** -23 * np.abs(y64)) * s
    return t, fp8_ulp(t, fmt) + err


def mm_sampled(a8, fa, b8, fb, sa, sb, layout, M, N, K, idx, batch=1,
               stride_a=None, stride_b=None, bias=None, bias_scale=None,
               bias_fmt=0):
    """GEMM at sampled outputs only; idx is an int array of (b, i, j) rows.

    Returns (y [len(idx)] as fp32, abs_sum [len(idx)] as fp64).
    """
    stride_a = M * K if stride_a is None else stride_a
    stride_b = N * K if stride_b is None else stride_b
    idx = np.asarray(idx, dtype=np.int64).reshape(-1, 3)
    inv = 1.0 / (np.float64(np.float32(sa)) * np.float64(np.float32(sb)))
    bias64 = _bias64(bias, bias_scale, bias_fmt, N)
    y = np.empty(len(idx), dtype=np.float32)
    s = np.empty(len(idx), dtype=np.float64)
    for b in np.unique(idx[:, 0]):
        sel = np.nonzero(idx[:, 0] == b)[0]
        A = _op_a(a8, fa, layout, M, K, int(b), stride_a)
        B = _op_b(b8, fb, layout, N, K, int(b), stride_b)
        rows = A[idx[sel, 1], :]            # [n, K]
        cols = B[:, idx[sel, 2]].T          # [n, K]
        d = np.einsum("nk,nk->n", rows, cols)
        y[sel] = bf16_round_from_f64(d * inv + bias64[idx[sel, 2]])
        s[sel] = np.einsum("nk,nk->n", np.abs(rows), np.abs(cols)) * inv
    return y, s


def tolerance(y, abs_sum):
    """Allowed |gpu - oracle| per output: 1 bf16 ulp of the oracle value
    plus 2^-16 of the scaled absolute sum."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.where(a > 0, np.maximum(ex - 1, -126), -126)
    return np.ldexp(1.0, e - 7) + 2.0 ** -16 * np.asarray(abs_sum, dtype=np.float64)
