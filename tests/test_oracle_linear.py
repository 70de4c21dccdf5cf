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


# ---------------------------------------------------------------------------
# Scale wiring of the backward, element by element.
#
# AstrAI commit log astrai/extension/fp8.py @f4c44ebf: the backward GEMMs use
# the scales the forward quantized with (bullet on carrying sx/sw into
# backward), captured before the ring finalize replaces them (bullet on the
# scale snapshot). On a fresh ring every scale is 1, so the wiring is only
# visible from the second step on; the tensors below give x, W and g scales
# that differ by large factors, and step 2 doubles every magnitude so that
# each ring's published scale differs from the one the step used.

def _torch_dec(codes, fmt):
    """Exact decode through torch's float8 types (an independent library)."""
    import torch
    t = torch.as_tensor(np.asarray(codes, np.uint8).reshape(-1))
    return t.view(torch.float8_e4m3fn if fmt == 0 else torch.float8_e5m2).to(torch.float64).numpy()


def _first_step_scale(t, fmt_max):
    """A ring's scale after one fold of amax a from the initial state:
    fmt_max / a in IEEE fp32 (the window holds a and zeros)."""
    a = np.float32(np.max(np.abs(np.asarray(t, np.float32))))
    return np.float32(np.float32(fmt_max) / a)


def _two_steps():
    T, K, N = 96, 80, 64
    x1 = bf16_normal((T, K), 0.02, 61).float().numpy()
    w1 = bf16_normal((N, K), 0.5, 62).float().numpy()
    g1 = bf16_normal((T, N), 1e-3, 63).float().numpy()
    # step 2: fresh draws at twice the magnitude (x2 exact in bf16)
    x2 = 2 * bf16_normal((T, K), 0.02, 64).float().numpy()
    w2 = 2 * bf16_normal((N, K), 0.5, 65).float().numpy()
    g2 = 2 * bf16_normal((T, N), 1e-3, 66).float().numpy()
    lin = oracle.Fp8LinearRef()
    lin.backward(g1, lin.forward(x1, w1)[2])
    y, ys, saved = lin.forward(x2, w2)
    dx, sdx, dw, sdw = lin.backward(g2, saved)
    return (x1, w1, g1, x2, w2, g2), lin, (y, ys, saved, dx, sdx, dw, sdw), (T, K, N)


def _direct(codes_a, fa, sa, shape_a, codes_b, fb, sb, shape_b, ta=False, tb=False):
    A = _torch_dec(codes_a, fa).reshape(shape_a) / np.float64(sa)
    B = _torch_dec(codes_b, fb).reshape(shape_b) / np.float64(sb)
    A = A.T if ta else A
    B = B.T if tb else B
    return A @ B, np.abs(A) @ np.abs(B)


def test_linear_backward_scale_wiring_element_wise():
    """Step 2: the codes are quantize_with_scale of the inputs with the
    scales published by step 1 (fmt_max / step-1 amax), and y, dX, dW equal
    the fp64 products of those codes divided by exactly the scales each
    operand was quantized with: y = (qx/sx)(qw/sw)^T, dX = (qg/sg)(qw/sw),
    dW = (qg/sg)^T (qx/sx), each within the GEMM tolerance."""
    (x1, w1, g1, x2, w2, g2), lin, (y, ys, saved, dx, sdx, dw, sdw), (T, K, N) = _two_steps()
    sx = _first_step_scale(x1, 448.0)
    sw = _first_step_scale(w1, 448.0)
    sg = _first_step_scale(g1, 57344.0)
    # the three scales are far apart, so any swap moves results by large factors
    assert sx / sw > 8 and sg / sx > 8
    qx = oracle.quantize_with_scale(x2.reshape(-1), sx, 0)
    qw = oracle.quantize_with_scale(w2.reshape(-1), sw, 0)
    qg = oracle.quantize_with_scale(g2.reshape(-1), sg, 1)
    assert np.array_equal(saved[0], qx) and np.array_equal(saved[1], qw)
    assert saved[2] == sx and saved[3] == sw

    ey, ey_abs = _direct(qx, 0, sx, (T, K), qw, 0, sw, (N, K), tb=True)
    assert np.all(np.abs(y - ey) <= oracle.tolerance(ey, ey_abs))
    edx, edx_abs = _direct(qg, 1, sg, (T, N), qw, 0, sw, (N, K))
    assert np.all(np.abs(dx - edx) <= oracle.tolerance(edx, edx_abs))
    edw, edw_abs = _direct(qg, 1, sg, (T, N), qx, 0, sx, (T, K), ta=True)
    assert np.all(np.abs(dw - edw) <= oracle.tolerance(edw, edw_abs))


def test_linear_backward_rejects_the_published_scales():
    """The comparison above is sharp enough to tell the snapshot from the
    scale the ring published after step 2 (fmt_max / the doubled amax), and
    from the other operand's scale: either substitution puts dX or dW out of
    tolerance."""
    (x1, w1, g1, x2, w2, g2), lin, (y, ys, saved, dx, sdx, dw, sdw), (T, K, N) = _two_steps()
    sx = _first_step_scale(x1, 448.0)
    sw = _first_step_scale(w1, 448.0)
    sg = _first_step_scale(g1, 57344.0)
    qx, qw = saved[0], saved[1]
    qg = oracle.quantize_with_scale(g2.reshape(-1), sg, 1)
    # rings after step 2: the window max is the step-2 amax, so the
    # published scales moved away from the snapshots the step used
    for ring, s in ((lin.rx, sx), (lin.rw, sw), (lin.rg, sg)):
        assert ring.scale != s
    wrong = [
        ("dX with the published W scale", dx, _direct(qg, 1, sg, (T, N), qw, 0, lin.rw.scale, (N, K))),
        ("dX with the x scale", dx, _direct(qg, 1, sg, (T, N), qw, 0, sx, (N, K))),
        ("dW with the published x scale", dw, _direct(qg, 1, sg, (T, N), qx, 0, lin.rx.scale, (T, K), ta=True)),
        ("dW with the W scale", dw, _direct(qg, 1, sg, (T, N), qx, 0, sw, (T, K), ta=True)),
        ("dX with the published g scale", dx, _direct(qg, 1, lin.rg.scale, (T, N), qw, 0, sw, (N, K))),
    ]
    for name, got, (alt, alt_abs) in wrong:
        assert np.any(np.abs(got - alt) > oracle.tolerance(alt, alt_abs)), name


# ---------------------------------------------------------------------------
# Worked points of the two tolerance formulas that are readings.

def test_bias_grad_tolerance_worked_points():
    """ulp_bf16(out) + 2^-14 * sum|g|, by hand: a column of 2048 ones sums to
    2048 = 2^11, whose bf16 spacing is 2^(11-7) = 16, plus 2^-14 * 2048 =
    1/8; a column of alternating +-1.5 sums to 0, where the spacing takes
    its floor 2^(-126-7), plus 2^-14 * 300."""
    ones = np.ones((2048, 1), np.float32)
    assert oracle.bias_grad_tolerance(np.array([2048.0]), ones)[0] == 16.125
    alt = np.tile(np.array([[1.5], [-1.5]], np.float32), (100, 1))
    tol = oracle.bias_grad_tolerance(np.array([0.0]), alt)[0]
    assert tol == 2.0 ** -133 + 2.0 ** -14 * 300.0
    # a non-power of two: 3.0 lies in [2, 4), spacing 2^(1-7)
    assert oracle.bias_grad_tolerance(np.array([-3.0]), np.array([[1.0], [-4.0]], np.float32))[0] == \
        2.0 ** -6 + 2.0 ** -14 * 5.0


def test_bias_grad_tolerance_covers_a_blocked_fp32_sum():
    """The bound's own derivation: fp32 partial sums over blocks of up to
    1024 rows in sequence, then the partials added in fp32, then one bf16
    rounding. That summation order, done here in numpy float32 on 8192 rows
    of wide-ranging values, stays inside the tolerance of the exact sum."""
    rng = np.random.default_rng(5)
    g = (rng.standard_normal((8192, 16)) * np.exp2(rng.integers(-6, 6, (8192, 16)))).astype(np.float32)
    exact = oracle.bias_grad(g)
    tol = oracle.bias_grad_tolerance(exact, g)
    parts = []
    for b in range(0, g.shape[0], 1024):
        acc = np.zeros(g.shape[1], np.float32)
        for r in range(b, min(b + 1024, g.shape[0])):
            acc = (acc + g[r]).astype(np.float32)
        parts.append(acc)
    tot = np.zeros(g.shape[1], np.float32)
    for p in parts:
        tot = (tot + p).astype(np.float32)
    got = oracle.bf16_round_from_f64(tot.astype(np.float64))
    assert np.all(np.abs(got - exact) <= tol)


def test_out8_tolerance_worked_points():
    """|dec(q) - clamp(y * s)| <= fp8 spacing at the clamped target +
    (2^-16 * abs_sum + 2^-23 * |y|) * s, by hand."""
    # y = 3, s = 2 (E4M3): target 6 = 1.5 * 2^2, spacing 2^(2-3) = 0.5;
    # error term (2^-16 * 4 + 2^-23 * 3) * 2
    t, tol = oracle.out8_tolerance(np.array([3.0]), np.array([4.0]), 2.0, 0)
    assert t[0] == 6.0 and tol[0] == 0.5 + 2.0 ** -13 + 6.0 * 2.0 ** -23
    # beyond the format maximum the target clamps: 1000 -> 448, spacing 32
    t, tol = oracle.out8_tolerance(np.array([1000.0]), np.array([0.0]), 1.0, 0)
    assert t[0] == 448.0 and tol[0] == 32.0 + 1000.0 * 2.0 ** -23
    # E5M2 below the maximum's negative: -70000 -> -57344, spacing 2^13
    t, tol = oracle.out8_tolerance(np.array([-70000.0]), np.array([0.0]), 1.0, 1)
    assert t[0] == -57344.0 and tol[0] == 2.0 ** 13 + 70000.0 * 2.0 ** -23
    # a subnormal target: 2^-8 * 0.25 = 2^-10 in E4M3's subnormal range,
    # spacing 2^-9
    t, tol = oracle.out8_tolerance(np.array([2.0 ** -8]), np.array([0.0]), 0.25, 0)
    assert t[0] == 2.0 ** -10 and tol[0] == 2.0 ** -9 + 2.0 ** -8 * 2.0 ** -23 * 0.25
