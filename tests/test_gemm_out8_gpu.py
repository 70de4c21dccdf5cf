"""GPU parity of fp8_mm_out8, the FP8-in / FP8-out GEMM with a delayed
output ring, against the oracle's mm_out8.

Bar per output: |dec(code) - clamp(y * s)| <= one FP8 spacing at the target
+ the GEMM's own error bound, times s (oracle.out8_tolerance): the GPU's fp32
y may sit on the other side of an FP8 rounding boundary than the exact one,
by at most the GEMM tolerance. The scale used is the ring's, exactly; the
reported amax is within the GEMM bound of the oracle's; the ring after each
call is the oracle's ring folded with that amax, exactly; nothing outside the
outputs is written.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2, NN, NT, TN
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import gpu_util
    return gpu_util


def _run_case(g, layout, M, N, K, fa, fb, out_fmt, seed, batch=1, bcast_b=False, bias_kind=0, pad_c=0):
    import fp8_delayed_scaling_quantize_b200 as fp8
    bb = 1 if bcast_b else batch
    a8 = W.fp8_codes((batch * M * K,), fa, seed)
    b8 = W.fp8_codes((bb * N * K,), fb, seed + 1)
    bias = bias_dev = bscale = bscale_dev = None
    if bias_kind == 1:
        t = W.bf16_normal((N,), 2.0, seed + 2)
        bias_dev = t.cuda()
        bias = t.view(torch.int16).numpy().view(np.uint16)
    elif bias_kind == 2:
        t = W.fp8_codes((N,), E5M2, seed + 2)
        bias, bias_dev = t.numpy(), t.cuda()
        bscale = np.float32(5.0)
        bscale_dev = torch.tensor([bscale], device="cuda")
    stride_c = M * N + pad_c
    stride_b = 0 if bcast_b else N * K
    ad, bd = a8.cuda(), b8.cuda()
    ring = g.new_ring(1.0)
    # ref folds the GPU's amax: the fp32 y that the amax is taken over is not
    # bit-defined (only held to the GEMM tolerance), so the ring's fold is
    # checked bit for bit given that amax; ref_own folds the oracle's own
    # amax and bounds the published scale by the amax tolerance
    ref = oracle.DelayedRing(1.0)
    ref_own = oracle.DelayedRing(1.0)
    for step, sa in enumerate((4.0, 0.5, 16.0)):
        sb = 1.5
        s_used = np.float32(ref.scale)
        out = torch.full((batch * stride_c + 64,), 0xEE, dtype=torch.uint8, device="cuda")
        amax = torch.full((1,), -1.0, device="cuda")
        scale = torch.full((1,), -1.0, device="cuda")
        fp8.fp8_mm_out8(ad, fa, bd, fb, torch.tensor([sa], device="cuda"), torch.tensor([sb], device="cuda"),
                        layout, M, N, K, batch, M * K, stride_b, stride_c, bias_dev, bscale_dev, E5M2, out_fmt, ring,
                        out, amax, scale)
        q, y64, s_abs, amax_want = oracle.mm_out8(a8.numpy(), fa, b8.numpy(), fb, sa, sb, layout, M, N, K, out_fmt,
                                                  s_used, batch=batch, stride_a=M * K, stride_b=stride_b, bias=bias,
                                                  bias_scale=bscale, bias_fmt=E5M2)
        got = out.cpu().numpy()
        codes = np.stack([got[b * stride_c: b * stride_c + M * N].reshape(M, N) for b in range(batch)])
        assert g.f32(scale)[0] == s_used, step
        target, tol = oracle.out8_tolerance(y64, s_abs, s_used, out_fmt)
        dec = oracle.decode_table(out_fmt)[codes]
        bad = ~(np.abs(dec - target) <= tol)
        assert not bad.any(), f"step {step}: {int(bad.sum())} codes outside the bound"
        assert (codes == q).mean() > 0.98, step  # all but boundary cases give the oracle's code itself
        a_gpu = g.f32(amax)[0]
        a_tol = 2.0 ** -16 * float(s_abs.max()) + 2.0 ** -22 * float(amax_want)
        assert abs(float(a_gpu) - float(amax_want)) <= a_tol
        ref.fold(a_gpu, out_fmt)
        ref_own.fold(amax_want, out_fmt)
        hist, rs, idx, acc, ticket = g.ring_state(ring)
        assert np.array_equal(hist, ref.hist) and rs == ref.scale and idx == ref.idx, step
        # the window maxima differ by at most a_tol, so the published scales
        # differ by that relative amount plus one fp32 rounding
        rel = a_tol / float(np.max(ref_own.hist))
        assert abs(float(rs) / float(ref_own.scale) - 1.0) <= rel / (1.0 - rel) + 2.0 ** -23, step
        assert acc == 0 and ticket == 0
        for b in range(batch):
            assert (got[b * stride_c + M * N: (b + 1) * stride_c] == 0xEE).all()
        assert (got[batch * stride_c:] == 0xEE).all()


@pytest.mark.parametrize("case", [
    (NT, 256, 256, 512, E4M3, E4M3, E4M3, 0), (NN, 200, 144, 384, E5M2, E4M3, E5M2, 1),
    (TN, 384, 512, 256, E5M2, E4M3, E4M3, 2), (NT, 64, 200, 128, E4M3, E4M3, E5M2, 1),
    (NT, 8, 512, 256, E4M3, E5M2, E4M3, 0), (NT, 1024, 1024, 512, E4M3, E4M3, E4M3, 1),
], ids=lambda c: f"{'NT NN TN'.split()[c[0]]}{c[1]}x{c[2]}x{c[3]}")
def test_out8_layouts_formats_bias(g, case):
    layout, M, N, K, fa, fb, out_fmt, bias_kind = case
    _run_case(g, layout, M, N, K, fa, fb, out_fmt, 3000 + M + N, bias_kind=bias_kind)


def test_out8_pair_tiles(g):
    """Large enough for SM-pair tiles: each CTA of a pair folds its own amax
    and takes its own ticket."""
    _run_case(g, NT, 2400, 4096, 2048, E4M3, E4M3, E4M3, 3100)


@pytest.mark.parametrize("layout", [NT, NN, TN])
def test_out8_batches(g, layout):
    _run_case(g, layout, 128, 256, 128, E4M3, E4M3, E5M2, 3200, batch=3, bcast_b=True, bias_kind=1, pad_c=48)


def test_out8_feeds_the_next_gemm(g):
    """The codes and the scale of an FP8-output GEMM are a valid operand of
    the next GEMM: y2 = out8 W2^T equals the oracle on those codes."""
    import fp8_delayed_scaling_quantize_b200 as fp8
    M, N, K, N2 = 256, 512, 384, 320
    a8 = W.fp8_codes((M * K,), E4M3, 3301)
    b8 = W.fp8_codes((N * K,), E4M3, 3302)
    w2 = W.fp8_codes((N2 * N,), E4M3, 3303)
    one = torch.ones(1, device="cuda")
    ring = g.new_ring(8.0)
    out = torch.empty(M * N, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, device="cuda")
    fp8.fp8_mm_out8(a8.cuda(), E4M3, b8.cuda(), E4M3, one, one, NT, M, N, K, 1, 0, 0, 0, None, None, 0, E4M3,
                    ring, out, None, sc)
    y2 = g.mm(out, E4M3, w2.cuda(), E4M3, sc, one, NT, M, N2, N)
    want, s = oracle.mm(out.cpu().numpy(), E4M3, w2.numpy(), E4M3, float(g.f32(sc)[0]), 1.0, NT, M, N2, N)
    g.assert_within(y2.float().cpu().numpy().reshape(M, N2), want[0], oracle.tolerance(want[0], s[0]), "chain")


@pytest.mark.parametrize("seed", range(16))
def test_out8_random_problems(g, seed):
    """Drawn problems (layout, formats, output format, sizes with the pitch
    rules kept and at least 4096 outputs, batches with B broadcast, padding,
    bias kind), each over three ring steps."""
    rng = np.random.default_rng(47000 + seed)
    layout = int(rng.choice([NT, NN, TN]))
    fa, fb, out_fmt = (int(v) for v in rng.integers(0, 2, 3))
    M = int(rng.integers(1, 40)) * 16 if layout == TN else int(rng.integers(16, 640))
    N = int(rng.integers(4, 40)) * 16 if layout != NT else int(rng.integers(64, 640))
    N = max(N, (4096 + M - 1) // M if layout == NT else N)
    K = int(rng.integers(1, 48)) * 16 if layout != TN else int(rng.integers(1, 768))
    batch = int(rng.choice([1, 1, 2]))
    bcast_b = batch > 1 and rng.random() < 0.5
    pad_c = int(rng.choice([0, 5, 16])) if batch > 1 else 0
    if M * N < 4096:
        M = (4096 + N - 1) // N if layout != TN else ((4096 + N - 1) // N + 15) // 16 * 16
    _run_case(g, layout, M, N, K, fa, fb, out_fmt, 48000 + 10 * seed, batch=batch, bcast_b=bcast_b,
              bias_kind=int(rng.integers(0, 3)), pad_c=pad_c)
