"""GPU parity of fp8_mm (through the C ABI) against the CPU oracle.

Bar: |gpu - oracle| <= ulp_bf16(oracle) + 2^-16 * sum_k |a b| / (sa sb) per
output (oracle.tolerance). Small shapes are compared in full; the full-size
workloads on sampled outputs (4096 random outputs plus 8 whole rows) in the
same launch configuration the bench uses.
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


def _dev(t):
    return t.contiguous().cuda()


def _scales(sa, sb):
    return (torch.tensor([sa], dtype=torch.float32, device="cuda"),
            torch.tensor([sb], dtype=torch.float32, device="cuda"))


def _shape_a(layout, M, K):
    return (K, M) if layout == TN else (M, K)


def _shape_b(layout, N, K):
    return (N, K) if layout == NT else (K, N)


def _full_check(g, layout, M, N, K, fa, fb, seed, batch=1, bcast_a=False, bcast_b=False,
                bias_kind=0, pad_c=0, sa=0.75, sb=1.5):
    ba = 1 if bcast_a else batch
    bb = 1 if bcast_b else batch
    a8 = W.fp8_codes((ba * M * K,), fa, seed)
    b8 = W.fp8_codes((bb * N * K,), fb, seed + 1)
    bias = bias_dev = bscale = bscale_dev = None
    if bias_kind == 1:
        bias = W.bf16_normal((N,), 0.1, seed + 2)
        bias_dev = _dev(bias)
        bias = bias.view(torch.int16).numpy().view(np.uint16)
    elif bias_kind == 2:
        b = W.fp8_codes((N,), E5M2, seed + 2)
        bias, bias_dev = b.numpy(), _dev(b)
        bscale = np.float32(5.0)
        bscale_dev = torch.tensor([bscale], device="cuda")
    sad, sbd = _scales(sa, sb)
    stride_c = M * N + pad_c
    out = torch.full((batch * stride_c + 64,), float("nan"), dtype=torch.bfloat16, device="cuda")
    g.mm(_dev(a8), fa, _dev(b8), fb, sad, sbd, layout, M, N, K, batch=batch,
         stride_a=0 if bcast_a else M * K, stride_b=0 if bcast_b else N * K,
         stride_c=stride_c, bias=bias_dev, bias_scale=bscale_dev, bias_fmt=E5M2, out=out)
    y, s = oracle.mm(a8.numpy(), fa, b8.numpy(), fb, sa, sb, layout, M, N, K, batch=batch,
                     stride_a=0 if bcast_a else M * K, stride_b=0 if bcast_b else N * K,
                     bias=bias, bias_scale=bscale, bias_fmt=E5M2)
    got = out.float().cpu().numpy()
    res = np.stack([got[b * stride_c: b * stride_c + M * N].reshape(M, N) for b in range(batch)])
    g.assert_within(res, y, oracle.tolerance(y, s), f"{layout} {M}x{N}x{K} b{batch}")
    # padding between batches and after the end is never written
    for b in range(batch):
        assert np.all(np.isnan(got[b * stride_c + M * N: (b + 1) * stride_c]))
    assert np.all(np.isnan(got[batch * stride_c:]))


@pytest.mark.parametrize("layout", [NT, NN, TN])
@pytest.mark.parametrize("shape", [(256, 256, 256), (128, 128, 128), (384, 512, 640),
                                   (304, 272, 144), (144, 144, 272), (16, 48, 32)])
def test_layouts_small(g, layout, shape):
    M, N, K = shape
    _full_check(g, layout, M, N, K, E4M3, E4M3, 10 + M + N + K)


@pytest.mark.parametrize("layout", [NT, NN, TN])
def test_mixed_formats_and_bias(g, layout):
    _full_check(g, layout, 208, 160, 384, E5M2, E4M3, 51, bias_kind=1)
    _full_check(g, layout, 144, 304, 256, E4M3, E5M2, 52, bias_kind=2)
    _full_check(g, layout, 64, 512, 1024, E5M2, E5M2, 53)


@pytest.mark.parametrize("N", [1, 7, 9, 63, 130, 257])
def test_nt_ragged_n(g, N):
    _full_check(g, NT, 200, N, 160, E4M3, E4M3, 60 + N, bias_kind=1)


@pytest.mark.parametrize("M", [1, 2, 8, 127, 129])
@pytest.mark.parametrize("layout", [NT, NN])
def test_ragged_m(g, M, layout):
    _full_check(g, layout, M, 256, 512, E4M3, E4M3, 70 + M, bias_kind=1)


@pytest.mark.parametrize("layout", [NT, NN, TN])
def test_batched_broadcast_and_padding(g, layout):
    _full_check(g, layout, 160, 144, 208, E4M3, E4M3, 80, batch=3, bcast_b=True, pad_c=40, bias_kind=1)
    _full_check(g, layout, 128, 256, 128, E4M3, E4M3, 81, batch=4, bcast_a=True)
    _full_check(g, layout, 96, 128, 96, E4M3, E4M3, 82, batch=5)


def test_odd_scales(g):
    _full_check(g, NT, 256, 256, 512, E4M3, E4M3, 90, sa=3.0e-3, sb=1.7e4, bias_kind=1)
    _full_check(g, TN, 256, 256, 512, E4M3, E4M3, 91, sa=0.5, sb=0.5)


# ------------------------------------------------------- full-size sampled ---

def _sample_idx(M, N, batch, seed, n=4096, rows=8):
    rng = np.random.default_rng(seed)
    idx = [np.stack([rng.integers(0, batch, n), rng.integers(0, M, n), rng.integers(0, N, n)], 1)]
    for r in rng.integers(0, M, rows):
        b = int(rng.integers(0, batch))
        idx.append(np.stack([np.full(N, b), np.full(N, r), np.arange(N)], 1))
    return np.concatenate(idx)


def _sampled_check(g, a8, fa, b8, fb, sa, sb, layout, M, N, K, batch=1, stride_a=None,
                   stride_b=None, bias=None, bias_np=None, seed=0, what=""):
    stride_a = M * K if stride_a is None else stride_a
    stride_b = N * K if stride_b is None else stride_b
    sad, sbd = _scales(sa, sb)
    out = g.mm(_dev(a8), fa, _dev(b8), fb, sad, sbd, layout, M, N, K, batch=batch,
               stride_a=stride_a, stride_b=stride_b, bias=bias)
    idx = _sample_idx(M, N, batch, seed)
    y, s = oracle.mm_sampled(a8.numpy(), fa, b8.numpy(), fb, sa, sb, layout, M, N, K, idx,
                             batch=batch, stride_a=stride_a, stride_b=stride_b, bias=bias_np)
    flat = out.float().view(batch, M, N)[torch.from_numpy(idx[:, 0]), torch.from_numpy(idx[:, 1]),
                                         torch.from_numpy(idx[:, 2])].cpu().numpy()
    g.assert_within(flat, y, oracle.tolerance(y, s), what)


@pytest.mark.parametrize("n", W.SQUARE_SIZES)
def test_square_sweep_sampled(g, n):
    a8 = W.fp8_codes((n * n,), E4M3, 3000 + n)
    b8 = W.fp8_codes((n * n,), E4M3, 3001 + n)
    sa, sb = (float(v) for v in W.uniform(0.5, 2.0, 3002 + n, 2))
    _sampled_check(g, a8, E4M3, b8, E4M3, sa, sb, NT, n, n, n, seed=n, what=f"square {n}")


def _current(g, x, fmt=E4M3):
    q, amax, scale = g.quantize(x.reshape(-1).cuda(), fmt, None)
    return q, float(g.f32(scale)[0])


@pytest.mark.parametrize("shape", W.SKINNY_SHAPES)
def test_skinny_with_bias(g, shape):
    M, N, K = shape
    a = W.bf16_normal((M, K), 1.0, 4000 + M)
    b = W.bf16_normal((N, K), 1.0, 4001 + M)
    bias = W.bf16_normal((N,), 0.1, 4002 + M)
    qa, sa = _current(g, a)
    qb, sb = _current(g, b)
    _sampled_check(g, qa.cpu(), E4M3, qb.cpu(), E4M3, sa, sb, NT, M, N, K, bias=_dev(bias),
                   bias_np=bias.view(torch.int16).numpy().view(np.uint16), seed=M, what=f"skinny {shape}")


@pytest.mark.parametrize("case", W.BATCHED)
def test_batched_configs(g, case):
    batch, M, N, K, bcast = case
    a = W.bf16_normal((batch, M, K), 1.0, 5000 + batch)
    b = W.bf16_normal((1 if bcast else batch, N, K), 1.0, 5001 + batch)
    qa, sa = _current(g, a)
    qb, sb = _current(g, b)
    _sampled_check(g, qa.cpu(), E4M3, qb.cpu(), E4M3, sa, sb, NT, M, N, K, batch=batch,
                   stride_b=0 if bcast else N * K, seed=batch, what=f"batched {case}")


def test_linear_stack_gemms_sampled(g):
    """Forward NT, dX NN and dW TN of every linear of the stack (step 0)."""
    tensors = W.stack_tensors(0)
    for li, ((name, d_in, d_out), t) in enumerate(zip(W.LINEARS, tensors)):
        qx, sx = _current(g, t["x"])
        qw, sw = _current(g, t["w"])
        qg, sg = _current(g, t["g"], E5M2)
        T = W.TOKENS
        _sampled_check(g, qx.cpu(), E4M3, qw.cpu(), E4M3, sx, sw, NT, T, d_out, d_in, seed=li,
                       what=f"{name} fwd")
        _sampled_check(g, qg.cpu(), E5M2, qw.cpu(), E4M3, sg, sw, NN, T, d_in, d_out, seed=li + 10,
                       what=f"{name} dX")
        _sampled_check(g, qg.cpu(), E5M2, qx.cpu(), E4M3, sg, sx, TN, d_out, d_in, T, seed=li + 20,
                       what=f"{name} dW")


def test_no_device_error_after_all(g):
    import fp8_delayed_scaling_quantize_b200 as fp8
    fp8.fp8_last_device_error()


# ------------------------------------------- SM-pair (256-row) tile path ---
# Shapes with at least one pair tile per SM (>= 148 tiles of 256 x 256) and
# at least 16 k-blocks run on SM pairs; compared in full, with ragged M (a
# last pair whose second CTA lies wholly past M), ragged N and K, every
# layout, bias and batches.

@pytest.mark.parametrize("layout,M,N,K", [
    (NT, 2400, 4096, 2048), (NT, 2368, 4000, 2032), (NN, 2560, 4096, 2032),
    (TN, 2560, 4096, 2056), (TN, 2368, 4096, 2048)])
def test_pair_tiles_full(g, layout, M, N, K):
    _full_check(g, layout, M, N, K, E4M3, E4M3, 1000 + M + N + K)


@pytest.mark.parametrize("layout", [NT, NN, TN])
def test_pair_tiles_bias_and_batches(g, layout):
    _full_check(g, layout, 1280, 2560, 2048, E5M2, E4M3, 1101, batch=3, bcast_b=True, pad_c=48, bias_kind=1)
    _full_check(g, layout, 2560, 4096, 2048, E4M3, E5M2, 1102, bias_kind=2)


# Narrow NT problems with a long K (few output tiles, many k-blocks): ragged
# M and N, bias of both kinds, broadcast batches.

@pytest.mark.parametrize("M,N,K,bias_kind", [(512, 512, 2048, 0), (1000, 1000, 1024, 1), (2048, 1024, 1024, 2),
                                             (136, 200, 4096, 1), (2048, 1024, 4096, 0)])
def test_narrow_long_k_nt(g, M, N, K, bias_kind):
    _full_check(g, NT, M, N, K, E4M3, E4M3, 1200 + M + N, bias_kind=bias_kind)


def test_narrow_long_k_nt_batches(g):
    _full_check(g, NT, 384, 640, 1024, E4M3, E5M2, 1301, batch=2, bcast_b=True, pad_c=32, bias_kind=1)


# Short problems (M <= 32, N >= 128, NT and NN) run with swapped operands: the
# kernel computes C^T = B^T A^T on tiles of 128 columns of C by 16 or 32 rows
# and writes C transposed. Every boundary of the 16/32-row tiles and of the
# switch back to unswapped tiles at 33 rows, ragged N, both bias kinds,
# batches with either operand broadcast, padded batch stride.

@pytest.mark.parametrize("M,N,K,bias_kind", [(1, 128, 256, 0), (7, 1000, 384, 1), (16, 4096, 1024, 2),
                                             (17, 256, 512, 1), (32, 640, 2048, 0), (33, 384, 256, 2),
                                             (63, 1000, 512, 1), (64, 136, 128, 0)])
def test_swapped_short_m_nt(g, M, N, K, bias_kind):
    _full_check(g, NT, M, N, K, E4M3, E5M2, 1400 + M + N, bias_kind=bias_kind)


@pytest.mark.parametrize("M,N,K,bias_kind", [(1, 144, 256, 1), (9, 1008, 384, 0), (16, 4096, 1024, 2),
                                             (31, 640, 512, 1), (48, 384, 2048, 0), (64, 128, 128, 1)])
def test_swapped_short_m_nn(g, M, N, K, bias_kind):
    _full_check(g, NN, M, N, K, E5M2, E4M3, 1500 + M + N, bias_kind=bias_kind)


@pytest.mark.parametrize("layout", [NT, NN])
def test_swapped_batches(g, layout):
    _full_check(g, layout, 12, 304, 256, E4M3, E4M3, 1601, batch=3, bcast_b=True, pad_c=24, bias_kind=1)
    _full_check(g, layout, 40, 256, 384, E5M2, E4M3, 1602, batch=2, bcast_a=True)
