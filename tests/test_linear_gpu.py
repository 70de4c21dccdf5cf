"""GPU parity of the FP8 training linear layer (autograd over the C ABI).

Against the oracle's composed linear step (same rings, same inputs): y, dX,
dW within the GEMM tolerance and the bias gradient within its own, over
three steps with changing magnitudes. Against a plain fp32 reference:
direction and norm of y and the gradients (the FP8 noise regression of the
AstrAI commit log astrai/extension/fp8.py @4dc5e923: grads match the bf16
reference by direction/norm)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f(t):
    return t.detach().float().cpu().numpy()


def test_linear_layer_matches_oracle_over_steps():
    from fp8_delayed_scaling_quantize_b200.linear import Fp8Linear
    T, K, N = 320, 256, 192
    layer = Fp8Linear(K, N, bias=True, device="cuda")
    with torch.no_grad():
        layer.weight.copy_(W.bf16_normal((N, K), 0.02, 11).cuda())
        layer.bias.copy_(W.bf16_normal((N,), 0.1, 12).cuda())
    ref = oracle.Fp8LinearRef()
    for step, f in enumerate((1.0, 3.0, 0.25)):
        x = (W.bf16_normal((T, K), 0.02, 20 + step).float() * f).to(torch.bfloat16).cuda().requires_grad_(True)
        g = (W.bf16_normal((T, N), 1e-3, 30 + step).float() * f).to(torch.bfloat16).cuda()
        y = layer(x)
        y.backward(g)
        wv = _f(layer.weight)
        yr, ys, saved = ref.forward(_f(x), wv, _bits(layer.bias))
        assert np.all(np.abs(_f(y) - yr) <= oracle.tolerance(yr, ys)), step
        dx, sdx, dw, sdw = ref.backward(_f(g), saved)
        assert np.all(np.abs(_f(x.grad) - dx) <= oracle.tolerance(dx, sdx)), step
        assert np.all(np.abs(_f(layer.weight.grad) - dw) <= oracle.tolerance(dw, sdw)), step
        db = oracle.bias_grad(_f(g))
        assert np.all(np.abs(_f(layer.bias.grad) - db) <= oracle.bias_grad_tolerance(db, _f(g))), step
        layer.weight.grad = None
        layer.bias.grad = None


def test_linear_layer_direction_against_fp32_and_3d_input():
    from fp8_delayed_scaling_quantize_b200.linear import Fp8Linear
    B, L, K, N = 4, 96, 512, 384
    layer = Fp8Linear(K, N, bias=False, device="cuda")
    x = W.bf16_normal((B, L, K), 1.0, 41).cuda().requires_grad_(True)
    g = W.bf16_normal((B, L, N), 1.0, 42).cuda()
    for _ in range(2):  # the second step quantizes with published delayed scales
        x.grad = None
        layer.weight.grad = None
        y = layer(x)
        y.backward(g)
    assert y.shape == (B, L, N) and x.grad.shape == x.shape and layer.bias is None
    xf, wf, gf = x.detach().float(), layer.weight.detach().float(), g.float()
    yf = xf @ wf.t()
    dxf = gf @ wf
    dwf = gf.reshape(-1, N).t() @ xf.reshape(-1, K)

    def cos(a, b):
        a, b = a.detach().float().reshape(-1), b.detach().float().reshape(-1)
        return float(a @ b / a.norm() / b.norm())

    assert cos(y, yf) > 0.995
    assert cos(x.grad, dxf) > 0.99          # E5M2 gradients: direction kept
    assert cos(layer.weight.grad, dwf) > 0.99
    assert abs(float(x.grad.float().norm() / dxf.norm()) - 1.0) < 0.05


def test_rings_checkpoint_through_state_dict():
    from fp8_delayed_scaling_quantize_b200.linear import Fp8Linear
    a = Fp8Linear(128, 64, device="cuda")
    x = W.bf16_normal((64, 128), 0.5, 51).cuda()
    for _ in range(3):
        a(x).sum().backward()
    b = Fp8Linear(128, 64, device="cuda")
    b.load_state_dict(a.state_dict())
    assert torch.equal(a.fp8_rings, b.fp8_rings)
    ya, yb = a(x), b(x)  # same weights, same rings -> identical outputs
    assert torch.equal(ya, yb)


@pytest.mark.parametrize("seed", range(8))
def test_linear_layer_random_shapes(seed):
    """Drawn shapes (tokens ragged, short ones included, as 2-D or 3-D
    input; d_in and d_out multiples of 16), with or without bias, two steps
    against the oracle's composed linear step."""
    from fp8_delayed_scaling_quantize_b200.linear import Fp8Linear
    rng = np.random.default_rng(49000 + seed)
    T = int(rng.choice([int(rng.integers(1, 33)), int(rng.integers(33, 700))]))
    K, N = (int(v) * 16 for v in rng.integers(1, 48, 2))
    bias = bool(rng.random() < 0.5)
    lead = (T,) if rng.random() < 0.5 else ((1, T) if T % 2 else (2, T // 2))
    layer = Fp8Linear(K, N, bias=bias, device="cuda")
    with torch.no_grad():
        layer.weight.copy_(W.bf16_normal((N, K), 0.05, 49100 + seed).cuda())
        if bias:
            layer.bias.copy_(W.bf16_normal((N,), 0.1, 49200 + seed).cuda())
    ref = oracle.Fp8LinearRef()
    for step, f in enumerate((1.0, float(rng.uniform(0.2, 5.0)))):
        x = (W.bf16_normal(lead + (K,), 0.5, 49300 + 10 * seed + step).float() * f).to(torch.bfloat16)
        x = x.cuda().requires_grad_(True)
        g = (W.bf16_normal(lead + (N,), 1e-2, 49400 + 10 * seed + step).float() * f).to(torch.bfloat16).cuda()
        y = layer(x)
        y.backward(g)
        what = f"step {step} T {T} lead {lead} K {K} N {N} bias {bias}"
        assert y.shape == lead + (N,) and x.grad.shape == x.shape, what
        yr, ys, saved = ref.forward(_f(x).reshape(-1, K), _f(layer.weight), _bits(layer.bias) if bias else None)
        assert np.all(np.abs(_f(y).reshape(-1, N) - yr) <= oracle.tolerance(yr, ys)), what
        dx, sdx, dw, sdw = ref.backward(_f(g).reshape(-1, N), saved)
        assert np.all(np.abs(_f(x.grad).reshape(-1, K) - dx) <= oracle.tolerance(dx, sdx)), what
        assert np.all(np.abs(_f(layer.weight.grad) - dw) <= oracle.tolerance(dw, sdw)), what
        if bias:
            db = oracle.bias_grad(_f(g).reshape(-1, N))
            assert np.all(np.abs(_f(layer.bias.grad) - db) <= oracle.bias_grad_tolerance(db, _f(g).reshape(-1, N))), what
            layer.bias.grad = None
        layer.weight.grad = None
