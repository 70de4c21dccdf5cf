"""Helpers shared by the GPU parity tests: device buffers and calls through
the C ABI (via the thin binding), and conversion of results to numpy."""

import numpy as np
import torch

import fp8_delayed_scaling_quantize_b200 as fp8

DEV = "cuda"


def new_ring(init_scale: float = 1.0):
    ring = torch.empty(fp8.FP8_RING_BYTES // 4, dtype=torch.int32, device=DEV)
    fp8.fp8_ring_init(ring, init_scale)
    return ring


def ring_state(ring):
    h = fp8.fp8_ring_get(ring)
    return np.array(list(h.hist), np.float32), np.float32(h.scale), int(h.idx), int(h.amax_bits), int(h.ticket)


def quantize(x_dev, fmt, ring=None):
    """Returns (codes uint8 tensor on the device, amax tensor[1], scale tensor[1])."""
    n = x_dev.numel()
    out = torch.empty(n, dtype=torch.uint8, device=DEV)
    amax = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    scale = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    fp8.fp8_quantize(x_dev if n else None, n, fmt, ring, out if n else None, amax, scale)
    return out, amax, scale


def quantize_ex(x_dev, dtype, fmt, ring=None, flags=0):
    """fp8_quantize_ex on a device tensor of any input type; returns
    (codes, amax tensor[1], scale tensor[1])."""
    n = x_dev.numel()
    out = torch.empty(max(n, 1), dtype=torch.uint8, device=DEV)
    amax = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    scale = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    fp8.fp8_quantize_ex(x_dev if n else None, dtype, n, fmt, ring, flags, out if n else None, amax, scale)
    return out[:n], amax, scale


def f32(t):
    return t.detach().float().cpu().numpy()


def codes(t):
    return t.detach().cpu().numpy().astype(np.uint8)


def mm(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch=1, stride_a=None, stride_b=None,
       stride_c=None, bias=None, bias_scale=None, bias_fmt=0, out=None, ws=None, split_k=0):
    """fp8_mm (fp8_mm_ws when a workspace is given) through the C ABI;
    allocates the bf16 output when not given."""
    stride_a = M * K if stride_a is None else stride_a
    stride_b = N * K if stride_b is None else stride_b
    stride_c = M * N if stride_c is None else stride_c
    if out is None:
        out = torch.empty(max(batch * stride_c, 1), dtype=torch.bfloat16, device=DEV)
    if ws is None and split_k == 0:
        fp8.fp8_mm(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c,
                   bias, bias_scale, bias_fmt, out)
    else:
        fp8.fp8_mm_ws(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c,
                      bias, bias_scale, bias_fmt, out, ws, split_k)
    return out


def workspace(nbytes):
    """A zero-filled GEMM workspace (uint8)."""
    return torch.zeros(max(int(nbytes), 4096), dtype=torch.uint8, device=DEV)


def assert_within(got, want, tol, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    bad = ~(err <= tol)
    if bad.any():
        i = np.argmax(np.where(bad, err - tol, -np.inf))
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst flat index {i}: "
            f"gpu {got.reshape(-1)[i]!r} oracle {want.reshape(-1)[i]!r} tol {np.asarray(tol).reshape(-1)[i] if np.ndim(tol) else tol!r}")
