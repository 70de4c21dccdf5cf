"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds no FP8 arithmetic: it only draws random numbers with
fixed seeds and describes shapes. Quantization, scales and products are
computed by the oracle on one side and by the CUDA library on the other.

Seeds follow ``seed = 1000 * workload + tensor_id``. All draws use torch's
CPU generator so the host bytes are identical wherever they are made.

Workloads (the shapes and distributions of the FP8 linear-layer path):

1. one NT GEMM M = N = K = 256; A, B bf16 ~ N(0, 1) current-scaled to E4M3;
   bias bf16 ~ N(0, 0.1) of length N; bf16 output.
2. one dim-1024 transformer linear stack at 2048 tokens (4 x 512): QKV
   1024 -> 3072, out 1024 -> 1024, MLP 1024 -> 4096 and 4096 -> 1024;
   x, W bf16 ~ N(0, 0.02) as E4M3, gradients ~ N(0, 1e-3) as E5M2;
   forward NT, dX NN, dW TN; delayed rings (H = 16) over 8 steps with each
   tensor's magnitude multiplied by U(0.5, 2) per step (a multiplicative
   walk per tensor role).
3. square NT E4M3 GEMMs on pre-quantized operands (uniform random codes
   without NaN, scales U(0.5, 2)), n in {1024, 2048, 4096, 8192}, no bias.
4. skinny / rectangular NT E4M3 GEMMs with bf16 bias: 64x8192x2048,
   1024x1536x2048 and decode shapes M in {1, 8} x N = 4096 x K = 4096.
5. batched E4M3 GEMMs: 64 x 512^3 independent, and 8 x 1024x2048x2048 with
   B broadcast (batch stride 0).
6. quantize inputs of the other types: every fp16 bit pattern, and fp32
   values over the whole fp32 range with the special values mixed in.
"""

import torch

# ----------------------------------------------------------------- draws ---


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def bf16_normal(shape, std: float, seed: int) -> torch.Tensor:
    """bf16 tensor ~ N(0, std^2) on the CPU (fp32 draw, then bf16)."""
    x = torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def f32_normal(shape, std: float, seed: int) -> torch.Tensor:
    """fp32 tensor ~ N(0, std^2) on the CPU."""
    return torch.randn(tuple(shape), generator=_gen(seed), dtype=torch.float32) * std


def uniform(lo: float, hi: float, seed: int, n: int = 1) -> torch.Tensor:
    """fp32 tensor of n draws ~ U(lo, hi)."""
    u = torch.rand(n, generator=_gen(seed), dtype=torch.float32)
    return lo + (hi - lo) * u


# Codes that are not finite numbers in each format (OFP8 rev. 1.0):
# E4M3 has NaN at S.1111.111; E5M2 has Inf at S.11111.00 and NaN above it.
_NON_FINITE = {0: (0x7F, 0xFF), 1: (0x7C, 0x7D, 0x7E, 0x7F, 0xFC, 0xFD, 0xFE, 0xFF)}


def fp8_codes(shape, fmt: int, seed: int) -> torch.Tensor:
    """uint8 tensor of uniform random finite codes of ``fmt``."""
    allowed = torch.tensor([c for c in range(256) if c not in _NON_FINITE[fmt]],
                           dtype=torch.uint8)
    i = torch.randint(0, len(allowed), tuple(shape), generator=_gen(seed))
    return allowed[i]


def bf16_bit_patterns() -> torch.Tensor:
    """Every one of the 65536 bf16 bit patterns, as a bf16 tensor."""
    return torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)


def f16_bit_patterns() -> torch.Tensor:
    """Every one of the 65536 fp16 bit patterns, as an fp16 tensor."""
    return torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(torch.float16)


def f32_mixed(n: int, seed: int) -> torch.Tensor:
    """fp32 tensor of n values spread over the whole fp32 range: normal draws
    scaled by 2^e with e ~ U{-140, ..., 130} (so subnormals, values that
    overflow any FP8 scale and everything between occur), random signs, and
    every 97th value replaced by one of +-0, +-inf, the smallest subnormal
    and the largest finite fp32."""
    g = _gen(seed)
    x = torch.randn(n, generator=g, dtype=torch.float64)
    e = torch.randint(-140, 131, (n,), generator=g).to(torch.float64)
    v = (x * torch.pow(2.0, e)).to(torch.float32)
    special = torch.tensor([0.0, -0.0, float("inf"), -float("inf"), 1.401298464324817e-45,
                            -1.401298464324817e-45, 3.4028234663852886e38, -3.4028234663852886e38],
                           dtype=torch.float32)
    idx = torch.arange(0, n, 97)
    v[idx] = special[torch.arange(len(idx)) % len(special)]
    return v


# ------------------------------------------------------------- workloads ---

SQUARE_SIZES = (1024, 2048, 4096, 8192)

SKINNY_SHAPES = ((64, 8192, 2048), (1024, 1536, 2048), (1, 4096, 4096), (8, 4096, 4096))

BATCHED = (
    # (batch, M, N, K, B broadcast)
    (64, 512, 512, 512, False),
    (8, 1024, 2048, 2048, True),
)

# linear stack: (name, d_in, d_out)
LINEARS = (("qkv", 1024, 3072), ("out", 1024, 1024),
           ("mlp_up", 1024, 4096), ("mlp_down", 4096, 1024))
TOKENS = 2048
STACK_STEPS = 8
X_STD, W_STD, G_STD = 0.02, 0.02, 1e-3


def stack_walk(steps: int = STACK_STEPS, seed: int = 2999):
    """Per tensor role and linear, the magnitude factors f_0 .. f_{steps-1}.

    f_0 = 1 and f_s = f_{s-1} * u_s with u_s ~ U(0.5, 2). Returns a dict
    keyed by (linear index, role) with role in {"x", "w", "g"}.
    """
    out = {}
    for li in range(len(LINEARS)):
        for ri, role in enumerate(("x", "w", "g")):
            u = uniform(0.5, 2.0, seed * 100 + li * 3 + ri, steps)
            f = [1.0]
            for s in range(1, steps):
                f.append(f[-1] * float(u[s]))
            out[(li, role)] = f
    return out


def stack_tensors(step: int, walk=None):
    """bf16 x, W, g of every linear at ``step`` (CPU tensors).

    Returns a list of dicts with keys x [T, d_in], w [d_out, d_in],
    g [T, d_out]. The draws use seed 1000*2 + 100*step + 3*linear + role,
    scaled by the walk factor of that tensor.
    """
    walk = stack_walk() if walk is None else walk
    out = []
    for li, (_, d_in, d_out) in enumerate(LINEARS):
        base = 2000 + 100 * step + 3 * li
        x = bf16_normal((TOKENS, d_in), X_STD * walk[(li, "x")][step], base + 0)
        w = bf16_normal((d_out, d_in), W_STD * walk[(li, "w")][step], base + 1)
        g = bf16_normal((TOKENS, d_out), G_STD * walk[(li, "g")][step], base + 2)
        out.append({"x": x, "w": w, "g": g})
    return out


def stack_flops() -> int:
    """FLOPs of one stack step: forward, dX and dW GEMMs of every linear."""
    return sum(3 * 2 * TOKENS * d_in * d_out for _, d_in, d_out in LINEARS)


def stack_quant_elems() -> int:
    """Elements quantized in one stack step (x, W and g of every linear)."""
    return sum(TOKENS * d_in + d_out * d_in + TOKENS * d_out for _, d_in, d_out in LINEARS)
