"""FP8 training linear layer on the fp8lite C ABI (torch.autograd).

After the AstrAI commit logs (``astrai/extension/fp8.py`` @4dc5e923 and
@f4c44ebf):

* a linear layer owns three delayed-scaling rings, for x, W and the output
  gradient g (bullet on the three _ScaleRing objects per linear);
* forward quantizes x and W to E4M3 and computes y = x W^T (+ bias fused in
  the GEMM epilogue); backward quantizes g to E5M2 and computes dX = g W and
  dW = g^T x with the scales the forward used (bullets on carrying the
  forward's scale to backward and on the scale snapshot);
* backward reads only what forward saved, so it runs in FP8 wherever it is
  called (bullet on the autograd Function owning the forward/backward pair);
* gradients are bf16; the bias gradient is the column sum of the bf16 g over
  the flattened leading dimensions, computed only when the bias needs a
  gradient (bullets on the conditional column sum and the 3-D backward).

Every computation runs in the library's CUDA kernels; torch provides the
buffers and the stream. The forward saves the FP8 codes of x and W (one byte
per element) rather than the bf16 tensors. The rings are a registered buffer
(`fp8_rings`, three 80-byte rings), so they travel with the module's
state_dict for checkpoint and resume.
"""

import torch

from . import (FP8_E4M3, FP8_E5M2, FP8_NN, FP8_NT, FP8_RING_BYTES, FP8_TN, fp8_bias_grad, fp8_mm, fp8_mm_grouped,
               fp8_quantize, fp8_quantize_many, fp8_ring_init)

_RING_WORDS = FP8_RING_BYTES // 4


def _quantize(t, n, fmt, ring):
    q = torch.empty(n, dtype=torch.uint8, device=t.device)
    amax = torch.empty(1, dtype=torch.float32, device=t.device)
    scale = torch.empty(1, dtype=torch.float32, device=t.device)
    fp8_quantize(t, n, fmt, ring, q, amax, scale)
    return q, scale


class Fp8LinearFunction(torch.autograd.Function):
    """y = x W^T + b with FP8 operands and delayed scaling (three rings)."""

    @staticmethod
    def forward(ctx, x, weight, bias, rings):
        N, K = weight.shape
        if x.shape[-1] != K:
            raise ValueError(f"input features {x.shape[-1]} != weight's {K}")
        if x.dtype != torch.bfloat16 or weight.dtype != torch.bfloat16:
            raise TypeError("Fp8Linear takes bf16 inputs and weights")
        x2 = x.reshape(-1, K).contiguous()
        w = weight.contiguous()
        T = x2.shape[0]
        # x and W in one quantize launch (each with its own ring)
        dev = x.device
        x8 = torch.empty(T * K, dtype=torch.uint8, device=dev)
        w8 = torch.empty(N * K, dtype=torch.uint8, device=dev)
        stats = torch.empty(4, dtype=torch.float32, device=dev)  # amax x, amax W, scale x, scale W
        amax_x, amax_w, sx, sw = stats[0:1], stats[1:2], stats[2:3], stats[3:4]
        fp8_quantize_many([(x2, T * K, FP8_E4M3, rings[0], x8, amax_x, sx),
                           (w, N * K, FP8_E4M3, rings[1], w8, amax_w, sw)])
        y = torch.empty(T, N, dtype=torch.bfloat16, device=x.device)
        b = bias.contiguous() if bias is not None else None
        fp8_mm(x8, FP8_E4M3, w8, FP8_E4M3, sx, sw, FP8_NT, T, N, K, 1, 0, 0, 0, b, None, 0, y)
        ctx.save_for_backward(x8, w8, sx, sw, rings)
        ctx.dims = (T, N, K)
        ctx.x_shape = x.shape
        ctx.has_bias = bias is not None
        return y.reshape(*x.shape[:-1], N)

    @staticmethod
    def backward(ctx, gy):
        x8, w8, sx, sw, rings = ctx.saved_tensors
        T, N, K = ctx.dims
        need_x, need_w, need_b = ctx.needs_input_grad[0], ctx.needs_input_grad[1], ctx.needs_input_grad[2]
        g2 = gy.reshape(-1, N).to(torch.bfloat16).contiguous()
        dx = dw = db = None
        if need_x or need_w:
            g8, sg = _quantize(g2, T * N, FP8_E5M2, rings[2])
            # dX = g W: A = g [T, N], B = W [N, K] (K-major rows of B are W's rows)
            # dW = g^T x: A = g [T, N] read MN-major, B = x [T, K]
            probs = []
            if need_x:
                dx = torch.empty(T, K, dtype=torch.bfloat16, device=gy.device)
                probs.append((g8, FP8_E5M2, w8, FP8_E4M3, sg, sw, FP8_NN, T, K, N, None, None, 0, dx))
            if need_w:
                dw = torch.empty(N, K, dtype=torch.bfloat16, device=gy.device)
                probs.append((g8, FP8_E5M2, x8, FP8_E4M3, sg, sx, FP8_TN, N, K, T, None, None, 0, dw))
            if len(probs) == 2:  # both read only g8: one launch shares the grid
                fp8_mm_grouped(probs)
            else:
                a8, fa, b8, fb, sa, sb, layout, M, Nn, Kk, _, _, _, out = probs[0]
                fp8_mm(a8, fa, b8, fb, sa, sb, layout, M, Nn, Kk, 1, 0, 0, 0, None, None, 0, out)
            if need_x:
                dx = dx.reshape(ctx.x_shape)
        if ctx.has_bias and need_b:
            db = torch.empty(N, dtype=torch.bfloat16, device=gy.device)
            fp8_bias_grad(g2, T, N, db)
        return dx, dw, db, None


class Fp8Linear(torch.nn.Module):
    """Drop-in training linear layer (bf16 parameters, FP8 compute).

    in_features and out_features must be multiples of 16 (the GEMMs read
    every operand through 16-byte-aligned rows).
    """

    def __init__(self, in_features, out_features, bias=True, device=None):
        super().__init__()
        if in_features % 16 or out_features % 16:
            raise ValueError("Fp8Linear needs in_features and out_features divisible by 16")
        self.in_features, self.out_features = in_features, out_features
        kw = {"device": device, "dtype": torch.bfloat16}
        self.weight = torch.nn.Parameter(torch.empty(out_features, in_features, **kw))
        self.bias = torch.nn.Parameter(torch.zeros(out_features, **kw)) if bias else None
        self.register_buffer("fp8_rings", torch.zeros(3, _RING_WORDS, dtype=torch.int32, device=device))
        self._rings_ready = False
        torch.nn.init.normal_(self.weight, std=in_features ** -0.5)

    def reset_scaling(self):
        """Reset the three rings (scale 1, empty history)."""
        for i in range(3):
            fp8_ring_init(self.fp8_rings[i], 1.0)
        self._rings_ready = True

    def _load_from_state_dict(self, *args, **kwargs):
        super()._load_from_state_dict(*args, **kwargs)
        self._rings_ready = True  # restored rings are used as they are

    def forward(self, x):
        if not self._rings_ready:
            self.reset_scaling()
        return Fp8LinearFunction.apply(x, self.weight, self.bias, self.fp8_rings)
