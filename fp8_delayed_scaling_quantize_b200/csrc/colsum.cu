// Bias gradient of a linear layer: the column sums of the bf16 output
// gradient g [rows, cols], accumulated in fp32 and rounded once to bf16.
//
// Method: AstrAI commit log astrai/extension/fp8.py @f4c44ebf -- the bias
// gradient is the sum of g over the leading (token) dimensions, and it is
// computed only when the bias actually needs a gradient (bullet on the
// column-sum that ran unconditionally); 3-D inputs are flattened first
// (bullet on the [B, L, d] backward fix). The gradient is taken from the bf16
// g, not from its FP8 codes (bullet on dequantizing a pre-quantized g before
// the bias sum).
//
// Layout: one block per 64-column strip, walking every row, so each column's
// sum is finished inside one block (one rounding, no workspace). A warp reads
// 64 adjacent columns of a row as 32 bf16x2 words (128 contiguous bytes), its
// 8 warps walk rows 8 apart with four rows in flight, and the 8 partial sums
// of each column meet in shared memory.

#include <cuda_runtime.h>

#include "common.cuh"

namespace fp8lite {
namespace {

constexpr int kColsPerBlock = 64;
constexpr int kWarps = 8;

__global__ void __launch_bounds__(32 * kWarps)
colsum_kernel(const uint32_t* __restrict__ g, int64_t rows, int64_t cols, uint16_t* __restrict__ out) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t col = int64_t(blockIdx.x) * kColsPerBlock + 2 * lane;  // this thread's two columns
    const int64_t words_per_row = cols >> 1;                             // cols is even
    float s0 = 0.0f, s1 = 0.0f;
    if (col < cols) {
        const uint32_t* p = g + (col >> 1);
        int64_t r = warp;
        // four rows in flight per thread
        for (; r + 3 * kWarps < rows; r += 4 * kWarps) {
            const uint32_t w0 = __ldg(p + (r + 0 * kWarps) * words_per_row);
            const uint32_t w1 = __ldg(p + (r + 1 * kWarps) * words_per_row);
            const uint32_t w2 = __ldg(p + (r + 2 * kWarps) * words_per_row);
            const uint32_t w3 = __ldg(p + (r + 3 * kWarps) * words_per_row);
            s0 += __uint_as_float(w0 << 16);
            s1 += __uint_as_float(w0 & 0xFFFF0000u);
            s0 += __uint_as_float(w1 << 16);
            s1 += __uint_as_float(w1 & 0xFFFF0000u);
            s0 += __uint_as_float(w2 << 16);
            s1 += __uint_as_float(w2 & 0xFFFF0000u);
            s0 += __uint_as_float(w3 << 16);
            s1 += __uint_as_float(w3 & 0xFFFF0000u);
        }
        for (; r < rows; r += kWarps) {
            const uint32_t w = __ldg(p + r * words_per_row);
            s0 += __uint_as_float(w << 16);
            s1 += __uint_as_float(w & 0xFFFF0000u);
        }
    }
    __shared__ float part[kWarps][kColsPerBlock];
    part[warp][2 * lane] = s0;
    part[warp][2 * lane + 1] = s1;
    __syncthreads();
    griddep_launch();
    if (threadIdx.x < kColsPerBlock) {
        const int64_t c = int64_t(blockIdx.x) * kColsPerBlock + threadIdx.x;
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += part[w][threadIdx.x];
        if (c < cols) {
            uint16_t h;
            asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(s));
            out[c] = h;
        }
    }
}

}  // namespace
}  // namespace fp8lite

using namespace fp8lite;

extern "C" fp8_status fp8_bias_grad(const void* g, int64_t rows, int64_t cols, void* out, void* stream) {
    if (!g || !out) return FP8_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || rows >= (int64_t(1) << 40) || cols >= (int64_t(1) << 31)) return FP8_ERR_INVALID_ARG;
    if (cols % 2 != 0) return FP8_ERR_ALIGNMENT;
    if (!aligned(g, 4) || !aligned(out, 2)) return FP8_ERR_ALIGNMENT;
    const int blocks = int((cols + kColsPerBlock - 1) / kColsPerBlock);
    return launch_pdl(colsum_kernel, blocks, 32 * kWarps, 0, as_stream(stream), 1, static_cast<const uint32_t*>(g),
                      rows, cols, static_cast<uint16_t*>(out));
}
