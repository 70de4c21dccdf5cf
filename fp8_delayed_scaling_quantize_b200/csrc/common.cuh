// Shared host/device helpers of the fp8lite library (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fp8lite.h"

namespace fp8lite {

// Largest finite magnitudes of the two OFP8 encodings.
constexpr float kE4M3Max = 448.0f;
constexpr float kE5M2Max = 57344.0f;

__host__ __device__ inline float fmt_max(int fmt) { return fmt == FP8_E4M3 ? kE4M3Max : kE5M2Max; }

inline bool valid_fmt(int f) { return f == FP8_E4M3 || f == FP8_E5M2; }

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Launch-error check after a kernel launch: a failed launch maps to FP8_ERR_CUDA.
inline fp8_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// fmt_max / m in IEEE fp32 (round-to-nearest division), overflow clamped to
// FLT_MAX. Used by both the ring finalize and current scaling.
__device__ __forceinline__ float scale_from_amax(float fmax, float m) {
    float s = __fdiv_rn(fmax, m);
    return isinf(s) ? 3.402823466e38f : s;
}

}  // namespace fp8lite
