// Shared host/device helpers of the fp8lite library (sm_100a).
#pragma once

#include <cstdint>
#include <utility>

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

// Programmatic dependent launch: a kernel launched with launch_pdl() may
// start while the previous kernel on the stream is finishing; it must call
// griddep_wait() before its first access to memory another kernel writes or
// reads. griddep_launch() lets the next kernel start its own prologue early.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialization; cluster > 1 launches
// clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
inline fp8_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             int cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = unsigned(cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cluster > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// fmt_max / m in IEEE fp32 (round-to-nearest division), overflow clamped to
// FLT_MAX. Used by both the ring finalize and current scaling.
__device__ __forceinline__ float scale_from_amax(float fmax, float m) {
    float s = __fdiv_rn(fmax, m);
    return isinf(s) ? 3.402823466e38f : s;
}

// The delayed-scaling fold of amax `a` into a ring [fp8.py@4dc5e923, bullet
// on the last-block epilogue]: hist[idx] = a, idx advances, and the window's
// maximum (the 15 kept entries and a) publishes fmt_max / max when it is
// finite and > 0 (otherwise the scale is kept). hist and idx must be the
// values read by the caller (h[], idx), which lets it issue those reads
// early.
__device__ __forceinline__ void ring_fold(volatile fp8_ring* r, const float (&h)[FP8_RING_HISTORY], uint32_t idx,
                                          float a, float fmax) {
    float wmax = a;
#pragma unroll
    for (int i = 0; i < FP8_RING_HISTORY; ++i)
        if (uint32_t(i) != idx) wmax = fmaxf(wmax, h[i]);
    r->hist[idx] = a;
    if (wmax > 0.0f && isfinite(wmax)) r->scale = scale_from_amax(fmax, wmax);
    r->idx = (idx + 1) & (FP8_RING_HISTORY - 1);
}

// Atomic add with acquire-release semantics at GPU scope (the last-block
// election of a ring finalize: a block's earlier amax publication is visible
// before its ticket moves, and the block drawing the last ticket sees all).
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Reads a ring's history and index (for ring_fold).
__device__ __forceinline__ uint32_t ring_read(volatile fp8_ring* r, float (&h)[FP8_RING_HISTORY]) {
#pragma unroll
    for (int i = 0; i < FP8_RING_HISTORY; ++i) h[i] = r->hist[i];
    return r->idx & (FP8_RING_HISTORY - 1);
}

}  // namespace fp8lite
