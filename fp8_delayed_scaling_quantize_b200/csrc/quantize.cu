// Per-tensor FP8 quantization with amax reduction and the delayed-scaling
// ring finalized on the device (sm_100a).
//
// Method: AstrAI commit log astrai/extension/fp8.py @4dc5e923 -- the amax is
// taken over the unquantized input (bullets on the amax bug), and the quantize
// kernel's last thread block (threadfence + counter election) folds the amax
// into hist[idx], reduces the window and publishes the next scale with no
// extra launch (bullet on the last-block epilogue). The scale used by the call
// is returned separately because the finalize replaces the ring's scale
// (astrai/extension/fp8.py @f4c44ebf, bullet on the scale snapshot).
//
// Kernel design (HBM-bound, 3 bytes per element when delayed):
//  * each thread moves 8 bf16 (one 16-byte load) -> 8 codes (one 8-byte
//    store); a warp's load instruction covers 512 contiguous bytes and its
//    store 256 contiguous bytes; four such units are in flight per thread;
//  * x * s is one fp32 multiply (round-to-nearest, no flush-to-zero), then
//    the hardware pair conversion cvt.rn.satfinite.{e4m3x2,e5m2x2}.f32 does
//    the nearest-even FP8 rounding with saturation -- never through fp16;
//  * amax: fmaxf per thread (NaN is ignored), then warp redux.sync max on the
//    bit patterns (non-negative floats order like unsigned integers), a
//    shared-memory pass over the block's warps and one atomicMax per block;
//  * delayed: one launch; the block that draws the last ticket finalizes the
//    ring and resets its accumulator and ticket, so the ring is ready for the
//    next call (and for CUDA-graph replay) with no host involvement;
//  * current: memset of the caller's amax word, an amax-only pass, then the
//    quantize pass that derives the scale from that amax. For tensors that
//    fit in L2 the second read is served from L2.

#include <cuda_runtime.h>

#include "common.cuh"

namespace fp8lite {
namespace {

// 512-thread blocks: half as many blocks (and per-block atomics on the
// ring's cache line) as 256 would need, measured faster at 2-8 M elements.
constexpr int kThreads = 512;
constexpr int kUnroll = 4;  // 16-byte units in flight per thread

enum Mode { kDelayed = 0, kCurrentQuant = 1, kAmaxOnly = 2 };

template <int FMT>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi) {
    // The first source lands in the upper byte, the second in the lower one.
    uint16_t r;
    if (FMT == FP8_E4M3) {
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    } else {
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    }
    return r;
}

// bf16 is the upper half of an fp32: widening is a bit shift, exact for
// every value including subnormals.
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int FMT>
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float s, float& m) {
    const float a = bf_lo(w0), b = bf_hi(w0), c = bf_lo(w1), d = bf_hi(w1);
    m = fmaxf(m, fabsf(a));
    m = fmaxf(m, fabsf(b));
    m = fmaxf(m, fabsf(c));
    m = fmaxf(m, fabsf(d));
    const uint32_t lo = cvt_pair<FMT>(__fmul_rn(a, s), __fmul_rn(b, s));
    const uint32_t hi = cvt_pair<FMT>(__fmul_rn(c, s), __fmul_rn(d, s));
    return lo | (hi << 16);
}

__device__ __forceinline__ void amax4(uint32_t w0, uint32_t w1, float& m) {
    m = fmaxf(m, fabsf(bf_lo(w0)));
    m = fmaxf(m, fabsf(bf_hi(w0)));
    m = fmaxf(m, fabsf(bf_lo(w1)));
    m = fmaxf(m, fabsf(bf_hi(w1)));
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Block-wide max of a non-negative, non-NaN float; result valid in thread 0.
__device__ __forceinline__ uint32_t block_max_bits(float m) {
    __shared__ uint32_t warp_max[kThreads / 32];
    uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) warp_max[warp] = bits;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = lane < kThreads / 32 ? warp_max[lane] : 0u;
        bits = __reduce_max_sync(0xffffffffu, v);
    }
    return bits;
}

// The quantize pass of one tensor, run by block `blk` of the `nblk` blocks
// given to it (a whole grid for fp8_quantize, a share of one for
// fp8_quantize_many). s_scale is the block's shared scale slot.
template <int FMT, int MODE>
__device__ __forceinline__ void quantize_body(const uint16_t* __restrict__ x, int64_t n, uint8_t* __restrict__ out8,
                                              fp8_ring* ring, uint32_t* amax_acc, float* amax_out, float* scale_out,
                                              int blk, int nblk, float& s_scale) {
    const float fmax = fmt_max(FMT);
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    uint2* ov = reinterpret_cast<uint2*>(out8);
    const int64_t units = n >> 3;  // 8 elements per unit
    const int64_t tid = int64_t(blk) * kThreads + threadIdx.x;
    const int64_t stride = int64_t(nblk) * kThreads;
    // The first round of input loads leaves before the scale is known (the
    // loads do not need it); for tensors of up to 2048 elements per thread
    // of the grid that is every load.
    int64_t base = tid;
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * stride;
        if (i < units) v[u] = __ldg(xv + i);
    }
    // One thread per block reads the scale (or the amax it comes from) and
    // shares it: thousands of warps loading one address would queue on a
    // single L2 line.
    if (MODE != kAmaxOnly) {
        if (threadIdx.x == 0) {
            float v;
            if (MODE == kDelayed) {
                v = *reinterpret_cast<volatile float*>(&ring->scale);
            } else {
                const float a = __uint_as_float(*reinterpret_cast<volatile uint32_t*>(amax_acc));
                v = (a > 0.0f && isfinite(a)) ? scale_from_amax(fmax, a) : 1.0f;
            }
            s_scale = v;
            if (blk == 0) *scale_out = v;
        }
        __syncthreads();
    }
    const float s = MODE == kAmaxOnly ? 1.0f : s_scale;
    float m = 0.0f;

    while (base < units) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * stride;
            if (i < units) {
                if (MODE == kAmaxOnly) {
                    amax4(v[u].x, v[u].y, m);
                    amax4(v[u].z, v[u].w, m);
                } else {
                    uint2 q;
                    q.x = quant4<FMT>(v[u].x, v[u].y, s, m);
                    q.y = quant4<FMT>(v[u].z, v[u].w, s, m);
                    ov[i] = q;
                }
            }
        }
        base += stride * kUnroll;
        if (base >= units) break;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * stride;
            if (i < units) v[u] = __ldg(xv + i);
        }
    }
    griddep_launch();  // the next kernel may start its prologue
    // ragged tail (n mod 8 elements): one thread, scalar
    if (tid == 0) {
        for (int64_t i = units << 3; i < n; ++i) {
            const float a = __uint_as_float(uint32_t(x[i]) << 16);
            m = fmaxf(m, fabsf(a));
            if (MODE != kAmaxOnly) out8[i] = uint8_t(cvt_pair<FMT>(__fmul_rn(a, s), 0.0f));
        }
    }

    const uint32_t bits = block_max_bits(m);
    if (threadIdx.x != 0) return;
    uint32_t* acc = MODE == kDelayed ? &ring->amax_bits : amax_acc;
    if (bits != 0u) atomicMax(acc, bits);
    if (MODE != kDelayed) return;

    // Last-block election: every block publishes its amax, then takes a
    // ticket with acquire-release semantics (its amax is visible before the
    // ticket moves); the block holding the final ticket sees every amax.
    const uint32_t ticket = atom_add_acq_rel(&ring->ticket, 1u);
    if (ticket != uint32_t(nblk) - 1) return;
    // The history and its index change only in this finalize, so they are
    // read together with the exchange of the accumulated amax: the 18
    // accesses leave at once and cost one round trip to L2.
    volatile fp8_ring* r = ring;
    float h[FP8_RING_HISTORY];
#pragma unroll
    for (int i = 0; i < FP8_RING_HISTORY; ++i) h[i] = r->hist[i];
    const uint32_t idx = r->idx & (FP8_RING_HISTORY - 1);
    const float a = __uint_as_float(atomicExch(&ring->amax_bits, 0u));
    // the window's maximum over the 15 kept entries and the new amax
    float wmax = a;
#pragma unroll
    for (int i = 0; i < FP8_RING_HISTORY; ++i)
        if (uint32_t(i) != idx) wmax = fmaxf(wmax, h[i]);
    r->hist[idx] = a;
    if (wmax > 0.0f && isfinite(wmax)) r->scale = scale_from_amax(fmax, wmax);
    r->idx = (idx + 1) & (FP8_RING_HISTORY - 1);
    if (amax_out) *amax_out = a;
    r->ticket = 0u;  // ready for the next call (visible at the kernel boundary)
}

template <int FMT, int MODE>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const uint16_t* __restrict__ x, int64_t n, uint8_t* __restrict__ out8,
                fp8_ring* ring, uint32_t* amax_acc, float* amax_out, float* scale_out) {
    __shared__ float s_scale;
    griddep_wait();  // inputs and the ring come from earlier kernels
    quantize_body<FMT, MODE>(x, n, out8, ring, amax_acc, amax_out, scale_out, blockIdx.x, gridDim.x, s_scale);
}

// Several delayed-scaling quantizations in one launch: job j owns blocks
// [first[j], first[j] + blocks[j]) of the grid and runs exactly what
// fp8_quantize does for it, its ring finalized by the last of its blocks.
struct QuantJobs {
    int count;
    int first[FP8_QUANTIZE_MAX_JOBS];
    int blocks[FP8_QUANTIZE_MAX_JOBS];
    int fmt[FP8_QUANTIZE_MAX_JOBS];
    const uint16_t* x[FP8_QUANTIZE_MAX_JOBS];
    int64_t n[FP8_QUANTIZE_MAX_JOBS];
    fp8_ring* ring[FP8_QUANTIZE_MAX_JOBS];
    uint8_t* out8[FP8_QUANTIZE_MAX_JOBS];
    float* amax_out[FP8_QUANTIZE_MAX_JOBS];
    float* scale_out[FP8_QUANTIZE_MAX_JOBS];
};

__global__ void __launch_bounds__(kThreads) quantize_many_kernel(const __grid_constant__ QuantJobs jobs) {
    __shared__ float s_scale;
    griddep_wait();
    int j = 0;
    while (j + 1 < jobs.count && int(blockIdx.x) >= jobs.first[j + 1]) ++j;
    const int blk = int(blockIdx.x) - jobs.first[j];
    if (jobs.fmt[j] == FP8_E4M3)
        quantize_body<FP8_E4M3, kDelayed>(jobs.x[j], jobs.n[j], jobs.out8[j], jobs.ring[j], nullptr,
                                          jobs.amax_out[j], jobs.scale_out[j], blk, jobs.blocks[j], s_scale);
    else
        quantize_body<FP8_E5M2, kDelayed>(jobs.x[j], jobs.n[j], jobs.out8[j], jobs.ring[j], nullptr,
                                          jobs.amax_out[j], jobs.scale_out[j], blk, jobs.blocks[j], s_scale);
}

__global__ void ring_write_kernel(fp8_ring* ring, fp8_ring value) {
    griddep_wait();
    const int t = threadIdx.x;
    if (t < FP8_RING_HISTORY) ring->hist[t] = value.hist[t];
    if (t == 0) {
        ring->scale = value.scale;
        ring->idx = value.idx;
        ring->amax_bits = 0u;
        ring->ticket = 0u;
    }
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        cached[dev] = c;
    }
    return cached[dev];
}

int grid_for(int64_t n) {
    const int64_t units = n >> 3;
    const int64_t want = (units + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
    const int64_t cap = int64_t(sm_count()) * (2048 / kThreads);
    int64_t g = want < cap ? want : cap;
    return int(g < 1 ? 1 : g);
}

template <int FMT>
fp8_status launch_quantize(const uint16_t* x, int64_t n, fp8_ring* ring, uint8_t* out8,
                           float* amax_out, float* scale_out, cudaStream_t st) {
    const int grid = grid_for(n);
    if (ring)
        return launch_pdl(quantize_kernel<FMT, kDelayed>, grid, kThreads, 0, st, 1, x, n, out8, ring,
                          (uint32_t*)nullptr, amax_out, scale_out);
    uint32_t* acc = reinterpret_cast<uint32_t*>(amax_out);
    if (cudaMemsetAsync(acc, 0, sizeof(uint32_t), st) != cudaSuccess) return FP8_ERR_CUDA;
    if (launch_pdl(quantize_kernel<FMT, kAmaxOnly>, grid, kThreads, 0, st, 1, x, n, out8, (fp8_ring*)nullptr, acc,
                   (float*)nullptr, (float*)nullptr) != FP8_OK)
        return FP8_ERR_CUDA;
    return launch_pdl(quantize_kernel<FMT, kCurrentQuant>, grid, kThreads, 0, st, 1, x, n, out8, (fp8_ring*)nullptr,
                      acc, (float*)nullptr, scale_out);
}

bool scale_ok(float s) { return s > 0.0f && s <= 3.402823466e38f; }

}  // namespace
}  // namespace fp8lite

using namespace fp8lite;

extern "C" const char* fp8_status_string(fp8_status s) {
    switch (s) {
        case FP8_OK: return "FP8_OK";
        case FP8_ERR_INVALID_ARG: return "FP8_ERR_INVALID_ARG";
        case FP8_ERR_ALIGNMENT: return "FP8_ERR_ALIGNMENT";
        case FP8_ERR_UNSUPPORTED: return "FP8_ERR_UNSUPPORTED";
        case FP8_ERR_CUDA: return "FP8_ERR_CUDA";
        case FP8_ERR_DEVICE_TIMEOUT: return "FP8_ERR_DEVICE_TIMEOUT";
    }
    return "FP8_ERR_UNKNOWN";
}

extern "C" int fp8_abi_version(void) { return FP8LITE_ABI_VERSION; }

extern "C" fp8_status fp8_ring_init(fp8_ring* ring, float init_scale, void* stream) {
    if (!ring) return FP8_ERR_INVALID_ARG;
    if (!aligned(ring, 4)) return FP8_ERR_ALIGNMENT;
    if (!scale_ok(init_scale)) return FP8_ERR_INVALID_ARG;
    fp8_ring v = {};
    v.scale = init_scale;
    ring_write_kernel<<<1, 32, 0, as_stream(stream)>>>(ring, v);
    return launch_status();
}

extern "C" fp8_status fp8_ring_get(const fp8_ring* ring, fp8_ring* host, void* stream) {
    if (!ring || !host) return FP8_ERR_INVALID_ARG;
    if (!aligned(ring, 4)) return FP8_ERR_ALIGNMENT;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(host, ring, sizeof(fp8_ring), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return FP8_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_ring_set(fp8_ring* ring, const fp8_ring* host, void* stream) {
    if (!ring || !host) return FP8_ERR_INVALID_ARG;
    if (!aligned(ring, 4)) return FP8_ERR_ALIGNMENT;
    if (host->idx >= FP8_RING_HISTORY || !scale_ok(host->scale)) return FP8_ERR_INVALID_ARG;
    ring_write_kernel<<<1, 32, 0, as_stream(stream)>>>(ring, *host);
    return launch_status();
}

extern "C" fp8_status fp8_quantize(const void* x, int64_t n, fp8_fmt fmt, fp8_ring* ring, uint8_t* out8,
                                   float* amax_out, float* scale_out, void* stream) {
    if (!valid_fmt(fmt)) return FP8_ERR_INVALID_ARG;
    if (n < 0 || n >= (int64_t(1) << 40)) return FP8_ERR_INVALID_ARG;
    if (!scale_out) return FP8_ERR_INVALID_ARG;
    if (n > 0 && (!x || !out8)) return FP8_ERR_INVALID_ARG;
    if (!ring && !amax_out) return FP8_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out8, 16)) return FP8_ERR_ALIGNMENT;
    if (ring && !aligned(ring, 4)) return FP8_ERR_ALIGNMENT;
    if (!aligned(scale_out, 4) || !aligned(amax_out, 4)) return FP8_ERR_ALIGNMENT;
    const uint16_t* xb = static_cast<const uint16_t*>(x);
    cudaStream_t st = as_stream(stream);
    return fmt == FP8_E4M3 ? launch_quantize<FP8_E4M3>(xb, n, ring, out8, amax_out, scale_out, st)
                           : launch_quantize<FP8_E5M2>(xb, n, ring, out8, amax_out, scale_out, st);
}

extern "C" fp8_status fp8_quantize_many(const fp8_quantize_job* jobs, int32_t count, void* stream) {
    if (!jobs || count < 1 || count > FP8_QUANTIZE_MAX_JOBS) return FP8_ERR_INVALID_ARG;
    QuantJobs q = {};
    q.count = count;
    int total = 0;
    for (int j = 0; j < count; ++j) {
        const fp8_quantize_job& in = jobs[j];
        if (!valid_fmt(in.fmt)) return FP8_ERR_INVALID_ARG;
        if (in.n < 0 || in.n >= (int64_t(1) << 40)) return FP8_ERR_INVALID_ARG;
        if (!in.ring || !in.scale_out) return FP8_ERR_INVALID_ARG;
        if (in.n > 0 && (!in.x || !in.out8)) return FP8_ERR_INVALID_ARG;
        if (!aligned(in.x, 16) || !aligned(in.out8, 16)) return FP8_ERR_ALIGNMENT;
        if (!aligned(in.ring, 4) || !aligned(in.scale_out, 4) || !aligned(in.amax_out, 4)) return FP8_ERR_ALIGNMENT;
        for (int k = 0; k < j; ++k)
            if (jobs[k].ring == in.ring) return FP8_ERR_INVALID_ARG;  // one ring, one call at a time
        q.first[j] = total;
        q.blocks[j] = grid_for(in.n);
        total += q.blocks[j];
        q.fmt[j] = int(in.fmt);
        q.x[j] = static_cast<const uint16_t*>(in.x);
        q.n[j] = in.n;
        q.ring[j] = in.ring;
        q.out8[j] = in.out8;
        q.amax_out[j] = in.amax_out;
        q.scale_out[j] = in.scale_out;
    }
    return launch_pdl(quantize_many_kernel, total, kThreads, 0, as_stream(stream), 1, q);
}
