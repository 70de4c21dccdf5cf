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
//    fit in L2 the second read is served from L2. A bf16 / fp16 tensor of
//    up to 65536 elements takes one launch instead: one 1024-thread block
//    holds it in registers, reduces the amax, derives the scale and
//    converts; up to 8 such tensors share one launch, a block each
//    (fp8_quantize_current_many);
//  * seeded delayed call: the current-scaling passes, then block 0 folds the
//    measured amax into the ring (astrai/extension/fp8.py @4dc5e923, bullet
//    on the _ScaleRing objects with their update and seed);
//  * inputs bf16, fp16 or fp32 (astrai/extension/fp8.py @f4c44ebf, bullet on
//    the quantize kernel templated on the input type): every value widens to
//    fp32 exactly; a unit is 8 elements (16 bytes of bf16/fp16, 32 of fp32).

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace fp8lite {
namespace {

// 512-thread blocks: half as many blocks (and per-block atomics on the
// ring's cache line) as 256 would need, measured faster at 2-8 M elements.
constexpr int kThreads = 512;
constexpr int kUnroll = 4;  // 16-byte units in flight per thread

// kDeferred: a delayed call whose fold is left to fp8_rings_fold, so that the
// ranks of a data-parallel group can first all-reduce the ring's amax.
enum Mode { kDelayed = 0, kCurrentQuant = 1, kAmaxOnly = 2, kSeed = 3, kDeferred = 4 };

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

// Eight consecutive input elements: 16 bytes of bf16 / fp16, 32 of fp32.
struct Unit {
    uint4 a, b;
};

template <int IN>
__device__ __forceinline__ void load_unit(const void* x, int64_t i, Unit& u) {
    if (IN == FP8_IN_F32) {
        const uint4* p = static_cast<const uint4*>(x) + 2 * i;
        u.a = __ldg(p);
        u.b = __ldg(p + 1);
    } else {
        u.a = __ldg(static_cast<const uint4*>(x) + i);
    }
}

__device__ __forceinline__ float h_lo(uint32_t w) { return __half2float(__ushort_as_half(uint16_t(w & 0xFFFFu))); }
__device__ __forceinline__ float h_hi(uint32_t w) { return __half2float(__ushort_as_half(uint16_t(w >> 16))); }

// The unit's values in fp32 (exact for all three input types).
template <int IN>
__device__ __forceinline__ void unit_f32(const Unit& u, float (&f)[8]) {
    const uint32_t w[4] = {u.a.x, u.a.y, u.a.z, u.a.w};
    if (IN == FP8_IN_BF16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = bf_lo(w[i]);
            f[2 * i + 1] = bf_hi(w[i]);
        }
    } else if (IN == FP8_IN_F16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = h_lo(w[i]);
            f[2 * i + 1] = h_hi(w[i]);
        }
    } else {
        const uint32_t v[4] = {u.b.x, u.b.y, u.b.z, u.b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[i] = __uint_as_float(w[i]);
            f[4 + i] = __uint_as_float(v[i]);
        }
    }
}

template <int IN>
__device__ __forceinline__ float load_elem(const void* x, int64_t i) {
    if (IN == FP8_IN_BF16) return __uint_as_float(uint32_t(static_cast<const uint16_t*>(x)[i]) << 16);
    if (IN == FP8_IN_F16) return __half2float(static_cast<const __half*>(x)[i]);
    return static_cast<const float*>(x)[i];
}

template <int FMT>
__device__ __forceinline__ uint2 quant8(const float (&f)[8], float s, float& m) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = cvt_pair<FMT>(__fmul_rn(f[2 * i], s), __fmul_rn(f[2 * i + 1], s));
    return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
}

__device__ __forceinline__ void amax8(const float (&f)[8], float& m) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
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

// The end of a block's pass: its amax goes to the accumulator (amax pass,
// delayed call), and the ring is finalized by the last block of a delayed call
// or by block 0 of a seeded call. m: this thread's amax.
template <int FMT, int MODE>
__device__ __forceinline__ void finish_block(float m, fp8_ring* ring, uint32_t* amax_acc, float* amax_out, int blk,
                                             int nblk) {
    const float fmax = fmt_max(FMT);
    // the quantize pass of current scaling (and of a seeded call) already
    // knows the amax: it came from the amax pass
    if (MODE == kCurrentQuant) return;
    if (MODE == kSeed) {
        if (blk != 0 || threadIdx.x != 0) return;  // block 0 folds the amax into the ring
    } else {
        constexpr bool kRing = MODE == kDelayed || MODE == kDeferred;
        const uint32_t bits = block_max_bits(m);
        if (threadIdx.x != 0) return;
        uint32_t* acc = kRing ? &ring->amax_bits : amax_acc;
        if (bits != 0u) atomicMax(acc, bits);
        if (!kRing) return;
        // Last-block election: every block publishes its amax, then takes a
        // ticket with acquire-release semantics (its amax is visible before
        // the ticket moves); the block holding the final ticket sees every
        // amax.
        const uint32_t ticket = atom_add_acq_rel(&ring->ticket, 1u);
        if (ticket != uint32_t(nblk) - 1) return;
        if (MODE == kDeferred) {  // the accumulator keeps this call's amax for the exchange and the fold
            if (amax_out) *amax_out = __uint_as_float(*reinterpret_cast<volatile uint32_t*>(&ring->amax_bits));
            reinterpret_cast<volatile fp8_ring*>(ring)->ticket = 0u;
            return;
        }
    }
    // The history and its index change only in this finalize, so they are
    // read together with the exchange of the accumulated amax: the 18
    // accesses leave at once and cost one round trip to L2.
    volatile fp8_ring* r = ring;
    float h[FP8_RING_HISTORY];
    const uint32_t idx = ring_read(r, h);
    const float a = MODE == kDelayed ? __uint_as_float(atomicExch(&ring->amax_bits, 0u))
                                     : __uint_as_float(*reinterpret_cast<volatile uint32_t*>(amax_acc));
    ring_fold(r, h, idx, a, fmax);
    if (MODE == kDelayed) {
        if (amax_out) *amax_out = a;
        r->ticket = 0u;  // ready for the next call (visible at the kernel boundary)
    }
}

// The scale a quantize pass uses, read by one thread per block and shared
// (thousands of warps loading one address would queue on a single L2 line):
// the ring's for a delayed call, fmt_max / amax from the amax pass otherwise.
// Block 0 also reports it in scale_out.
template <int FMT, int MODE>
__device__ __forceinline__ float read_scale(fp8_ring* ring, uint32_t* amax_acc, float* scale_out, int blk,
                                            float& s_scale) {
    if (threadIdx.x == 0) {
        float v;
        if (MODE == kDelayed || MODE == kDeferred) {
            v = *reinterpret_cast<volatile float*>(&ring->scale);
        } else {  // current scaling, also the seeded call: from the measured amax
            const float a = __uint_as_float(*reinterpret_cast<volatile uint32_t*>(amax_acc));
            v = (a > 0.0f && isfinite(a)) ? scale_from_amax(fmt_max(FMT), a) : 1.0f;
        }
        s_scale = v;
        if (blk == 0) *scale_out = v;
    }
    __syncthreads();
    return s_scale;
}

// The quantize pass of one tensor, run by block `blk` of the `nblk` blocks
// given to it (a whole grid for fp8_quantize, a share of one for
// fp8_quantize_many). s_scale is the block's shared scale slot.
template <int FMT, int MODE, int IN>
__device__ __forceinline__ void quantize_body(const void* __restrict__ x, int64_t n, uint8_t* __restrict__ out8,
                                              fp8_ring* ring, uint32_t* amax_acc, float* amax_out, float* scale_out,
                                              int blk, int nblk, float& s_scale) {
    // units in flight per thread: 64 bytes of input whatever the type
    constexpr int U = IN == FP8_IN_F32 ? kUnroll / 2 : kUnroll;
    uint2* ov = reinterpret_cast<uint2*>(out8);
    const int64_t units = n >> 3;  // 8 elements per unit
    const int64_t tid = int64_t(blk) * kThreads + threadIdx.x;
    const int64_t stride = int64_t(nblk) * kThreads;
    // The first round of input loads leaves before the scale is known (the
    // loads do not need it); for tensors of up to 2048 elements per thread
    // of the grid that is every load.
    int64_t base = tid;
    Unit v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = base + u * stride;
        if (i < units) load_unit<IN>(x, i, v[u]);
    }
    const float s = MODE == kAmaxOnly ? 1.0f : read_scale<FMT, MODE>(ring, amax_acc, scale_out, blk, s_scale);
    float m = 0.0f;

    while (base < units) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * stride;
            if (i < units) {
                float f[8];
                unit_f32<IN>(v[u], f);
                if (MODE == kAmaxOnly) amax8(f, m);
                else                   ov[i] = quant8<FMT>(f, s, m);
            }
        }
        base += stride * U;
        if (base >= units) break;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * stride;
            if (i < units) load_unit<IN>(x, i, v[u]);
        }
    }
    griddep_launch();  // the next kernel may start its prologue
    // ragged tail (n mod 8 elements): one thread, scalar
    if (tid == 0) {
        for (int64_t i = units << 3; i < n; ++i) {
            const float a = load_elem<IN>(x, i);
            m = fmaxf(m, fabsf(a));
            if (MODE != kAmaxOnly) out8[i] = uint8_t(cvt_pair<FMT>(__fmul_rn(a, s), 0.0f));
        }
    }

    finish_block<FMT, MODE>(m, ring, amax_acc, amax_out, blk, nblk);
}

template <int FMT, int MODE, int IN>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const void* __restrict__ x, int64_t n, uint8_t* __restrict__ out8,
                fp8_ring* ring, uint32_t* amax_acc, float* amax_out, float* scale_out) {
    __shared__ float s_scale;
    griddep_wait();  // inputs and the ring come from earlier kernels
    quantize_body<FMT, MODE, IN>(x, n, out8, ring, amax_acc, amax_out, scale_out, blockIdx.x, gridDim.x, s_scale);
}

// Current scaling of a small tensor in one launch: one block of 1024 threads
// holds every 8-element unit in registers, reduces the amax, derives the
// scale and converts, so the call needs neither the accumulator memset nor a
// second pass over the input (the same arithmetic as the two-pass path, so
// the same codes, amax and scale). bf16 / fp16 inputs of up to 65536
// elements.
constexpr int kSmallThreads = 1024;
constexpr int kSmallUnits = 8;  // units per thread
constexpr int64_t kSmallMax = int64_t(kSmallThreads) * kSmallUnits * 8;

template <int FMT, int IN>
__device__ __forceinline__ void small_current_body(const void* __restrict__ x, int64_t n, uint8_t* __restrict__ out8,
                                                   float* amax_out, float* scale_out, uint32_t (&warp_max)[32],
                                                   float& s_scale) {
    static_assert(IN != FP8_IN_F32, "fp32 units do not fit the registers of a 1024-thread block");
    const int64_t units = n >> 3;
    const int tail = int(n - (units << 3));
    Unit v[kSmallUnits];
#pragma unroll
    for (int k = 0; k < kSmallUnits; ++k) {
        const int64_t i = threadIdx.x + int64_t(k) * kSmallThreads;
        if (i < units) load_unit<IN>(x, i, v[k]);
    }
    float t[7];
    float m = 0.0f;
    if (threadIdx.x == 0) {
        for (int j = 0; j < tail; ++j) {
            t[j] = load_elem<IN>(x, (units << 3) + j);
            m = fmaxf(m, fabsf(t[j]));
        }
    }
#pragma unroll
    for (int k = 0; k < kSmallUnits; ++k) {
        const int64_t i = threadIdx.x + int64_t(k) * kSmallThreads;
        if (i < units) {
            float f[8];
            unit_f32<IN>(v[k], f);
            amax8(f, m);
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
    if (lane == 0) warp_max[warp] = bits;
    __syncthreads();
    if (warp == 0) {
        bits = __reduce_max_sync(0xffffffffu, warp_max[lane]);
        if (lane == 0) {
            const float a = __uint_as_float(bits);
            const float sc = (a > 0.0f && isfinite(a)) ? scale_from_amax(fmt_max(FMT), a) : 1.0f;
            s_scale = sc;
            if (amax_out) *amax_out = a;
            *scale_out = sc;
        }
    }
    __syncthreads();
    const float s = s_scale;
    griddep_launch();
    uint2* ov = reinterpret_cast<uint2*>(out8);
#pragma unroll
    for (int k = 0; k < kSmallUnits; ++k) {
        const int64_t i = threadIdx.x + int64_t(k) * kSmallThreads;
        if (i < units) {
            float f[8], unused = 0.0f;
            unit_f32<IN>(v[k], f);
            ov[i] = quant8<FMT>(f, s, unused);
        }
    }
    if (threadIdx.x == 0)
        for (int j = 0; j < tail; ++j) out8[(units << 3) + j] = uint8_t(cvt_pair<FMT>(__fmul_rn(t[j], s), 0.0f));
}

template <int FMT, int IN>
__global__ void __launch_bounds__(kSmallThreads)
quantize_small_current_kernel(const void* __restrict__ x, int64_t n, uint8_t* __restrict__ out8, float* amax_out,
                              float* scale_out) {
    __shared__ uint32_t warp_max[kSmallThreads / 32];
    __shared__ float s_scale;
    griddep_wait();
    small_current_body<FMT, IN>(x, n, out8, amax_out, scale_out, warp_max, s_scale);
}

// Current scaling of up to FP8_QUANTIZE_MAX_JOBS small tensors in one
// launch: block j runs job j exactly as quantize_small_current_kernel runs a
// single tensor (so the same codes, amax and scale).
struct SmallJobs {
    const void* x[FP8_QUANTIZE_MAX_JOBS];
    int64_t n[FP8_QUANTIZE_MAX_JOBS];
    uint8_t* out8[FP8_QUANTIZE_MAX_JOBS];
    float* amax_out[FP8_QUANTIZE_MAX_JOBS];
    float* scale_out[FP8_QUANTIZE_MAX_JOBS];
    int kind[FP8_QUANTIZE_MAX_JOBS];  // 2 * fmt + dtype (bf16 or fp16)
};

__global__ void __launch_bounds__(kSmallThreads) quantize_small_current_many_kernel(const __grid_constant__ SmallJobs q) {
    __shared__ uint32_t warp_max[kSmallThreads / 32];
    __shared__ float s_scale;
    griddep_wait();
    const int j = blockIdx.x;
    switch (q.kind[j]) {
        case 2 * FP8_E4M3 + FP8_IN_BF16:
            small_current_body<FP8_E4M3, FP8_IN_BF16>(q.x[j], q.n[j], q.out8[j], q.amax_out[j], q.scale_out[j],
                                                      warp_max, s_scale);
            break;
        case 2 * FP8_E4M3 + FP8_IN_F16:
            small_current_body<FP8_E4M3, FP8_IN_F16>(q.x[j], q.n[j], q.out8[j], q.amax_out[j], q.scale_out[j],
                                                     warp_max, s_scale);
            break;
        case 2 * FP8_E5M2 + FP8_IN_BF16:
            small_current_body<FP8_E5M2, FP8_IN_BF16>(q.x[j], q.n[j], q.out8[j], q.amax_out[j], q.scale_out[j],
                                                      warp_max, s_scale);
            break;
        default:
            small_current_body<FP8_E5M2, FP8_IN_F16>(q.x[j], q.n[j], q.out8[j], q.amax_out[j], q.scale_out[j],
                                                     warp_max, s_scale);
            break;
    }
}

// Quantize of a [rows, cols] tensor that also writes the transposed codes
// [cols, rows] (LAYOUT FP8_QL_COL: only those; FP8_QL_BOTH: both, from one read
// of the input). A block walks 128 x 64 tiles (rows x columns): each thread
// quantizes two 8-element units of a row (rows lr and lr + 64, exactly as the
// flat kernel does, so both orientations hold the same bytes), writes them to
// the row-major codes, and drops their codes into a shared-memory tile held
// column-major; after a barrier each thread reads 16 consecutive codes of one
// tile column (16 consecutive rows of one input column) and writes them to the
// transposed codes. The next tile's loads leave before the current tile is
// processed. rows and cols are multiples of 8.
constexpr int kTileR = 128, kTileC = 64;
constexpr int kTileStride = kTileR + 4;  // bytes per shared tile column: 4-byte reads, 2-way conflicts on the writes

template <int IN>
__device__ __forceinline__ void load_tile_units(const void* x, int64_t rows, int64_t cols, int64_t r0, int64_t c0,
                                                int lr, int lc, Unit (&v)[2], bool (&have)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t r = r0 + lr + h * (kTileR / 2);
        have[h] = r < rows && c0 + lc < cols;
        if (have[h]) load_unit<IN>(x, (r * cols + c0 + lc) >> 3, v[h]);
    }
}

template <int FMT, int MODE, int IN, int LAYOUT>
__global__ void __launch_bounds__(kThreads)
quantize2d_kernel(const void* __restrict__ x, int64_t rows, int64_t cols, uint8_t* __restrict__ out8,
                  uint8_t* __restrict__ out8_t, fp8_ring* ring, uint32_t* amax_acc, float* amax_out,
                  float* scale_out) {
    static_assert(kThreads * 16 == kTileR * kTileC, "two units per thread and tile");
    __shared__ float s_scale;
    __shared__ __align__(16) uint8_t tile[kTileC][kTileStride];
    griddep_wait();
    const int64_t tcols = (cols + kTileC - 1) / kTileC;
    const int64_t tiles = ((rows + kTileR - 1) / kTileR) * tcols;
    const int lr = threadIdx.x >> 3;         // tile rows lr and lr + 64 this thread loads
    const int lc = (threadIdx.x & 7) * 8;    // its first tile column
    const int oc = threadIdx.x >> 3;         // tile column (transposed row) it writes
    const int orow = (threadIdx.x & 7) * 16; // its first tile row there
    // the first tile's loads leave before the scale is known
    int64_t t = blockIdx.x;
    Unit v[2];
    bool have[2] = {false, false};
    int64_t r0 = 0, c0 = 0;
    if (t < tiles) {
        r0 = (t / tcols) * kTileR;
        c0 = (t % tcols) * kTileC;
        load_tile_units<IN>(x, rows, cols, r0, c0, lr, lc, v, have);
    }
    const float s = read_scale<FMT, MODE>(ring, amax_acc, scale_out, blockIdx.x, s_scale);
    float m = 0.0f;
    while (t < tiles) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint2 q = make_uint2(0u, 0u);
            const int r = lr + h * (kTileR / 2);
            if (have[h]) {
                float f[8];
                unit_f32<IN>(v[h], f);
                q = quant8<FMT>(f, s, m);
                if (LAYOUT == FP8_QL_BOTH) *reinterpret_cast<uint2*>(out8 + (r0 + r) * cols + c0 + lc) = q;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                tile[lc + k][r] = uint8_t(q.x >> (8 * k));
                tile[lc + 4 + k][r] = uint8_t(q.y >> (8 * k));
            }
        }
        __syncthreads();
        const int64_t tr0 = r0, tc0 = c0;
        t += gridDim.x;
        if (t < tiles) {  // the next tile's loads, in flight while this one is written out
            r0 = (t / tcols) * kTileR;
            c0 = (t % tcols) * kTileC;
            load_tile_units<IN>(x, rows, cols, r0, c0, lr, lc, v, have);
        }
#pragma unroll
        for (int g8 = 0; g8 < 2; ++g8) {  // two groups of 8 rows (rows is a multiple of 8)
            const int rr = orow + 8 * g8;
            if (tc0 + oc < cols && tr0 + rr < rows) {
                const uint32_t w0 = *reinterpret_cast<const uint32_t*>(&tile[oc][rr]);
                const uint32_t w1 = *reinterpret_cast<const uint32_t*>(&tile[oc][rr + 4]);
                *reinterpret_cast<uint2*>(out8_t + (tc0 + oc) * rows + tr0 + rr) = make_uint2(w0, w1);
            }
        }
        __syncthreads();  // the shared tile is free for the next tile
    }
    griddep_launch();
    finish_block<FMT, MODE>(m, ring, amax_acc, amax_out, blockIdx.x, gridDim.x);
}

// Several delayed-scaling quantizations in one launch: job j owns blocks
// [first[j], first[j] + blocks[j]) of the grid and runs exactly what
// fp8_quantize does for it, its ring finalized by the last of its blocks.
struct QuantJobs {
    int count;
    int first[FP8_QUANTIZE_MAX_JOBS];
    int blocks[FP8_QUANTIZE_MAX_JOBS];
    int fmt[FP8_QUANTIZE_MAX_JOBS];
    int dtype[FP8_QUANTIZE_MAX_JOBS];
    const void* x[FP8_QUANTIZE_MAX_JOBS];
    int64_t n[FP8_QUANTIZE_MAX_JOBS];
    fp8_ring* ring[FP8_QUANTIZE_MAX_JOBS];
    uint8_t* out8[FP8_QUANTIZE_MAX_JOBS];
    float* amax_out[FP8_QUANTIZE_MAX_JOBS];
    float* scale_out[FP8_QUANTIZE_MAX_JOBS];
};

template <int MODE>
__global__ void __launch_bounds__(kThreads) quantize_many_kernel(const __grid_constant__ QuantJobs jobs) {
    __shared__ float s_scale;
    griddep_wait();
    int j = 0;
    while (j + 1 < jobs.count && int(blockIdx.x) >= jobs.first[j + 1]) ++j;
    const int blk = int(blockIdx.x) - jobs.first[j];
#define FP8LITE_JOB(F, I)                                                                                        \
    quantize_body<F, MODE, I>(jobs.x[j], jobs.n[j], jobs.out8[j], jobs.ring[j], nullptr, jobs.amax_out[j],     \
                                  jobs.scale_out[j], blk, jobs.blocks[j], s_scale)
    const int dt = jobs.dtype[j];
    if (jobs.fmt[j] == FP8_E4M3) {
        if (dt == FP8_IN_BF16)     FP8LITE_JOB(FP8_E4M3, FP8_IN_BF16);
        else if (dt == FP8_IN_F16) FP8LITE_JOB(FP8_E4M3, FP8_IN_F16);
        else                       FP8LITE_JOB(FP8_E4M3, FP8_IN_F32);
    } else {
        if (dt == FP8_IN_BF16)     FP8LITE_JOB(FP8_E5M2, FP8_IN_BF16);
        else if (dt == FP8_IN_F16) FP8LITE_JOB(FP8_E5M2, FP8_IN_F16);
        else                       FP8LITE_JOB(FP8_E5M2, FP8_IN_F32);
    }
#undef FP8LITE_JOB
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

// Folds each ring's accumulated amax (a deferred call's, after the group's
// all-reduce) into its history exactly as a delayed call's last block does.
constexpr int kMaxFoldRings = 64;
struct FoldFmts {
    int fmt[kMaxFoldRings];
};

__global__ void rings_fold_kernel(fp8_ring* rings, int count, const __grid_constant__ FoldFmts f) {
    griddep_wait();
    const int i = threadIdx.x;
    if (i < count) {
        volatile fp8_ring* r = rings + i;
        float h[FP8_RING_HISTORY];
        const uint32_t idx = ring_read(r, h);
        ring_fold(r, h, idx, __uint_as_float(r->amax_bits), fmt_max(f.fmt[i]));
        r->amax_bits = 0u;
    }
    griddep_launch();
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

// Blocks of a single-tensor launch. Every block adds its amax and takes a
// ticket on the ring's one cache line, and those same-address atomics queue
// (about 2 ns each on B200), so below 64 M elements the grid is kept at one
// to two blocks per SM: at least one per SM, so that every SM's loads are in
// flight (as long as each thread still gets a unit), and at most two, each
// thread looping over further rounds of kUnroll units. From 64 M elements on
// the atomics are a small part of the time and four blocks per SM keep more
// loads in flight. Measured on B200 (delayed E4M3, back-to-back launches,
// microseconds, grid of up to four blocks per SM -> this one): 1M elements
// 3.81 -> 3.52, 2M 3.81 -> 3.73, 8M 7.04 -> 5.65, 16M 10.63 -> 9.48; 256M
// elements took 125.8 with four blocks per SM and 129.9 with two.
int grid_for(int64_t n) {
    const int64_t units = n >> 3;
    const int64_t sms = sm_count();
    const int64_t want = (units + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
    const int64_t busy = (units + kThreads - 1) / kThreads;  // blocks whose every thread has a unit
    const int64_t cap = (n >= (int64_t(1) << 26) ? 4 : 2) * sms;
    int64_t g = want < sms ? sms : want;
    if (g > cap) g = cap;
    if (g > busy) g = busy;
    return int(g < 1 ? 1 : g);
}

// Blocks of each job of a grouped launch: the whole launch gets the blocks
// one large tensor would (two per SM), shared in proportion to the jobs'
// sizes, each job at least one block and at most one unit per thread. Every
// job's atomics go to its own ring, so fewer blocks in all means less
// queueing on each ring's line. Measured on B200 on the linear stack's
// step-start launch (every weight and the first activation, 14.7 M elements,
// microseconds): each job sized as its own launch 9.46, in proportion 8.93.
void grid_many(const fp8_quantize_job* jobs, int count, int* blocks) {
    int64_t all = 0;
    for (int j = 0; j < count; ++j) all += jobs[j].n;
    const int64_t budget = 2 * int64_t(sm_count());
    for (int j = 0; j < count; ++j) {
        const int64_t share = all > 0 ? (budget * jobs[j].n + all - 1) / all : 1;
        const int64_t busy = ((jobs[j].n >> 3) + kThreads - 1) / kThreads;
        const int64_t g = share < busy ? share : busy;
        blocks[j] = int(g < 1 ? 1 : g);
    }
}

template <int FMT, int IN>
fp8_status launch_quantize(const void* x, int64_t n, fp8_ring* ring, bool seed, bool defer, uint8_t* out8,
                           float* amax_out, float* scale_out, cudaStream_t st) {
    const int grid = grid_for(n);
    if (ring && defer)
        return launch_pdl(quantize_kernel<FMT, kDeferred, IN>, grid, kThreads, 0, st, 1, x, n, out8, ring,
                          (uint32_t*)nullptr, amax_out, scale_out);
    if (ring && !seed)
        return launch_pdl(quantize_kernel<FMT, kDelayed, IN>, grid, kThreads, 0, st, 1, x, n, out8, ring,
                          (uint32_t*)nullptr, amax_out, scale_out);
    if constexpr (IN != FP8_IN_F32) {
        // current scaling of a small tensor: one launch (measured on B200, an
        // NT 256^3 operand: 8.0 us for the memset and two passes)
        if (!ring && n <= kSmallMax)
            return launch_pdl(quantize_small_current_kernel<FMT, IN>, 1, kSmallThreads, 0, st, 1, x, n, out8,
                              amax_out, scale_out);
    }
    uint32_t* acc = reinterpret_cast<uint32_t*>(amax_out);
    if (cudaMemsetAsync(acc, 0, sizeof(uint32_t), st) != cudaSuccess) return FP8_ERR_CUDA;
    if (launch_pdl(quantize_kernel<FMT, kAmaxOnly, IN>, grid, kThreads, 0, st, 1, x, n, out8, (fp8_ring*)nullptr,
                   acc, (float*)nullptr, (float*)nullptr) != FP8_OK)
        return FP8_ERR_CUDA;
    if (seed)
        return launch_pdl(quantize_kernel<FMT, kSeed, IN>, grid, kThreads, 0, st, 1, x, n, out8, ring, acc,
                          (float*)nullptr, scale_out);
    return launch_pdl(quantize_kernel<FMT, kCurrentQuant, IN>, grid, kThreads, 0, st, 1, x, n, out8,
                      (fp8_ring*)nullptr, acc, (float*)nullptr, scale_out);
}

template <int FMT>
fp8_status launch_quantize_in(fp8_dtype dtype, const void* x, int64_t n, fp8_ring* ring, bool seed, bool defer,
                              uint8_t* out8, float* amax_out, float* scale_out, cudaStream_t st) {
    switch (dtype) {
        case FP8_IN_BF16:
            return launch_quantize<FMT, FP8_IN_BF16>(x, n, ring, seed, defer, out8, amax_out, scale_out, st);
        case FP8_IN_F16:
            return launch_quantize<FMT, FP8_IN_F16>(x, n, ring, seed, defer, out8, amax_out, scale_out, st);
        default:
            return launch_quantize<FMT, FP8_IN_F32>(x, n, ring, seed, defer, out8, amax_out, scale_out, st);
    }
}

bool valid_dtype(int d) { return d == FP8_IN_BF16 || d == FP8_IN_F16 || d == FP8_IN_F32; }

template <int FMT, int IN, int LAYOUT>
fp8_status launch_quantize_2d(const void* x, int64_t rows, int64_t cols, fp8_ring* ring, bool seed, uint8_t* out8,
                              uint8_t* out8_t, float* amax_out, float* scale_out, cudaStream_t st) {
    const int64_t tiles = ((rows + kTileR - 1) / kTileR) * ((cols + kTileC - 1) / kTileC);
    const int64_t cap = int64_t(sm_count()) * (2048 / kThreads);
    const int grid = int(tiles < 1 ? 1 : tiles < cap ? tiles : cap);
    if (ring && !seed)
        return launch_pdl(quantize2d_kernel<FMT, kDelayed, IN, LAYOUT>, grid, kThreads, 0, st, 1, x, rows, cols, out8,
                          out8_t, ring, (uint32_t*)nullptr, amax_out, scale_out);
    // current scaling or a seeded call: the flat amax pass first
    uint32_t* acc = reinterpret_cast<uint32_t*>(amax_out);
    const int64_t n = rows * cols;
    if (cudaMemsetAsync(acc, 0, sizeof(uint32_t), st) != cudaSuccess) return FP8_ERR_CUDA;
    if (launch_pdl(quantize_kernel<FMT, kAmaxOnly, IN>, grid_for(n), kThreads, 0, st, 1, x, n, (uint8_t*)nullptr,
                   (fp8_ring*)nullptr, acc, (float*)nullptr, (float*)nullptr) != FP8_OK)
        return FP8_ERR_CUDA;
    if (seed)
        return launch_pdl(quantize2d_kernel<FMT, kSeed, IN, LAYOUT>, grid, kThreads, 0, st, 1, x, rows, cols, out8,
                          out8_t, ring, acc, (float*)nullptr, scale_out);
    return launch_pdl(quantize2d_kernel<FMT, kCurrentQuant, IN, LAYOUT>, grid, kThreads, 0, st, 1, x, rows, cols,
                      out8, out8_t, (fp8_ring*)nullptr, acc, (float*)nullptr, scale_out);
}

template <int FMT, int LAYOUT>
fp8_status launch_quantize_2d_in(fp8_dtype dtype, const void* x, int64_t rows, int64_t cols, fp8_ring* ring, bool seed,
                                 uint8_t* out8, uint8_t* out8_t, float* amax_out, float* scale_out, cudaStream_t st) {
    switch (dtype) {
        case FP8_IN_BF16:
            return launch_quantize_2d<FMT, FP8_IN_BF16, LAYOUT>(x, rows, cols, ring, seed, out8, out8_t, amax_out,
                                                                scale_out, st);
        case FP8_IN_F16:
            return launch_quantize_2d<FMT, FP8_IN_F16, LAYOUT>(x, rows, cols, ring, seed, out8, out8_t, amax_out,
                                                               scale_out, st);
        default:
            return launch_quantize_2d<FMT, FP8_IN_F32, LAYOUT>(x, rows, cols, ring, seed, out8, out8_t, amax_out,
                                                               scale_out, st);
    }
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

extern "C" fp8_status fp8_quantize_ex(const void* x, fp8_dtype dtype, int64_t n, fp8_fmt fmt, fp8_ring* ring,
                                      uint32_t flags, uint8_t* out8, float* amax_out, float* scale_out,
                                      void* stream) {
    if (!valid_fmt(fmt) || !valid_dtype(dtype)) return FP8_ERR_INVALID_ARG;
    if ((flags & ~uint32_t(FP8_QUANTIZE_SEED_RING | FP8_QUANTIZE_DEFER_FOLD)) != 0u) return FP8_ERR_INVALID_ARG;
    const bool seed = (flags & FP8_QUANTIZE_SEED_RING) != 0u;
    const bool defer = (flags & FP8_QUANTIZE_DEFER_FOLD) != 0u;
    if ((seed || defer) && !ring) return FP8_ERR_INVALID_ARG;
    if (seed && defer) return FP8_ERR_INVALID_ARG;
    if (n < 0 || n >= (int64_t(1) << 40)) return FP8_ERR_INVALID_ARG;
    if (!scale_out) return FP8_ERR_INVALID_ARG;
    if (n > 0 && (!x || !out8)) return FP8_ERR_INVALID_ARG;
    if ((!ring || seed) && !amax_out) return FP8_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out8, 16)) return FP8_ERR_ALIGNMENT;
    if (ring && !aligned(ring, 4)) return FP8_ERR_ALIGNMENT;
    if (!aligned(scale_out, 4) || !aligned(amax_out, 4)) return FP8_ERR_ALIGNMENT;
    cudaStream_t st = as_stream(stream);
    return fmt == FP8_E4M3
               ? launch_quantize_in<FP8_E4M3>(dtype, x, n, ring, seed, defer, out8, amax_out, scale_out, st)
               : launch_quantize_in<FP8_E5M2>(dtype, x, n, ring, seed, defer, out8, amax_out, scale_out, st);
}

extern "C" fp8_status fp8_quantize_2d(const void* x, fp8_dtype dtype, int64_t rows, int64_t cols, fp8_fmt fmt,
                                      fp8_ring* ring, uint32_t flags, fp8_quant_layout layout, uint8_t* out8,
                                      uint8_t* out8_t, float* amax_out, float* scale_out, void* stream) {
    if (layout != FP8_QL_ROW && layout != FP8_QL_COL && layout != FP8_QL_BOTH) return FP8_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || (cols > 0 && rows >= (int64_t(1) << 40) / cols)) return FP8_ERR_INVALID_ARG;
    if (flags & FP8_QUANTIZE_DEFER_FOLD) return FP8_ERR_INVALID_ARG;  // offered by the flat quantize only
    if (layout == FP8_QL_ROW)  // the row-major codes alone are the flat quantize
        return fp8_quantize_ex(x, dtype, rows * cols, fmt, ring, flags, out8, amax_out, scale_out, stream);
    if (!valid_fmt(fmt) || !valid_dtype(dtype)) return FP8_ERR_INVALID_ARG;
    if ((flags & ~uint32_t(FP8_QUANTIZE_SEED_RING)) != 0u) return FP8_ERR_INVALID_ARG;
    const bool seed = (flags & FP8_QUANTIZE_SEED_RING) != 0u;
    if (seed && !ring) return FP8_ERR_INVALID_ARG;
    if (!scale_out || ((!ring || seed) && !amax_out)) return FP8_ERR_INVALID_ARG;
    const int64_t n = rows * cols;
    if (n > 0 && (!x || !out8_t || (layout == FP8_QL_BOTH && !out8))) return FP8_ERR_INVALID_ARG;
    if (rows % 8 != 0 || cols % 8 != 0) return FP8_ERR_ALIGNMENT;
    if (!aligned(x, 16) || !aligned(out8, 16) || !aligned(out8_t, 16)) return FP8_ERR_ALIGNMENT;
    if (ring && !aligned(ring, 4)) return FP8_ERR_ALIGNMENT;
    if (!aligned(scale_out, 4) || !aligned(amax_out, 4)) return FP8_ERR_ALIGNMENT;
    cudaStream_t st = as_stream(stream);
    if (fmt == FP8_E4M3)
        return layout == FP8_QL_COL
                   ? launch_quantize_2d_in<FP8_E4M3, FP8_QL_COL>(dtype, x, rows, cols, ring, seed, out8, out8_t,
                                                                 amax_out, scale_out, st)
                   : launch_quantize_2d_in<FP8_E4M3, FP8_QL_BOTH>(dtype, x, rows, cols, ring, seed, out8, out8_t,
                                                                  amax_out, scale_out, st);
    return layout == FP8_QL_COL
               ? launch_quantize_2d_in<FP8_E5M2, FP8_QL_COL>(dtype, x, rows, cols, ring, seed, out8, out8_t, amax_out,
                                                             scale_out, st)
               : launch_quantize_2d_in<FP8_E5M2, FP8_QL_BOTH>(dtype, x, rows, cols, ring, seed, out8, out8_t,
                                                              amax_out, scale_out, st);
}

extern "C" fp8_status fp8_rings_fold(fp8_ring* rings, int32_t count, const int32_t* fmts, void* stream) {
    if (!rings || !fmts || count < 1 || count > kMaxFoldRings) return FP8_ERR_INVALID_ARG;
    if (!aligned(rings, 4)) return FP8_ERR_ALIGNMENT;
    FoldFmts f = {};
    for (int i = 0; i < count; ++i) {
        if (!valid_fmt(fmts[i])) return FP8_ERR_INVALID_ARG;
        f.fmt[i] = fmts[i];
    }
    return launch_pdl(rings_fold_kernel, 1, kMaxFoldRings, 0, as_stream(stream), 1, rings, int(count), f);
}

extern "C" fp8_status fp8_quantize(const void* x, int64_t n, fp8_fmt fmt, fp8_ring* ring, uint8_t* out8,
                                   float* amax_out, float* scale_out, void* stream) {
    return fp8_quantize_ex(x, FP8_IN_BF16, n, fmt, ring, 0u, out8, amax_out, scale_out, stream);
}

extern "C" fp8_status fp8_quantize_many_ex(const fp8_quantize_job* jobs, int32_t count, uint32_t flags,
                                           void* stream) {
    if (!jobs || count < 1 || count > FP8_QUANTIZE_MAX_JOBS) return FP8_ERR_INVALID_ARG;
    if ((flags & ~uint32_t(FP8_QUANTIZE_DEFER_FOLD)) != 0u) return FP8_ERR_INVALID_ARG;
    QuantJobs q = {};
    q.count = count;
    int total = 0;
    for (int j = 0; j < count; ++j)  // sizes first: the grid is shared in proportion to them
        if (jobs[j].n < 0 || jobs[j].n >= (int64_t(1) << 40)) return FP8_ERR_INVALID_ARG;
    int blocks[FP8_QUANTIZE_MAX_JOBS];
    grid_many(jobs, count, blocks);
    for (int j = 0; j < count; ++j) {
        const fp8_quantize_job& in = jobs[j];
        if (!valid_fmt(in.fmt) || !valid_dtype(in.dtype)) return FP8_ERR_INVALID_ARG;
        if (in.n < 0 || in.n >= (int64_t(1) << 40)) return FP8_ERR_INVALID_ARG;
        if (!in.ring || !in.scale_out) return FP8_ERR_INVALID_ARG;
        if (in.n > 0 && (!in.x || !in.out8)) return FP8_ERR_INVALID_ARG;
        if (!aligned(in.x, 16) || !aligned(in.out8, 16)) return FP8_ERR_ALIGNMENT;
        if (!aligned(in.ring, 4) || !aligned(in.scale_out, 4) || !aligned(in.amax_out, 4)) return FP8_ERR_ALIGNMENT;
        for (int k = 0; k < j; ++k)
            if (jobs[k].ring == in.ring) return FP8_ERR_INVALID_ARG;  // one ring, one call at a time
        q.first[j] = total;
        q.blocks[j] = blocks[j];
        total += q.blocks[j];
        q.fmt[j] = int(in.fmt);
        q.dtype[j] = int(in.dtype);
        q.x[j] = in.x;
        q.n[j] = in.n;
        q.ring[j] = in.ring;
        q.out8[j] = in.out8;
        q.amax_out[j] = in.amax_out;
        q.scale_out[j] = in.scale_out;
    }
    if (flags & FP8_QUANTIZE_DEFER_FOLD)
        return launch_pdl(quantize_many_kernel<kDeferred>, total, kThreads, 0, as_stream(stream), 1, q);
    return launch_pdl(quantize_many_kernel<kDelayed>, total, kThreads, 0, as_stream(stream), 1, q);
}

extern "C" fp8_status fp8_quantize_many(const fp8_quantize_job* jobs, int32_t count, void* stream) {
    return fp8_quantize_many_ex(jobs, count, 0u, stream);
}

extern "C" fp8_status fp8_quantize_current_many(const fp8_quantize_job* jobs, int32_t count, void* stream) {
    if (!jobs || count < 1 || count > FP8_QUANTIZE_MAX_JOBS) return FP8_ERR_INVALID_ARG;
    SmallJobs q = {};
    for (int j = 0; j < count; ++j) {
        const fp8_quantize_job& in = jobs[j];
        if (!valid_fmt(in.fmt) || !valid_dtype(in.dtype)) return FP8_ERR_INVALID_ARG;
        if (in.ring || !in.scale_out || in.n < 0) return FP8_ERR_INVALID_ARG;
        if (in.n > 0 && (!in.x || !in.out8)) return FP8_ERR_INVALID_ARG;
        if (in.dtype == FP8_IN_F32 || in.n > kSmallMax) return FP8_ERR_UNSUPPORTED;
        if (!aligned(in.x, 16) || !aligned(in.out8, 16)) return FP8_ERR_ALIGNMENT;
        if (!aligned(in.scale_out, 4) || !aligned(in.amax_out, 4)) return FP8_ERR_ALIGNMENT;
        q.x[j] = in.x;
        q.n[j] = in.n;
        q.out8[j] = in.out8;
        q.amax_out[j] = in.amax_out;
        q.scale_out[j] = in.scale_out;
        q.kind[j] = 2 * int(in.fmt) + int(in.dtype);
    }
    return launch_pdl(quantize_small_current_many_kernel, count, kSmallThreads, 0, as_stream(stream), 1, q);
}
