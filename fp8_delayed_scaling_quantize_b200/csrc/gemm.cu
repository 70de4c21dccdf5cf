// Per-tensor-scaled FP8 GEMM with fused bias and bf16 output, on the sm_100a
// 5th-generation tensor cores (tcgen05, kind::f8f6f4).
//
// Method: AstrAI commit logs -- astrai/extension/fp8.py @f4c44ebf (bias added
// in fp32 before the single bf16 rounding; 3-D operands with stride-0
// broadcast; bf16-only output), tests/extension/test_fp8_mma.py @cebdd45d
// (bias_scale slot: bf16 bias when null, dequantized fp8 bias otherwise) and
// csrc/kernels/fp8/gemm.cuh @5e76fbd1 (the NT / NN / TN operand layouts of a
// linear layer's forward, dX and dW).
//
// Design (B200-first; the pages' sm_89 mma.sync / ldmatrix / cp.async / PRMT
// kernel is prior art only):
//  * persistent CTAs (one per SM at most), each walking output tiles
//    BM x BN = 128 x {64,128,256} in M-fastest order so CTAs that run together
//    share the B (weight) tile in L2;
//  * 6 warps with fixed roles: warp 0 issues TMA loads (one lane), warp 1
//    owns TMEM and issues tcgen05.mma (one lane), warps 2-5 run the epilogue;
//  * operands arrive by TMA in 128-byte-swizzled shared-memory stages of
//    BK = 128 bytes of K, in their stored orientation: K-major for A in
//    NT/NN and B in NT, MN-major for A in TN and B in NN/TN (the tensor core
//    reads MN-major 8-bit operands directly, so dX / dW need no transposed
//    copies). TMA zero-fills every M, N, K tail and batch end;
//  * each stage is 4 MMAs of 128 x BN x 32 accumulating in TMEM (fp32);
//    tcgen05.commit releases the stage back to the producer;
//  * two TMEM accumulators (2 x BN columns): the epilogue of tile i overlaps
//    the main loop of tile i+1;
//  * epilogue: tcgen05.ld 32 columns at a time, y = acc * (1/sa)(1/sb) +
//    bias in fp32 (one fma), one round-to-nearest-even to bf16, guarded
//    stores (exact M / N tails);
//  * every mbarrier wait is bounded by a time limit; a wait that gives up
//    records FP8_ERR_DEVICE_TIMEOUT in the library's device error word and the
//    CTA stops issuing work and exits through the normal teardown.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace fp8lite {

__device__ uint32_t g_device_error = 0;

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 128;  // bytes = elements of K per stage
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

struct GemmParams {
    int M, N, K;
    int m_tiles, n_tiles, k_blocks, total_tiles;
    int group_m;  // tiles are walked in groups of this many M-tile rows
    int a_bcast, b_bcast;
    uint32_t idesc;
    const float* sa;
    const float* sb;
    const void* bias;
    const float* bias_scale;
    int bias_kind;  // 0 none, 1 bf16, 2 fp8
    int bias_fmt;
    uint16_t* out;
    int64_t stride_c;
    int vec_store;  // 16-byte stores allowed (N, stride_c multiples of 8, base aligned)
    int tma_store;  // tiles leave through shared memory and TMA stores (same conditions)
};

// Wait for phase `parity` of the mbarrier at `bar`, giving up after
// `limit_ns`: then the library's device error word is set and false returned.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 0 && globaltimer_ns() - t0 > limit_ns) {
            atomicOr(&g_device_error, 1u);
            return false;
        }
    }
}

// Diagnostic: one thread waits, through the same bounded wait the GEMM
// uses, on a shared-memory barrier that nothing ever arrives at.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    wait_bounded(b, 0, limit_ns);
}

// One FP8 code -> fp32 (exact: every E4M3 / E5M2 value is an fp16 value).
__device__ __forceinline__ float fp8_to_f32(uint8_t c, int fmt) {
    uint32_t h;
    const uint16_t in = c;
    if (fmt == FP8_E4M3) {
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
    } else {
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(in));
    }
    return __half2float(__ushort_as_half(uint16_t(h & 0xFFFFu)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Shared-memory plan of one CTA. CTAS = 2: an MMA pair, each CTA holding its
// 128 rows of A and BN/2 columns of B per stage.
template <int BN, int STAGES, int CTAS>
struct Smem {
    static constexpr int kABytes = BM * BK;
    static constexpr int kBBytes = (BN / CTAS) * BK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStageTx = CTAS * kStageBytes;  // bytes landing on the leader's full barrier
    // per epilogue warp, two 32x32 bf16 staging buffers (64-byte swizzle)
    static constexpr int kStgBufBytes = 32 * 32 * 2;
    static constexpr int kStgOffset = STAGES * kStageBytes;
    static constexpr int kBiasOffset = kStgOffset + 4 * 2 * kStgBufBytes;  // BN fp32 bias values
    static constexpr int kBarOffset = kBiasOffset + BN * 4;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], then the TMEM slot
    static constexpr int kBytes = kBarOffset + (2 * STAGES + 4) * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
    static constexpr uint32_t kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;
};

// Tile order: batch outermost; inside a batch, groups of `group_m` M-tile
// rows, walked M-fastest within the group, then N. A wave of concurrently
// running tiles then covers a compact block of rows and columns whose A and B
// panels stay resident in L2 (an M-fastest walk over all rows streams the
// whole A through L2 every wave).
__device__ __forceinline__ void tile_coords(int t, const GemmParams& p, int& mb, int& nb, int& b) {
    const int per_batch = p.m_tiles * p.n_tiles;
    b = t / per_batch;
    const int r = t - b * per_batch;
    const int per_group = p.group_m * p.n_tiles;
    const int g = r / per_group;
    const int first_m = g * p.group_m;
    const int rows = min(p.group_m, p.m_tiles - first_m);
    const int i = r - g * per_group;
    mb = first_m + i % rows;
    nb = i / rows;
}

__device__ __forceinline__ void epilogue_bar() {
    // named barrier 1 over the 4 epilogue warps (128 threads)
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// One kernel for both tile shapes: CTAS = 1 computes 128 x BN tiles per CTA;
// CTAS = 2 runs as clusters of two CTAs on two SMs computing 256 x BN tiles
// with tcgen05 cta_group::2 -- the leader issues the MMAs, each CTA loads its
// own 128 rows of A and BN/2 columns of B (halving each SM's operand
// traffic) and writes its own 128 output rows.
template <int BN, bool A_MN, bool B_MN, int STAGES, bool HAS_BIAS, int CTAS>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_c, const GemmParams p) {
    using L = Smem<BN, STAGES, CTAS>;
    static_assert(!(B_MN && CTAS == 2 && BN != 256), "MN-major B halves must be whole 128-byte atoms");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_addr(smem);
    const uint32_t s_a = s_base;
    const uint32_t s_b = s_base + STAGES * L::kABytes;
    const uint32_t bar_full = s_base + L::kBarOffset;
    const uint32_t bar_empty = bar_full + STAGES * 8;
    const uint32_t bar_tfull = bar_empty + STAGES * 8;
    const uint32_t bar_tempty = bar_tfull + 2 * 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBarOffset + (2 * STAGES + 4) * 8);
    float* s_bias = reinterpret_cast<float*>(smem + L::kBiasOffset);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = CTAS == 2 ? cluster_ctarank() : 0u;  // 0 = the pair's leader
    const bool leader = rank == 0;
    const int unit0 = blockIdx.x / CTAS;     // this CTA's first tile (a pair shares it)
    const int unit_step = gridDim.x / CTAS;  // tiles advance by the number of CTAs (pairs)

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, CTAS * 4 * 32);
        }
        fence_mbar_init();
        tma_prefetch(&tm_a);
        tma_prefetch(&tm_b);
        if (p.tma_store) tma_prefetch(&tm_c);
    }
    if (warp == 1) {
        tmem_alloc<CTAS>(smem_addr(tmem_slot), L::kTmemCols);
        tmem_relinquish<CTAS>();
    }
    tc_fence_before();
    __syncthreads();
    if (CTAS == 2) cluster_sync();  // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The prologue above overlaps the previous kernel's tail; operands,
    // scales and the output are touched only after it has completed.
    griddep_wait();
    griddep_launch();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = unit0; t < p.total_tiles && ok; t += unit_step) {
                int mb, nb, b;
                tile_coords(t, p, mb, nb, b);
                const int ba = p.a_bcast ? 0 : b;
                const int bb = p.b_bcast ? 0 : b;
                const int m0 = mb * BM * CTAS + int(rank) * BM;
                const int n0 = nb * BN + int(rank) * (BN / CTAS);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!wait_bounded(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
                    const uint32_t full = bar_full + 8 * stage;
                    if (leader) mbar_arrive_expect_tx(full, L::kStageTx);
                    const uint32_t da = s_a + stage * L::kABytes;
                    const uint32_t db = s_b + stage * L::kBBytes;
                    if (CTAS == 1) {
                        if (A_MN) tma_load_3d(da, &tm_a, full, m0, kb * BK, ba);
                        else      tma_load_3d(da, &tm_a, full, kb * BK, m0, ba);
                        if (B_MN) {
#pragma unroll
                            for (int h = 0; h < BN / 128; ++h)
                                tma_load_3d(db + h * 128 * BK, &tm_b, full, n0 + h * 128, kb * BK, bb);
                        } else {
                            tma_load_3d(db, &tm_b, full, kb * BK, n0, bb);
                        }
                    } else {
                        const uint32_t lfull = map_to_rank(full, 0);  // the leader's barrier
                        if (A_MN) tma_load_3d_pair(da, &tm_a, lfull, m0, kb * BK, ba);
                        else      tma_load_3d_pair(da, &tm_a, lfull, kb * BK, m0, ba);
                        if (B_MN) tma_load_3d_pair(db, &tm_b, lfull, n0, kb * BK, bb);
                        else      tma_load_3d_pair(db, &tm_b, lfull, kb * BK, n0, bb);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            // drain: wait until the MMAs released every stage still in use
            for (int i = 0; i < STAGES && ok; ++i) {
                if (!wait_bounded(bar_empty + 8 * stage, phase ^ 1)) break;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer ---
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int t = unit0; t < p.total_tiles && ok; t += unit_step, ++it) {
                const int buf = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!wait_bounded(bar_tempty + 8 * buf, acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!wait_bounded(bar_full + 8 * stage, phase)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t da = s_a + stage * L::kABytes;
                    const uint32_t db = s_b + stage * L::kBBytes;
#pragma unroll
                    for (int j = 0; j < BK / 32; ++j) {
                        // K-major: the 32-byte K step moves inside the swizzle atom;
                        // MN-major: it skips 32 rows of 128 bytes (4 atoms).
                        const uint64_t adesc = A_MN ? smem_desc_sw128(da + j * 32 * 128, 128 * BK, 1024)
                                                    : smem_desc_sw128(da + j * 32, 16, 1024);
                        const uint64_t bdesc = B_MN ? smem_desc_sw128(db + j * 32 * 128, 128 * BK, 1024)
                                                    : smem_desc_sw128(db + j * 32, 16, 1024);
                        mma_f8f6f4<CTAS>(d_tmem, adesc, bdesc, p.idesc, (kb | j) != 0);
                    }
                    // release the stage (in both CTAs of a pair)
                    if (CTAS == 1) mma_commit(bar_empty + 8 * stage);
                    else           mma_commit_pair(bar_empty + 8 * stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (CTAS == 1) mma_commit(bar_tfull + 8 * buf);
                else           mma_commit_pair(bar_tfull + 8 * buf);
            }
        }
    } else {
        // ----------------------------------------------------- epilogue ---
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row_in_tile = q * 32 + lane;
        const int etid = threadIdx.x - 64;  // 0..127 over the epilogue warps
        const float inv = (1.0f / __ldg(p.sa)) * (1.0f / __ldg(p.sb));
        const float bscale = (HAS_BIAS && p.bias_kind == 2) ? __ldg(p.bias_scale) : 1.0f;
        const uint32_t s_stg = s_base + L::kStgOffset;
        int stg_n = 0;  // TMA stores issued by this warp
        bool failed = false;
        int it = 0;
        for (int t = unit0; t < p.total_tiles; t += unit_step, ++it) {
            int mb, nb, b;
            tile_coords(t, p, mb, nb, b);
            const int buf = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            const int m0 = mb * BM * CTAS + int(rank) * BM;  // this CTA's first output row
            if (HAS_BIAS) {
                // the tile's BN bias values, dequantized once into shared memory
                epilogue_bar();  // the previous tile's readers are done
                for (int j = etid; j < BN; j += 128) {
                    const int col = nb * BN + j;
                    float v = 0.0f;
                    if (col < p.N) {
                        if (p.bias_kind == 1) {
                            v = __uint_as_float(uint32_t(__ldg(static_cast<const uint16_t*>(p.bias) + col)) << 16);
                        } else {
                            v = __fdiv_rn(fp8_to_f32(__ldg(static_cast<const uint8_t*>(p.bias) + col), p.bias_fmt),
                                          bscale);
                        }
                    }
                    s_bias[j] = v;
                }
                epilogue_bar();
            }
            // every lane waits, then the warp agrees (and reconverges) before
            // the warp-collective TMEM loads. After a wait gave up, the warp
            // keeps walking the tiles without waiting so that the epilogue
            // warps still meet at every named barrier above.
            if (!failed) {
                const bool ok = wait_bounded(bar_tfull + 8 * buf, acc_phase);
                failed = !__all_sync(0xffffffffu, ok);
            }
            if (failed) continue;
            tc_fence_after();
            const int row = m0 + row_in_tile;
            uint16_t* orow = p.out + int64_t(b) * p.stride_c + int64_t(row) * p.N;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) + buf * BN + c * 32, r);
                tmem_ld_wait();
                const int col0 = nb * BN + c * 32;
                if (col0 >= p.N) continue;                       // warp-uniform
                if (!p.tma_store && row >= p.M) continue;
                float y[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float bias = HAS_BIAS ? s_bias[c * 32 + i] : 0.0f;
                    y[i] = fmaf(__uint_as_float(r[i]), inv, bias);
                }
                if (p.tma_store) {
                    // stage the warp's 32 x 32 bf16 block (64-byte swizzle: the
                    // 16-byte chunk index XOR (row / 2) mod 4 keeps the 8 lanes of
                    // a store phase on distinct banks), then one TMA store; it
                    // clips the M / N tails of the output
                    const uint32_t stg = s_stg + (q * 2 + (stg_n & 1)) * L::kStgBufBytes;
                    if (stg_n >= 2) {
                        if (lane == 0) bulk_wait_read<1>();
                        __syncwarp();
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t w0 = pack_bf16x2(y[8 * j + 0], y[8 * j + 1]);
                        const uint32_t w1 = pack_bf16x2(y[8 * j + 2], y[8 * j + 3]);
                        const uint32_t w2 = pack_bf16x2(y[8 * j + 4], y[8 * j + 5]);
                        const uint32_t w3 = pack_bf16x2(y[8 * j + 6], y[8 * j + 7]);
                        const uint32_t addr = stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1),
                                     "r"(w2), "r"(w3)
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tm_c, stg, col0, m0 + q * 32, b);
                        bulk_commit();
                    }
                    ++stg_n;
                } else if (p.vec_store && col0 + 32 <= p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + col0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack_bf16x2(y[8 * v + 0], y[8 * v + 1]);
                        w.y = pack_bf16x2(y[8 * v + 2], y[8 * v + 3]);
                        w.z = pack_bf16x2(y[8 * v + 4], y[8 * v + 5]);
                        w.w = pack_bf16x2(y[8 * v + 6], y[8 * v + 7]);
                        dst[v] = w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const uint32_t w = pack_bf16x2(y[i], y[i + 1]);
                        if (col0 + i < p.N) orow[col0 + i] = uint16_t(w & 0xFFFFu);
                        if (col0 + i + 1 < p.N) orow[col0 + i + 1] = uint16_t(w >> 16);
                    }
                }
            }
            tc_fence_before();
            // release the accumulator to the MMA issuer (the pair's leader)
            if (CTAS == 1) mbar_arrive(bar_tempty + 8 * buf);
            else           mbar_arrive_cluster(map_to_rank(bar_tempty + 8 * buf, 0));
        }
        // the staging buffers must outlive the stores that read them, and the
        // output must be complete when the grid is
        if (p.tma_store && lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (CTAS == 2) cluster_sync();  // neither CTA leaves while the other may still signal it
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc<CTAS>(tmem_base, L::kTmemCols);
    }
}

// ------------------------------------------------------------- host side ---

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 3-D map over uint8 codes: (inner, outer, batch) with a 128-byte swizzle.
// A broadcast operand (batch stride 0) gets a batch extent of 1.
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t batch,
              uint64_t batch_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint64_t pitch = inner;
    if (batch_stride_bytes == 0) {
        batch = 1;
        batch_stride_bytes = ((pitch * outer + 15) / 16) * 16;
    }
    cuuint64_t dims[3] = {inner, outer, batch};
    cuuint64_t strides[2] = {pitch, batch_stride_bytes};
    cuuint32_t box[3] = {box_inner, box_outer, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the bf16 output (N, M, batch), 32 x 32 boxes with a 64-byte
// swizzle matching the epilogue's staging layout.
bool make_out_map(CUtensorMap* map, void* base, uint64_t n, uint64_t m, uint64_t batch, uint64_t batch_stride_bytes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if (batch <= 1 || batch_stride_bytes == 0) {
        batch = 1;
        batch_stride_bytes = ((n * m * 2 + 15) / 16) * 16;
    }
    cuuint64_t dims[3] = {n, m, batch};
    cuuint64_t strides[2] = {n * 2, batch_stride_bytes};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
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

struct HostArgs {
    int fa, fb;
    const void* b8;
    int64_t batch, stride_b;
};

template <int BN, bool A_MN, bool B_MN, int STAGES, bool HAS_BIAS, int CTAS>
fp8_status launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, GemmParams p,
                      const HostArgs& h, cudaStream_t st) {
    using L = Smem<BN, STAGES, CTAS>;
    auto kern = fp8_gemm_kernel<BN, A_MN, B_MN, STAGES, HAS_BIAS, CTAS>;
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return FP8_ERR_CUDA;
        attr_set[dev] = true;
    }
    p.idesc = sm100::instr_desc_f8(h.fa, h.fb, A_MN ? 1 : 0, B_MN ? 1 : 0, BM * CTAS, BN);
    p.m_tiles = (p.M + BM * CTAS - 1) / (BM * CTAS);
    p.n_tiles = (p.N + BN - 1) / BN;
    const int64_t tiles = int64_t(p.m_tiles) * p.n_tiles * h.batch;
    p.total_tiles = int(tiles);
    p.group_m = CTAS == 2 ? 8 : 16;  // about sqrt(concurrent tiles) rows per group
    const int64_t units_max = sm_count() / CTAS;
    const int units = int(tiles < units_max ? tiles : units_max);
    return launch_pdl(kern, units * CTAS, kThreads, L::kAlloc, st, CTAS, ta, tb, tc, p);
}

template <int BN, bool A_MN, bool B_MN, int STAGES, int CTAS>
fp8_status launch(const CUtensorMap& ta, const CUtensorMap& tb, GemmParams p, const HostArgs& h, cudaStream_t st) {
    CUtensorMap tc = {};
    if (p.tma_store && !make_out_map(&tc, p.out, p.N, p.M, h.batch, uint64_t(p.stride_c) * 2)) return FP8_ERR_CUDA;
    return p.bias_kind ? launch_one<BN, A_MN, B_MN, STAGES, true, CTAS>(ta, tb, tc, p, h, st)
                       : launch_one<BN, A_MN, B_MN, STAGES, false, CTAS>(ta, tb, tc, p, h, st);
}

// Tile choice for 148 SMs by a small cost model: a persistent grid walks
// ceil(tiles / CTAs) rounds of tiles, each costing k_blocks times the
// per-k-block time of that tile shape, plus the one epilogue left exposed at
// the end. The per-k-block times (microseconds at the clocks seen under load)
// and epilogue times were measured on B200 with this kernel: 128x256 0.48,
// 128x128 0.40, 128x64 0.30, an SM pair's 256x256 0.43. Pairs are used only
// with at least one 256x256 tile per SM (below that their coarser grain
// loses). MN-major B needs whole 128-byte swizzle atoms along N per CTA.
struct TileChoice {
    bool pair;
    int bn;
};

inline TileChoice choose_tile(int64_t M, int64_t N, int64_t K, int64_t batch, bool b_mn, int64_t sms) {
    const int64_t kb = (K + BK - 1) / BK;
    auto cost = [&](int64_t rows, int bn, int64_t units, double t_k, double t_epi) {
        const int64_t tiles = ((M + rows - 1) / rows) * ((N + bn - 1) / bn) * batch;
        const int64_t rounds = (tiles + units - 1) / units;
        return double(rounds) * double(kb) * t_k + t_epi;
    };
    const int64_t pair_tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + 255) / 256) * batch;
    if (M > BM && N > 128 && pair_tiles >= sms) return {true, 256};
    TileChoice best = {false, 256};
    double best_cost = cost(BM, 256, sms, 0.48, 2.0);
    const double c128 = cost(BM, 128, sms, 0.40, 1.0);
    if (c128 < best_cost) { best = {false, 128}; best_cost = c128; }
    if (!b_mn) {
        const double c64 = cost(BM, 64, sms, 0.30, 0.5);
        if (c64 < best_cost) { best = {false, 64}; best_cost = c64; }
    }
    return best;
}

template <bool A_MN, bool B_MN>
fp8_status dispatch(const CUtensorMap& ta, GemmParams p, const HostArgs& h, cudaStream_t st) {
    const TileChoice tc = choose_tile(p.M, p.N, p.K, h.batch, B_MN, sm_count());
    const bool pair = tc.pair;
    const int bn = tc.bn;
    CUtensorMap tb;
    const uint64_t sb_bytes = uint64_t(h.stride_b);
    const uint32_t b_box_n = pair ? bn / 2 : bn;  // N extent one CTA loads
    const bool ok = B_MN ? make_map(&tb, h.b8, p.N, p.K, h.batch, sb_bytes, 128, BK)
                         : make_map(&tb, h.b8, p.K, p.N, h.batch, sb_bytes, BK, b_box_n);
    if (!ok) return FP8_ERR_CUDA;
    if (pair) return launch<256, A_MN, B_MN, 6, 2>(ta, tb, p, h, st);
    if (bn == 256) return launch<256, A_MN, B_MN, 4, 1>(ta, tb, p, h, st);
    if (bn == 128) return launch<128, A_MN, B_MN, 6, 1>(ta, tb, p, h, st);
    if constexpr (!B_MN) return launch<64, A_MN, B_MN, 8, 1>(ta, tb, p, h, st);
    return FP8_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace fp8lite

using namespace fp8lite;

extern "C" fp8_status fp8_mm(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb, const float* sa,
                             const float* sb, fp8_layout layout, int64_t M, int64_t N, int64_t K, int64_t batch,
                             int64_t stride_a, int64_t stride_b, int64_t stride_c, const void* bias,
                             const float* bias_scale, fp8_fmt bias_fmt, void* out, void* stream) {
    if (!valid_fmt(fa) || !valid_fmt(fb)) return FP8_ERR_INVALID_ARG;
    if (layout != FP8_NT && layout != FP8_NN && layout != FP8_TN) return FP8_ERR_INVALID_ARG;
    if (!a8 || !b8 || !sa || !sb || !out) return FP8_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1 || batch < 1) return FP8_ERR_INVALID_ARG;
    if (stride_a < 0 || stride_b < 0 || stride_c < 0) return FP8_ERR_INVALID_ARG;
    if (bias_scale && !bias) return FP8_ERR_INVALID_ARG;
    if (bias && bias_scale && !valid_fmt(bias_fmt)) return FP8_ERR_INVALID_ARG;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) ||
        batch >= (int64_t(1) << 31))
        return FP8_ERR_UNSUPPORTED;
    if (batch > 1 && stride_c < M * N) return FP8_ERR_INVALID_ARG;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + 63) / 64) * batch;
    if (tiles >= (int64_t(1) << 31)) return FP8_ERR_UNSUPPORTED;

    const bool a_mn = layout == FP8_TN;
    const bool b_mn = layout != FP8_NT;
    // contiguous extent of each operand = TMA row pitch in bytes
    const int64_t a_pitch = a_mn ? M : K;
    const int64_t b_pitch = b_mn ? N : K;
    if (a_pitch % 16 != 0 || b_pitch % 16 != 0) return FP8_ERR_ALIGNMENT;
    if (!aligned(a8, 16) || !aligned(b8, 16)) return FP8_ERR_ALIGNMENT;
    if (stride_a % 16 != 0 || stride_b % 16 != 0) return FP8_ERR_ALIGNMENT;
    if (!aligned(out, 4) || !aligned(sa, 4) || !aligned(sb, 4)) return FP8_ERR_ALIGNMENT;
    if (bias && !bias_scale && !aligned(bias, 2)) return FP8_ERR_ALIGNMENT;
    if (batch == 1) { stride_a = 0; stride_b = 0; }

    GemmParams p = {};
    p.M = int(M);
    p.N = int(N);
    p.K = int(K);
    p.k_blocks = int((K + BK - 1) / BK);
    p.a_bcast = stride_a == 0;
    p.b_bcast = stride_b == 0;
    p.sa = sa;
    p.sb = sb;
    p.bias = bias;
    p.bias_scale = bias_scale;
    p.bias_kind = bias ? (bias_scale ? 2 : 1) : 0;
    p.bias_fmt = bias_fmt;
    p.out = static_cast<uint16_t*>(out);
    p.stride_c = stride_c;
    p.vec_store = (N % 8 == 0) && (stride_c % 8 == 0) && aligned(out, 16);
    p.tma_store = p.vec_store;

    CUtensorMap ta;
    bool ok = a_mn ? make_map(&ta, a8, M, K, batch, uint64_t(stride_a), 128, BK)
                   : make_map(&ta, a8, K, M, batch, uint64_t(stride_a), BK, BM);
    if (!ok) return FP8_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    const HostArgs h = {int(fa), int(fb), b8, batch, stride_b};
    switch (layout) {
        case FP8_NT: return dispatch<false, false>(ta, p, h, st);
        case FP8_NN: return dispatch<false, true>(ta, p, h, st);
        default:     return dispatch<true, true>(ta, p, h, st);
    }
}

extern "C" fp8_status fp8_last_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return FP8_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
    const uint32_t zero = 0;
    if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return FP8_ERR_CUDA;
    return v ? FP8_ERR_DEVICE_TIMEOUT : FP8_OK;
}

extern "C" fp8_status fp8_selftest_wait_timeout(uint32_t limit_us, void* stream) {
    if (limit_us == 0 || limit_us > 1000000u) return FP8_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 1, 0, as_stream(stream)>>>(uint64_t(limit_us) * 1000ull);
    return launch_status();
}
