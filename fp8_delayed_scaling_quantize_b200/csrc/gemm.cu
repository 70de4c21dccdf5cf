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
//    BM x BN = 128 x {64,128,256}, or 256 x 256 on an SM pair (tcgen05
//    cta_group::2, clusters of two, no TMA multicast), in groups of M-tile
//    rows walked M-fastest, so that the tiles running together share their
//    A and B panels in L2;
//  * 6 warps with fixed roles: warp 0 issues TMA loads (one lane), warp 1
//    owns TMEM and issues tcgen05.mma (one lane), warps 2-5 run the epilogue
//    (one per TMEM lane quarter);
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
//    bias in fp32 (one fma), one round-to-nearest-even to bf16, staged as
//    128 x 32 tiles in shared memory and written by one TMA store each (TMA
//    clips the M / N tails);
//  * short problems (M <= 32, NT and NN) swap the operands, C^T = B^T A^T,
//    so that C's few rows become an MMA N of 16 or 32;
//  * split K: a tile's k-blocks are shared by several CTAs, whose fp32
//    partials go through a caller workspace (the last CTA to finish adds
//    them), through the library's static scratch, or, for short problems
//    without a workspace, to split 0 of a cluster through distributed shared
//    memory; partials are always added in split order;
//  * grouped launches: up to 4 problems (a linear's dX and dW) share one
//    persistent grid, each work unit looking up its problem in a table;
//  * every mbarrier wait is bounded by a time limit; a wait that gives up
//    records FP8_ERR_DEVICE_TIMEOUT in the library's device error word and the
//    CTA stops issuing work and exits through the normal teardown.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace fp8lite {

__device__ uint32_t g_device_error = 0;

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 128;  // bytes = elements of K per stage
constexpr int kEpiThreads = 128;            // 4 epilogue warps, one per TMEM lane quarter
constexpr int kThreads = 64 + kEpiThreads;  // producer warp, MMA warp, epilogue
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
    // split K: every tile is `split` work units of up to kb_per k-blocks each
    int split, kb_per, total_units;
    // swapped short problems: the splits of a tile run as one cluster and the
    // others' fp32 partials reach split 0 through its shared memory (no workspace)
    int csplit;
    float* ws;         // fp32 partial slots: [tile][rank][split] x (128 x BN)
    uint32_t* ws_cnt;  // per (tile, rank): {units arrived, partials written}
    // FP8 output (fp8_mm_out8): format, delayed-scaling ring, the scale used, the amax
    int out_fmt;
    fp8_ring* out_ring;
    float* out_scale;
    float* out_amax;
};

// Grouped launch (fp8_mm_grouped): several independent problems share one
// persistent grid. Work units [unit_end of the previous entry, unit_end) are
// the tiles of entry i; each role looks its unit's entry up here. An entry is
// a problem, or a column range of one: the host may give a problem's last
// columns their own entry with 128-wide tiles, so that the tiles of the
// grid's last round are cheaper.
constexpr int kMaxGroup = FP8_MM_MAX_GROUP;
constexpr int kMaxEntries = kMaxGroup + 1;
struct GroupProblem {
    CUtensorMap ta, tb, tc;  // operand maps and the output's store map
    int M, N, k_blocks, m_tiles, n_tiles, unit_end;
    int a_mn, b_mn;
    uint32_t idesc;
    int bias_kind, bias_fmt, tma_store, vec_store;
    int bn, n_base;  // this entry's tile width (128 or the launch's BN) and first output column
    const float* sa;
    const float* sb;
    const void* bias;
    const float* bias_scale;
    uint16_t* out;
};
template <bool GROUP>
struct GroupTab {};  // single-problem launches carry no table
template <>
struct GroupTab<true> {
    GroupProblem q[kMaxEntries];
    int count;
};

// The i-th work unit of a CTA whose first unit is unit0, the persistent grid
// holding unit_step CTAs (pairs). A grouped launch walks its rounds in
// alternating directions: CTA c takes unit c of the first round, unit
// step-1-c of the second, and so on. Its units come longest K first, so the
// CTAs that drew the short tiles of one round take the first units of the
// next, and no CTA stacks a second tile on a long one while others idle.
template <bool GROUP>
__device__ __forceinline__ int unit_of(int i, int unit0, int unit_step) {
    return i * unit_step + ((GROUP && (i & 1)) ? unit_step - 1 - unit0 : unit0);
}

// The problem that work unit u of a grouped launch belongs to, and the
// unit's tile index within it.
__device__ __forceinline__ const GroupProblem& group_problem(const GroupTab<true>& g, int u, int& t) {
    int i = 0;
    while (i + 1 < g.count && u >= g.q[i].unit_end) ++i;
    t = i == 0 ? u : u - g.q[i - 1].unit_end;
    return g.q[i];
}

// Wait for phase `parity` of the mbarrier at `bar`, giving up after
// `limit_ns`: then the library's device error word is set and false returned.
__device__ __forceinline__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((i & 1023u) == 0 && globaltimer_ns() - t0 > limit_ns) {
            atomicOr(&g_device_error, 1u);
            return false;
        }
    }
}

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

// wait_bounded by every lane of a warp, with one verdict for all of them.
__device__ __forceinline__ bool wait_bounded_warp(uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, wait_bounded(bar, parity));
}

// True in one lane of the (fully active) warp.
__device__ __forceinline__ bool elect_one() {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r));
    return r != 0;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* ptr) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* ptr, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// Wait until the counter at `ptr` reaches `want`, giving up (device error
// word set, false returned) after `limit_ns`.
__device__ __forceinline__ bool wait_count(const uint32_t* ptr, uint32_t want, uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire_u32(ptr) >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(32);
        if (ld_acquire_u32(ptr) >= want) return true;
        if ((i & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) {
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

// Two fp32 values to a pair of FP8 codes (nearest-even, saturating), the
// first in the low byte.
__device__ __forceinline__ uint32_t cvt_fp8x2(int fmt, float lo, float hi) {
    uint16_t r;
    if (fmt == FP8_E4M3) asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    else                 asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
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
    // three 128-row x 32-column bf16 staging tiles (64-byte swizzle), used in
    // turn, so that a chunk waits only for the store two chunks back; 24 KB
    // in all, so that a waiting kernel's small blocks still fit on the SM
    // beside this CTA
    static constexpr int kStgBufs = 3;
    static constexpr int kStgBytes = BM * 32 * 2;
    static constexpr int kStgOffset = STAGES * kStageBytes;  // a multiple of 1024
    static constexpr int kBiasOffset = kStgOffset + kStgBufs * kStgBytes;  // BN fp32 bias values
    static constexpr int kBarOffset = kBiasOffset + BN * 4;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], then the TMEM slot and the split ticket
    static constexpr int kBytes = kBarOffset + (2 * STAGES + 4) * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
    static constexpr uint32_t kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;
    static_assert(kStgOffset % 1024 == 0, "staging tiles need 1024-byte alignment");
    static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
};

// The tile walk's scalars, read once into registers.
struct TileWalk {
    int m_tiles, n_tiles, group_m;
};

// Tile order: batch outermost; inside a batch, groups of `group_m` M-tile
// rows, walked M-fastest within the group, then N. A wave of concurrently
// running tiles then covers a compact block of rows and columns whose A and B
// panels stay resident in L2 (an M-fastest walk over all rows streams the
// whole A through L2 every wave).
__device__ __forceinline__ void tile_coords(int t, const TileWalk& w, int& mb, int& nb, int& b) {
    const int per_batch = w.m_tiles * w.n_tiles;
    b = t / per_batch;
    const int r = t - b * per_batch;
    const int per_group = w.group_m * w.n_tiles;
    const int g = r / per_group;
    const int first_m = g * w.group_m;
    const int rows = min(w.group_m, w.m_tiles - first_m);
    const int i = r - g * per_group;
    mb = first_m + i % rows;
    nb = i / rows;
}

// Keeps a value's computation (a kernel-parameter read) at this point of the
// program: the first read of each parameter is a slow constant-cache miss, so
// the kernel issues them all together while its set-up runs.
template <typename T>
__device__ __forceinline__ T pin(T v) {
    asm volatile("" : "+r"(v));
    return v;
}

// Named barrier 1: the epilogue warps.
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

// Barrier 1, returning whether any epilogue thread passed true.
__device__ __forceinline__ bool epilogue_bar_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, p;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(v)), "n"(kEpiThreads)
        : "memory");
    return r != 0;
}

// One 128 x 32 bf16 block of the epilogue: to the staging tile whose last
// store is known to have read it (64-byte swizzle: 16-byte piece j of row r at
// (j ^ (r / 2 mod 4)) * 16, so the 8 lanes of a store phase hit distinct
// banks), then one TMA store by the lead thread, which clips the M / N tails
// of the output. n_st counts the stores issued so far (they take the staging
// tiles in turn).
template <typename L>
__device__ __forceinline__ void stage_and_store(uint32_t stg0, int n_st, int row_in_tile, const float (&y)[32],
                                                bool store_lead, const CUtensorMap* map_c, int col0, int m0, int b) {
    const uint32_t stg = stg0 + uint32_t(n_st % L::kStgBufs) * L::kStgBytes;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t addr = stg + row_in_tile * 64 + ((j ^ ((row_in_tile >> 1) & 3)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pack_bf16x2(y[8 * j + 0], y[8 * j + 1])),
                     "r"(pack_bf16x2(y[8 * j + 2], y[8 * j + 3])), "r"(pack_bf16x2(y[8 * j + 4], y[8 * j + 5])),
                     "r"(pack_bf16x2(y[8 * j + 6], y[8 * j + 7]))
                     : "memory");
    }
    fence_proxy_async_smem();
    // the store two blocks back has read its tile, which the next block
    // reuses (only the newest store may still be reading); the barrier
    // publishes that and this block
    if (store_lead) bulk_wait_read<L::kStgBufs - 2>();
    epilogue_bar();
    if (store_lead) {
        tma_store_3d(map_c, stg, col0, m0, b);
        bulk_commit();
    }
}

// One kernel for both tile shapes: CTAS = 1 computes 128 x BN tiles per CTA;
// CTAS = 2 runs as clusters of two CTAs on two SMs computing 256 x BN tiles
// with tcgen05 cta_group::2 -- the leader issues the MMAs, each CTA loads its
// own 128 rows of A and BN/2 columns of B (halving each SM's operand
// traffic) and writes its own 128 output rows.
//
// Epilogue: 4 warps, one per TMEM lane quarter. Every 32 columns of the tile
// become a 128 x 32 bf16 tile in shared memory that one thread writes with a
// single TMA store (8 stores for a 128 x 256 tile).
//
// GROUP: the units are the tiles of up to kMaxEntries table entries (one SM
// per tile, no split, no batches); operand majors, maps, tile width, first
// column, scales, bias and output come from the entry of each unit, A_MN /
// B_MN only give the defaults and BN is the widest tile.
template <int BN, bool A_MN, bool B_MN, int STAGES, bool HAS_BIAS, int CTAS, bool SPLIT, bool SWAP, bool OUT8,
          bool GROUP = false>
__global__ void __maxnreg__(168)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_c, const GemmParams p,
                const __grid_constant__ GroupTab<GROUP> grp) {
    using L = Smem<BN, STAGES, CTAS>;
    static_assert(!(B_MN && CTAS == 2 && BN != 256), "MN-major B halves must be whole 128-byte atoms");
    static_assert(!GROUP || (CTAS == 1 && !SPLIT && !SWAP && !OUT8), "grouped launches use plain one-SM tiles");
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
    uint32_t* ticket_slot = tmem_slot + 1;  // split K: the epilogue's arrival ticket
    const uint32_t bar_red = smem_addr(tmem_slot + 2);  // cluster split: the other splits' partials are in
    float* s_bias = reinterpret_cast<float*>(smem + L::kBiasOffset);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = CTAS == 2 ? cluster_ctarank() : 0u;  // 0 = the pair's leader
    const bool leader = rank == 0;
    const int unit0 = blockIdx.x / CTAS;     // this CTA's first work unit (a pair shares it)
    const int unit_step = gridDim.x / CTAS;  // units advance by the number of CTAs (pairs)

    // every parameter the roles read, fetched together now
    const int total_units = pin(p.total_units);
    const int k_blocks = pin(p.k_blocks);
    const int split = SPLIT ? pin(p.split) : 1;  // without SPLIT the split-K code compiles away
    const int kb_per = SPLIT ? pin(p.kb_per) : k_blocks;
    const TileWalk walk = {pin(p.m_tiles), pin(p.n_tiles), pin(p.group_m)};
    const int a_bcast = pin(p.a_bcast), b_bcast = pin(p.b_bcast);
    const uint32_t idesc = pin(p.idesc);
    int M = pin(p.M), N = pin(p.N);  // per unit in a grouped launch
    int tma_store = pin(p.tma_store), vec_store = pin(p.vec_store);
    const int csplit = (SWAP && SPLIT) ? pin(p.csplit) : 0;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, CTAS * kEpiThreads);
        }
        if (csplit) mbar_init(bar_red, uint32_t(split - 1) * kEpiThreads);
        fence_mbar_init();
        if constexpr (GROUP) {
            for (int i = 0; i < grp.count; ++i) {
                tma_prefetch(&grp.q[i].ta);
                tma_prefetch(&grp.q[i].tb);
                if (grp.q[i].tma_store) tma_prefetch(&grp.q[i].tc);
            }
        } else {
            tma_prefetch(&tm_a);
            tma_prefetch(&tm_b);
            if (tma_store) tma_prefetch(&tm_c);
        }
    }
    if (warp == 1) {
        tmem_alloc<CTAS>(smem_addr(tmem_slot), L::kTmemCols);
        tmem_relinquish<CTAS>();
    }
    tc_fence_before();
    __syncthreads();
    // the cluster's barriers exist before any remote arrive
    if (CTAS == 2 || csplit) cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The prologue above overlaps the previous kernel's tail; operands,
    // scales and the output are touched only after it has completed. Each
    // role waits for it separately, so that the producer can work out its
    // first unit's tile (pure arithmetic on the parameters) before.

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        // The whole warp walks the units and waits on the barriers, so the
        // loop's values stay warp-uniform; one elected lane issues the loads.
        const bool issuer = elect_one();
        struct Plan {
            const CUtensorMap* map_a;
            const CUtensorMap* map_b;
            int kb0, kb1, m0, n0, ba, bb, ebn;
            uint32_t stage_tx;
            bool a_mn, b_mn;
        };
        // the loads of work unit u: maps, k-block range, tile origin, batch
        auto plan = [&](int u) {
            Plan pl;
            int t = u / split;
            pl.map_a = &tm_a;
            pl.map_b = &tm_b;
            pl.a_mn = A_MN;
            pl.b_mn = B_MN;
            TileWalk w = walk;
            int kbs = k_blocks;
            int n_base = 0;
            pl.ebn = BN;  // the unit's tile width
            if constexpr (GROUP) {
                const GroupProblem& q = group_problem(grp, u, t);
                pl.map_a = &q.ta;
                pl.map_b = &q.tb;
                pl.a_mn = q.a_mn;
                pl.b_mn = q.b_mn;
                w = {q.m_tiles, q.n_tiles, walk.group_m};
                kbs = q.k_blocks;
                pl.ebn = q.bn;
                n_base = q.n_base;
            }
            pl.kb0 = GROUP ? 0 : (u - t * split) * kb_per;
            pl.kb1 = GROUP ? kbs : min(k_blocks, pl.kb0 + kb_per);
            int mb, nb, b;
            tile_coords(t, w, mb, nb, b);
            pl.ba = a_bcast ? 0 : b;
            pl.bb = b_bcast ? 0 : b;
            pl.m0 = mb * BM * CTAS + int(rank) * BM;
            pl.n0 = n_base + nb * pl.ebn + int(rank) * (BN / CTAS);
            pl.stage_tx = GROUP ? uint32_t(L::kABytes + pl.ebn * BK) : uint32_t(L::kStageTx);
            return pl;
        };
        Plan pl = {};
        if (unit0 < total_units) pl = plan(unit0);  // before the wait: it reads no memory
        griddep_wait();
        griddep_launch();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int i = 0, u = unit0; u < total_units && ok;) {
            const CUtensorMap* map_a = pl.map_a;
            const CUtensorMap* map_b = pl.map_b;
            const bool a_mn = pl.a_mn, b_mn = pl.b_mn;
            const int kb0 = pl.kb0, kb1 = pl.kb1, m0 = pl.m0, n0 = pl.n0, ba = pl.ba, bb = pl.bb, ebn = pl.ebn;
            const uint32_t stage_tx = pl.stage_tx;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!wait_bounded_warp(bar_empty + 8 * stage, phase ^ 1)) { ok = false; break; }
                const uint32_t full = bar_full + 8 * stage;
                const uint32_t da = s_a + stage * L::kABytes;
                const uint32_t db = s_b + stage * L::kBBytes;
                if (issuer) {
                    if (leader) mbar_arrive_expect_tx(full, stage_tx);
                    if (CTAS == 1) {
                        if (a_mn) tma_load_3d(da, map_a, full, m0, kb * BK, ba);
                        else      tma_load_3d(da, map_a, full, kb * BK, m0, ba);
                        if (b_mn) {
#pragma unroll
                            for (int h = 0; h < BN / 128; ++h)
                                if (h * 128 < ebn) tma_load_3d(db + h * 128 * BK, map_b, full, n0 + h * 128, kb * BK, bb);
                        } else {
                            tma_load_3d(db, map_b, full, kb * BK, n0, bb);
                        }
                    } else {
                        const uint32_t lfull = map_to_rank(full, 0);  // the leader's barrier
                        if (A_MN) tma_load_3d_pair(da, &tm_a, lfull, m0, kb * BK, ba);
                        else      tma_load_3d_pair(da, &tm_a, lfull, kb * BK, m0, ba);
                        if (B_MN) tma_load_3d_pair(db, &tm_b, lfull, n0, kb * BK, bb);
                        else      tma_load_3d_pair(db, &tm_b, lfull, kb * BK, n0, bb);
                    }
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            u = unit_of<GROUP>(++i, unit0, unit_step);
            if (u < total_units) pl = plan(u);
        }
        // drain: wait until the MMAs released every stage still in use
        for (int i = 0; i < STAGES && ok; ++i) {
            if (!wait_bounded_warp(bar_empty + 8 * stage, phase ^ 1)) break;
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer ---
        griddep_wait();
        griddep_launch();
        // As the producer: the warp walks and waits together, one elected
        // lane issues every MMA and commit (a commit tracks the MMAs of the
        // thread that issues it, so it is always the same lane).
        const bool issuer = elect_one();
        if (leader) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int u = unit0; u < total_units && ok; u = unit_of<GROUP>(++it, unit0, unit_step)) {
                int t = u / split;
                bool a_mn = A_MN, b_mn = B_MN;
                uint32_t id = idesc;
                int kbs = k_blocks;
                if constexpr (GROUP) {
                    const GroupProblem& q = group_problem(grp, u, t);
                    a_mn = q.a_mn;
                    b_mn = q.b_mn;
                    id = q.idesc;
                    kbs = q.k_blocks;
                }
                const int kb0 = GROUP ? 0 : (u - t * split) * kb_per;
                const int kb1 = GROUP ? kbs : min(k_blocks, kb0 + kb_per);
                const int buf = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!wait_bounded_warp(bar_tempty + 8 * buf, acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                const uint64_t a_desc0 = a_mn ? smem_desc_sw128(s_a, 128 * BK, 1024) : smem_desc_sw128(s_a, 16, 1024);
                const uint64_t b_desc0 = b_mn ? smem_desc_sw128(s_b, 128 * BK, 1024) : smem_desc_sw128(s_b, 16, 1024);
                const uint64_t a_step = a_mn ? 256u : 2u, b_step = b_mn ? 256u : 2u;
                for (int kb = kb0; kb < kb1; ++kb) {
                    // the stage's operands arrive through the async proxy and
                    // complete on this barrier: the MMAs may read them without
                    // a tcgen05 fence (that is needed only after the epilogue's
                    // hand-back of the accumulator, above)
                    if (!wait_bounded_warp(bar_full + 8 * stage, phase)) { ok = false; break; }
                    // the stage's descriptors: stage 0's plus the stage offset in
                    // the start-address field (16-byte units; no carry out of it,
                    // shared memory is below 256 KB). Each next 32-deep K slice is
                    // +32 bytes inside the swizzle atom (K-major) or 32 rows of
                    // 128 bytes further (MN-major).
                    const uint64_t adesc = a_desc0 + uint64_t(stage) * (L::kABytes >> 4);
                    const uint64_t bdesc = b_desc0 + uint64_t(stage) * (L::kBBytes >> 4);
                    if (issuer) {
                        mma_kblock_f8f6f4<CTAS>(d_tmem, adesc, bdesc, a_step, b_step, id, kb != kb0);
                        // release the stage (in both CTAs of a pair)
                        if (CTAS == 1) mma_commit(bar_empty + 8 * stage);
                        else           mma_commit_pair(bar_empty + 8 * stage);
                    }
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (issuer) {
                    if (CTAS == 1) mma_commit(bar_tfull + 8 * buf);
                    else           mma_commit_pair(bar_tfull + 8 * buf);
                }
                __syncwarp();
            }
        }
    } else {
        // ----------------------------------------------------- epilogue ---
        griddep_wait();
        griddep_launch();
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int row_in_tile = q * 32 + lane;
        const int etid = threadIdx.x - 64;  // 0 .. kEpiThreads-1
        const bool store_lead = etid == 0;  // issues the TMA stores
        const uint32_t stg0 = s_base + L::kStgOffset;
        int n_st = 0;  // TMA stores issued so far (they take the staging tiles in turn)
        float inv = (1.0f / __ldg(p.sa)) * (1.0f / __ldg(p.sb));
        int bias_kind = p.bias_kind, bias_fmt = p.bias_fmt;
        const void* bias_ptr = p.bias;
        float bscale = (HAS_BIAS && bias_kind == 2) ? __ldg(p.bias_scale) : 1.0f;
        uint16_t* out_base = p.out;
        const CUtensorMap* map_c = &tm_c;
        // FP8 output: the ring's scale before this call (every CTA reads it
        // before any CTA can fold: the fold waits for all CTAs' tickets)
        float s_out = 1.0f, m_out = 0.0f;
        if (OUT8) {
            s_out = *reinterpret_cast<volatile float*>(&p.out_ring->scale);
            if (blockIdx.x == 0 && etid == 0) *p.out_scale = s_out;
        }
        bool failed = false;
        int it = 0;
        for (int u = unit0; u < total_units; u = unit_of<GROUP>(++it, unit0, unit_step)) {
            int t = u / split;
            const int split_id = u - t * split;
            TileWalk w = walk;
            int ebn = BN, n_base = 0;  // the unit's tile width and first column
            if constexpr (GROUP) {
                const GroupProblem& q = group_problem(grp, u, t);
                w = {q.m_tiles, q.n_tiles, walk.group_m};
                ebn = q.bn;
                n_base = q.n_base;
                M = q.M;
                N = q.N;
                tma_store = q.tma_store;
                vec_store = q.vec_store;
                map_c = &q.tc;
                out_base = q.out;
                bias_kind = q.bias_kind;
                bias_fmt = q.bias_fmt;
                bias_ptr = q.bias;
                inv = (1.0f / __ldg(q.sa)) * (1.0f / __ldg(q.sb));
                bscale = (HAS_BIAS && bias_kind == 2) ? __ldg(q.bias_scale) : 1.0f;
            }
            int mb, nb, b;
            tile_coords(t, w, mb, nb, b);
            const int buf = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            const int m0 = mb * BM * CTAS + int(rank) * BM;  // this CTA's first output row
            if (HAS_BIAS && !SWAP) {
                // the tile's BN bias values, dequantized once into shared memory
                epilogue_bar();  // the previous tile's readers are done
                for (int j = etid; j < ebn; j += kEpiThreads) {
                    const int col = n_base + nb * ebn + j;
                    float v = 0.0f;
                    if (col < N && bias_kind != 0) {  // a grouped launch may mix problems with and without bias
                        if (bias_kind == 1) {
                            v = __uint_as_float(uint32_t(__ldg(static_cast<const uint16_t*>(bias_ptr) + col)) << 16);
                        } else {
                            v = __fdiv_rn(fp8_to_f32(__ldg(static_cast<const uint8_t*>(bias_ptr) + col), bias_fmt),
                                          bscale);
                        }
                    }
                    s_bias[j] = v;
                }
                epilogue_bar();
            }
            // every lane waits, then all epilogue warps agree (and each warp
            // reconverges) before the warp-collective TMEM loads. After a wait
            // gave up, they all keep walking the units without waiting, so that
            // they still meet at every named barrier.
            if (!failed) failed = !wait_bounded(bar_tfull + 8 * buf, acc_phase);
            failed = epilogue_bar_or(failed);
            if (failed) continue;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (uint32_t(q * 32) << 16) + buf * BN;
            // Split K: the unit that arrives last at its tile finishes it; the
            // others leave their fp32 partial in the workspace. Slot layout:
            // 16-byte piece v of CW-column chunk c of tile row r sits at
            // ((c * CW / 4 + v) * 128 + r) * 16, so each store and load
            // instruction of a warp covers 512 contiguous bytes.
            constexpr int CW = SWAP ? 16 : 32;  // accumulator columns per TMEM load
            const float4* slots = nullptr;
            if (SPLIT && split > 1 && csplit) {
                // cluster split: CTA r of the cluster is split r of the tile
                // (one tile per cluster); splits 1.. push their partials into
                // split 0's staging area (free in swapped launches), slot r - 1,
                // laid out as the workspace's slots, and arrive on its barrier
                if (split_id != 0) {
                    const uint32_t dst = map_to_rank(stg0 + uint32_t(split_id - 1) * (BM * BN * 4), 0);
#pragma unroll 1
                    for (int c = 0; c < BN / CW; ++c) {
                        if (nb * BN + c * CW >= N) break;  // uniform; split 0 skips it too
                        uint32_t r[CW];
                        tmem_ld<CW>(t_row + c * CW, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int v = 0; v < CW / 4; ++v)
                            st_cluster_v4(dst + uint32_t(((c * (CW / 4) + v) * 128 + row_in_tile) * 16),
                                          __uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                          __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
                    }
                    mbar_arrive_cluster(map_to_rank(bar_red, 0));  // release: the stores above come first
                    tc_fence_before();
                    mbar_arrive(bar_tempty + 8 * buf);
                    continue;
                }
                if (!failed) failed = !wait_bounded_cluster(bar_red, 0);
                failed = epilogue_bar_or(failed);
                if (failed) continue;
            } else if (SPLIT && split > 1) {
                uint32_t* cnt = p.ws_cnt + 2 * (t * CTAS + int(rank));
                slots = reinterpret_cast<const float4*>(p.ws) + size_t(t * CTAS + int(rank)) * split * (BM * BN / 4);
                if (etid == 0) *ticket_slot = atomicAdd(cnt, 1u);
                epilogue_bar();
                const bool last = *ticket_slot == uint32_t(split - 1);
                if (!last) {
                    float4* mine = const_cast<float4*>(slots) + size_t(split_id) * (BM * BN / 4);
#pragma unroll 1
                    for (int c = 0; c < BN / CW; ++c) {
                        if (nb * BN + c * CW >= N) break;  // uniform; the finisher skips it too
                        uint32_t r[CW];
                        tmem_ld<CW>(t_row + c * CW, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int v = 0; v < CW / 4; ++v)
                            __stcg(mine + (c * (CW / 4) + v) * 128 + row_in_tile,
                                   make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                               __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                    }
                    __threadfence();
                    epilogue_bar();
                    if (etid == 0) red_release_add(cnt + 1, 1u);
                    tc_fence_before();
                    if (CTAS == 1) mbar_arrive(bar_tempty + 8 * buf);
                    else           mbar_arrive_cluster(map_to_rank(bar_tempty + 8 * buf, 0));
                    continue;
                }
                if (etid == 0) {
                    wait_count(cnt + 1, uint32_t(split - 1));
                    cnt[0] = 0u;  // the tile's counters are ready for the next call
                    cnt[1] = 0u;
                }
                epilogue_bar();
            }
            const int row = m0 + row_in_tile;
            // swapped operands: this thread's TMEM lane is output column `row`
            // of C (the kernel's M is C's N), its accumulator columns are C's rows
            float bias_row = 0.0f;
            if (SWAP && HAS_BIAS && row < M) {
                if (bias_kind == 1)
                    bias_row = __uint_as_float(uint32_t(__ldg(static_cast<const uint16_t*>(bias_ptr) + row)) << 16);
                else
                    bias_row = __fdiv_rn(fp8_to_f32(__ldg(static_cast<const uint8_t*>(bias_ptr) + row), bias_fmt),
                                         bscale);
            }
            uint16_t* orow = SWAP ? out_base + int64_t(b) * p.stride_c + row
                                  : out_base + int64_t(b) * p.stride_c + int64_t(row) * N;
            if constexpr (!SPLIT && !SWAP && !OUT8) {
                if (tma_store) {
                    // The common case, pipelined: chunk c + 1's accumulator
                    // columns leave TMEM while chunk c is converted, staged and
                    // stored (two register sets, the wait tied to the set it
                    // waits for).
                    const int col_first = n_base + nb * ebn;
                    const int left = (N - col_first + 31) / 32;
                    const int nch = left < ebn / 32 ? left : ebn / 32;
                    auto emit = [&](const uint32_t (&r)[32], int c) {
                        float y[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const float bias = HAS_BIAS ? s_bias[c * 32 + i] : 0.0f;
                            y[i] = fmaf(__uint_as_float(r[i]), inv, bias);
                        }
                        stage_and_store<L>(stg0, n_st, row_in_tile, y, store_lead, map_c, col_first + c * 32, m0, b);
                        ++n_st;
                    };
                    uint32_t ra[32], rb[32];
                    tmem_ld<32>(t_row, ra);
                    tmem_ld_wait_tied(ra);
#pragma unroll 1
                    for (int c = 0; c < nch; c += 2) {
                        __syncwarp();
                        if (c + 1 < nch) tmem_ld<32>(t_row + (c + 1) * 32, rb);
                        emit(ra, c);
                        if (c + 1 >= nch) break;
                        tmem_ld_wait_tied(rb);
                        __syncwarp();
                        if (c + 2 < nch) tmem_ld<32>(t_row + (c + 2) * 32, ra);
                        emit(rb, c + 1);
                        if (c + 2 < nch) tmem_ld_wait_tied(ra);
                    }
                    tc_fence_before();
                    if (CTAS == 1) mbar_arrive(bar_tempty + 8 * buf);
                    else           mbar_arrive_cluster(map_to_rank(bar_tempty + 8 * buf, 0));
                    continue;
                }
            }
#pragma unroll 1
            for (int c = 0; c < ebn / CW; ++c) {
                const int col0 = n_base + nb * ebn + c * CW;
                if (col0 >= N) break;  // uniform over the epilogue warps
                uint32_t r[CW];
                tmem_ld<CW>(t_row + c * CW, r);
                tmem_ld_wait();
                if (SPLIT && split > 1) {
                    // the sum over the splits in split order, whatever order
                    // they arrived in (the result does not depend on timing)
                    float acc[CW];
#pragma unroll 1
                    for (int sp = 0; sp < split; ++sp) {
                        if (sp == split_id) {
#pragma unroll
                            for (int i = 0; i < CW; ++i)
                                acc[i] = sp == 0 ? __uint_as_float(r[i]) : acc[i] + __uint_as_float(r[i]);
                        } else if (csplit) {
                            const uint32_t src = stg0 + uint32_t(sp - 1) * (BM * BN * 4) +
                                                 uint32_t(((c * (CW / 4)) * 128 + row_in_tile) * 16);
#pragma unroll
                            for (int v = 0; v < CW / 4; ++v) {
                                float4 x;
                                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                             : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                                             : "r"(src + uint32_t(v * 128 * 16)));
                                acc[4 * v] = acc[4 * v] + x.x;
                                acc[4 * v + 1] = acc[4 * v + 1] + x.y;
                                acc[4 * v + 2] = acc[4 * v + 2] + x.z;
                                acc[4 * v + 3] = acc[4 * v + 3] + x.w;
                            }
                        } else {
                            const float4* src =
                                slots + size_t(sp) * (BM * BN / 4) + c * (CW / 4) * 128 + row_in_tile;
#pragma unroll
                            for (int v = 0; v < CW / 4; ++v) {
                                const float4 x = __ldcg(src + v * 128);
                                acc[4 * v] = sp == 0 ? x.x : acc[4 * v] + x.x;
                                acc[4 * v + 1] = sp == 0 ? x.y : acc[4 * v + 1] + x.y;
                                acc[4 * v + 2] = sp == 0 ? x.z : acc[4 * v + 2] + x.z;
                                acc[4 * v + 3] = sp == 0 ? x.w : acc[4 * v + 3] + x.w;
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < CW; ++i) r[i] = __float_as_uint(acc[i]);
                }
                if constexpr (SWAP) {
                    // C[col0 + i][row]: lanes hold consecutive columns, so each
                    // store instruction of a warp writes 64 contiguous bytes
                    if (row < M) {
#pragma unroll
                        for (int i = 0; i < CW; ++i) {
                            if (col0 + i >= N) break;
                            const float y = fmaf(__uint_as_float(r[i]), inv, bias_row);
                            uint16_t h;
                            asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(y));
                            orow[int64_t(col0 + i) * M] = h;
                        }
                    }
                } else {
                    float y[CW];
#pragma unroll
                    for (int i = 0; i < CW; ++i) {
                        const float bias = HAS_BIAS ? s_bias[c * CW + i] : 0.0f;
                        y[i] = fmaf(__uint_as_float(r[i]), inv, bias);
                    }
                    if constexpr (OUT8) {
                        // q = sat_rne(fp32(y * s_out)); the amax is over the
                        // unquantized y of this call's own outputs only
                        if (row < M) {
                            uint32_t w[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
#pragma unroll
                                for (int k = 0; k < 4; ++k)
                                    if (col0 + 4 * j + k < N) m_out = fmaxf(m_out, fabsf(y[4 * j + k]));
                                w[j] = cvt_fp8x2(p.out_fmt, __fmul_rn(y[4 * j], s_out), __fmul_rn(y[4 * j + 1], s_out)) |
                                       (cvt_fp8x2(p.out_fmt, __fmul_rn(y[4 * j + 2], s_out),
                                                  __fmul_rn(y[4 * j + 3], s_out)) << 16);
                            }
                            uint8_t* dst = reinterpret_cast<uint8_t*>(out_base) + int64_t(b) * p.stride_c +
                                           int64_t(row) * N + col0;
                            if (vec_store && col0 + 32 <= N) {
                                reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
                                reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
                            } else {
#pragma unroll
                                for (int i = 0; i < 32; ++i)
                                    if (col0 + i < N) dst[i] = uint8_t(w[i >> 2] >> (8 * (i & 3)));
                            }
                        }
                    } else if (tma_store) {
                        // the 128 x 32 bf16 block goes to the staging tile whose last
                        // store is known to have read it (64-byte swizzle: 16-byte
                        // piece j of row r at (j ^ (r / 2 mod 4)) * 16, so the 8
                        // lanes of a store phase hit distinct banks); then one TMA
                        // store, which clips the M / N tails of the output
                        const uint32_t stg = stg0 + uint32_t(n_st % L::kStgBufs) * L::kStgBytes;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t addr = stg + row_in_tile * 64 + ((j ^ ((row_in_tile >> 1) & 3)) << 4);
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                         "r"(pack_bf16x2(y[8 * j + 0], y[8 * j + 1])),
                                         "r"(pack_bf16x2(y[8 * j + 2], y[8 * j + 3])),
                                         "r"(pack_bf16x2(y[8 * j + 4], y[8 * j + 5])),
                                         "r"(pack_bf16x2(y[8 * j + 6], y[8 * j + 7]))
                                         : "memory");
                        }
                        fence_proxy_async_smem();
                        // the store two blocks back has read its tile, which the next
                        // block reuses (only the newest store may still be reading);
                        // the barrier publishes that and this block
                        if (store_lead) bulk_wait_read<L::kStgBufs - 2>();
                        epilogue_bar();
                        if (store_lead) {
                            tma_store_3d(map_c, stg, col0, m0, b);
                            bulk_commit();
                        }
                        ++n_st;
                    } else if (row < M) {
                        if (vec_store && col0 + 32 <= N) {
                            uint4* dst = reinterpret_cast<uint4*>(orow + col0);
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                uint4 x;
                                x.x = pack_bf16x2(y[8 * v + 0], y[8 * v + 1]);
                                x.y = pack_bf16x2(y[8 * v + 2], y[8 * v + 3]);
                                x.z = pack_bf16x2(y[8 * v + 4], y[8 * v + 5]);
                                x.w = pack_bf16x2(y[8 * v + 6], y[8 * v + 7]);
                                dst[v] = x;
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; i += 2) {
                                const uint32_t x = pack_bf16x2(y[i], y[i + 1]);
                                if (col0 + i < N) orow[col0 + i] = uint16_t(x & 0xFFFFu);
                                if (col0 + i + 1 < N) orow[col0 + i + 1] = uint16_t(x >> 16);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            // release the accumulator to the MMA issuer (the pair's leader)
            if (CTAS == 1) mbar_arrive(bar_tempty + 8 * buf);
            else           mbar_arrive_cluster(map_to_rank(bar_tempty + 8 * buf, 0));
        }
        // the staging tiles must outlive the stores that read them; the global
        // writes themselves complete with the grid (a dependent kernel's
        // griddepcontrol.wait and stream order both see them)
        if ((GROUP || tma_store) && store_lead) bulk_wait_read<0>();
        if constexpr (OUT8) {
            // the CTA's amax of the output: one atomicMax, then a ticket; the
            // CTA holding the last ticket folds it into the output's ring
            uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(m_out));
            epilogue_bar();  // the bias slots are free now
            uint32_t* red = reinterpret_cast<uint32_t*>(s_bias);
            if (lane == 0) red[q] = bits;
            epilogue_bar();
            if (etid == 0) {
                bits = max(max(red[0], red[1]), max(red[2], red[3]));
                fp8_ring* ring = p.out_ring;
                if (bits != 0u) atomicMax(&ring->amax_bits, bits);
                const uint32_t ticket = atom_add_acq_rel(&ring->ticket, 1u);
                if (ticket == gridDim.x - 1) {
                    volatile fp8_ring* rr = ring;
                    float h[FP8_RING_HISTORY];
                    const uint32_t idx = ring_read(rr, h);
                    const float a = __uint_as_float(atomicExch(&ring->amax_bits, 0u));
                    ring_fold(rr, h, idx, a, fmt_max(p.out_fmt));
                    if (p.out_amax) *p.out_amax = a;
                    rr->ticket = 0u;
                }
            }
        }
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

// 3-D map over the bf16 output (N, M, batch), 32-column x 128-row boxes with
// a 64-byte swizzle matching the epilogue's staging tiles.
bool make_out_map(CUtensorMap* map, void* base, uint64_t n, uint64_t m, uint64_t batch, uint64_t batch_stride_bytes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if (batch <= 1 || batch_stride_bytes == 0) {
        batch = 1;
        batch_stride_bytes = ((n * m * 2 + 15) / 16) * 16;
    }
    cuuint64_t dims[3] = {n, m, batch};
    cuuint64_t strides[2] = {n * 2, batch_stride_bytes};
    cuuint32_t box[3] = {32, uint32_t(BM), 1};
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

template <int BN, bool A_MN, bool B_MN, int STAGES, bool HAS_BIAS, int CTAS, bool SPLIT, bool SWAP, bool OUT8>
fp8_status launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, GemmParams p,
                      const HostArgs& h, cudaStream_t st) {
    using L = Smem<BN, STAGES, CTAS>;
    auto kern = fp8_gemm_kernel<BN, A_MN, B_MN, STAGES, HAS_BIAS, CTAS, SPLIT, SWAP, OUT8>;
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
    p.kb_per = (p.k_blocks + p.split - 1) / p.split;
    const int64_t work = tiles * p.split;
    p.total_units = int(work);
    const int64_t units_max = sm_count() / CTAS;
    const int units = int(work < units_max ? work : units_max);
    // a cluster split runs each tile's splits as one cluster (every unit in
    // the grid's one round, so the grid is a whole number of clusters)
    const int cluster = p.csplit ? p.split : CTAS;
    return launch_pdl(kern, units * CTAS, kThreads, L::kAlloc, st, cluster, ta, tb, tc, p, GroupTab<false>{});
}

template <int BN, bool A_MN, bool B_MN, int STAGES, int CTAS, bool SWAP = false, bool OUT8 = false>
fp8_status launch(const CUtensorMap& ta, const CUtensorMap& tb, GemmParams p, const HostArgs& h, cudaStream_t st) {
    CUtensorMap tc = {};
    if (p.tma_store && !make_out_map(&tc, p.out, p.N, p.M, h.batch, uint64_t(p.stride_c) * 2)) return FP8_ERR_CUDA;
    if constexpr (OUT8) {  // no split, no swap
        return p.bias_kind ? launch_one<BN, A_MN, B_MN, STAGES, true, CTAS, false, false, true>(ta, tb, tc, p, h, st)
                           : launch_one<BN, A_MN, B_MN, STAGES, false, CTAS, false, false, true>(ta, tb, tc, p, h, st);
    } else {
        if (p.split > 1)
            return p.bias_kind
                       ? launch_one<BN, A_MN, B_MN, STAGES, true, CTAS, true, SWAP, false>(ta, tb, tc, p, h, st)
                       : launch_one<BN, A_MN, B_MN, STAGES, false, CTAS, true, SWAP, false>(ta, tb, tc, p, h, st);
        return p.bias_kind ? launch_one<BN, A_MN, B_MN, STAGES, true, CTAS, false, SWAP, false>(ta, tb, tc, p, h, st)
                           : launch_one<BN, A_MN, B_MN, STAGES, false, CTAS, false, SWAP, false>(ta, tb, tc, p, h, st);
    }
}

// Tile choice for 148 SMs by a small cost model: a persistent grid walks
// ceil(units / CTAs) rounds of work units, each costing its k-blocks times
// the per-k-block time of that tile shape, plus the one epilogue left exposed
// at the end. The per-k-block and epilogue constants were fitted on B200 to
// this kernel: 128x256 0.48, 128x128 0.40, 128x64 0.30 and an SM pair's
// 256x256 0.43. While its tensor core runs, an SM takes in operands at about
// 65 bytes per clock, so a one-SM k-block costs more than its MMAs (a
// 128 x 128 k-block loads 32 KB for half the MMA work of a 128 x 256 one,
// which loads 48 KB), and the wider tile costs less per output. Pairs of
// 256 x 256 are used only with at least one such tile per SM (below that
// their coarser grain loses) and at least 16 k-blocks: with 4 or 8 (K = 512,
// 1024) each CTA's 128 x 256 epilogue outlasts its main loop and pairs lost
// to one SM's 128 x 256 on every shape measured (4096^2 x 1024 18.9 against
// 20.4 us, 64 x 512^3 16.2 against 19.3), while from 16 on they won
// (4096^2 x 2048 28.5 against 31.0). The pair's 256 x 128 tile (24 KB per SM per
// k-block) measured slower than one SM's 128 x 128 on the shapes it could
// serve and is not chosen.
//
// Split K (split_req >= 2, with a workspace): a tile becomes `split` units
// over consecutive k-block ranges; the unit that finishes last adds the
// others' fp32 partials and runs the epilogue. The automatic choice
// (split_req = 0) does not split these unswapped tiles: on every shape
// measured on B200 the partials' round trip through L2 cost more than the
// shorter main loop saved (short problems, swapped below, do split).
constexpr size_t kSplitCntBytes = 4096;  // two counters per (tile, CTA of the tile)
constexpr int kMaxSplit = 4;

struct TileChoice {
    bool pair;
    int bn;
    int split;  // 0: the requested split is not possible for this problem
};

inline size_t split_ws_bytes(int64_t tiles, int ctas, int bn, int split) {
    return kSplitCntBytes + size_t(tiles) * ctas * split * BM * bn * sizeof(float);
}

inline int64_t tile_count(int64_t M, int64_t N, int64_t batch, bool pair, int bn) {
    const int64_t rows = BM * (pair ? 2 : 1);
    return ((M + rows - 1) / rows) * ((N + bn - 1) / bn) * batch;
}

inline TileChoice choose_tile(int64_t M, int64_t N, int64_t K, int64_t batch, bool b_mn, int64_t sms,
                              int split_req) {
    const int64_t kb = (K + BK - 1) / BK;
    const int split = split_req < 2 ? 1 : split_req;
    const int64_t kb_per = (kb + split - 1) / split;
    if (split > 1 && (split - 1) * kb_per >= kb) return {false, 256, 0};  // every unit needs k-blocks
    auto cost = [&](bool pair, int bn, double t_k, double t_epi) {
        const int ctas = pair ? 2 : 1;
        const int64_t units = sms / ctas;
        const int64_t tiles = tile_count(M, N, batch, pair, bn);
        if (split > 1 && size_t(tiles) * ctas * 2 * sizeof(uint32_t) > kSplitCntBytes) return 1e30;
        const int64_t rounds = (tiles * split + units - 1) / units;
        return double(rounds) * double(kb_per) * t_k + t_epi;
    };
    if (split == 1 && M > BM && N > 128 && kb >= 16 && tile_count(M, N, batch, true, 256) >= sms)
        return {true, 256, 1};
    const bool pair_ok = M > BM;  // a pair's second CTA would hold only padding otherwise
    const TileChoice c[4] = {{false, 256, split}, {false, 128, split}, {false, 64, split}, {true, 256, split}};
    const double t[4] = {cost(false, 256, 0.48, 2.0), cost(false, 128, 0.40, 1.0),
                         b_mn ? 1e30 : cost(false, 64, 0.30, 0.5),
                         (split > 1 && pair_ok && N > 128) ? cost(true, 256, 0.43, 2.0) : 1e30};
    TileChoice best = {false, 256, 0};
    double best_cost = 1e30;
    for (int i = 0; i < 4; ++i)
        if (t[i] < best_cost) { best = c[i]; best_cost = t[i]; }
    // With at most 4 k-blocks a 128 x 256 tile's epilogue (about 2.1 us)
    // outlasts its main loop while a 128 x 128 tile's (about 1.1 us) does not,
    // so the rounds times the epilogue decide between the two widths. Measured
    // on B200 over ten such shapes, this picks the faster of them in every case
    // with a clear difference: 128 for 64 x 512^3 (15.1 us against 16.2) and
    // 4096^2 x 512 (14.1 against 14.7), 256 for 2048^2 x 256 (5.4 against 5.6)
    // and 4096 x 2048 x 128 (7.1 against 7.9), among others.
    if (!best.pair && (best.bn == 256 || best.bn == 128) && split == 1 && kb <= 4) {
        const int64_t r256 = (tile_count(M, N, batch, false, 256) + sms - 1) / sms;
        const int64_t r128 = (tile_count(M, N, batch, false, 128) + sms - 1) / sms;
        best = {false, double(r128) * 1.1 < double(r256) * 2.1 ? 128 : 256, 1};
    }
    return best;
}

template <bool A_MN, bool B_MN, bool OUT8 = false>
fp8_status dispatch(const CUtensorMap& ta, GemmParams p, const HostArgs& h, void* ws, size_t ws_bytes,
                    int split_req, cudaStream_t st) {
    const TileChoice tc = choose_tile(p.M, p.N, p.K, h.batch, B_MN, sm_count(), split_req);
    if (tc.split == 0) return FP8_ERR_UNSUPPORTED;
    const bool pair = tc.pair;
    const int bn = tc.bn;
    p.split = tc.split;
    if (tc.split > 1) {
        const int64_t tiles = tile_count(p.M, p.N, h.batch, pair, bn);
        if (!ws || ws_bytes < split_ws_bytes(tiles, pair ? 2 : 1, bn, tc.split)) return FP8_ERR_INVALID_ARG;
        p.ws_cnt = static_cast<uint32_t*>(ws);
        p.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kSplitCntBytes);
    }
    CUtensorMap tb;
    const uint64_t sb_bytes = uint64_t(h.stride_b);
    const uint32_t b_box_n = pair ? bn / 2 : bn;  // N extent one CTA loads
    const bool ok = B_MN ? make_map(&tb, h.b8, p.N, p.K, h.batch, sb_bytes, 128, BK)
                         : make_map(&tb, h.b8, p.K, p.N, h.batch, sb_bytes, BK, b_box_n);
    if (!ok) return FP8_ERR_CUDA;
    if (pair) return launch<256, A_MN, B_MN, 6, 2, false, OUT8>(ta, tb, p, h, st);
    if (bn == 256) return launch<256, A_MN, B_MN, 4, 1, false, OUT8>(ta, tb, p, h, st);
    if (bn == 128) return launch<128, A_MN, B_MN, 6, 1, false, OUT8>(ta, tb, p, h, st);
    if constexpr (!B_MN) return launch<64, A_MN, B_MN, 8, 1, false, OUT8>(ta, tb, p, h, st);
    return FP8_ERR_UNSUPPORTED;
}

// Swapped operands for short problems (M <= 32, N >= 128, NT or NN): the
// kernel computes C^T = B^T A^T, so that C's N runs along the tensor core's
// 128-row M and C's few rows become an MMA N of 16 or 32; the epilogue
// writes C transposed. (TN is excluded: its A would become an MN-major B
// operand narrower than a 128-byte swizzle atom. From 33 rows on, the
// unswapped 128 x 64 tile was as fast or faster on B200: at 64 x 8192 x 2048
// it keeps 128 SMs busy where the swapped 128 x 64 tiles keep 64.)
inline bool swap_ab(int64_t M, int64_t N, fp8_layout layout) {
    return M <= 32 && N >= 128 && layout != FP8_TN;
}

inline int swap_bn(int64_t M) { return M <= 16 ? 16 : 32; }

// The split a swapped problem takes (0: the requested split is impossible).
// Automatic (split_req 0): few 128-column tiles with a long K leave most SMs
// idle, and their partials are small (128 x 16..64 fp32), so splitting pays
// where the main loop it saves exceeds the fix-up: about 0.28 us per k-block
// saved against 2.2 + 0.02 * BN * split us, with every unit in one round (both
// constants measured on B200 over 1, 8, 16, 32 and 64-row problems).
inline int swap_split(int64_t M, int64_t N, int64_t K, int64_t batch, int split_req, int64_t sms) {
    const int64_t kb = (K + BK - 1) / BK;
    const int64_t tiles = ((N + BM - 1) / BM) * batch;
    auto possible = [&](int s) {
        const int64_t kb_per = (kb + s - 1) / s;
        return (s - 1) * kb_per < kb && size_t(tiles) * 2 * sizeof(uint32_t) <= kSplitCntBytes;
    };
    if (split_req == 1) return 1;
    if (split_req >= 2) return possible(split_req) ? split_req : 0;
    const int bn = swap_bn(M);
    int best = 1;
    double best_gain = 0.0;
    for (int s = 2; s <= kMaxSplit; ++s) {
        if (!possible(s) || tiles * s > sms) continue;
        const double gain = double(kb - (kb + s - 1) / s) * 0.28 - (2.2 + 0.02 * bn * s);
        if (gain > best_gain) { best = s; best_gain = gain; }
    }
    return best;
}

template <bool A_MN>
fp8_status dispatch_swap(const uint8_t* a8, int fa, const uint8_t* b8, int fb, int64_t M, int64_t N, int64_t K,
                         int64_t batch, int64_t stride_a, int64_t stride_b, GemmParams p, void* ws, size_t ws_bytes,
                         int split_req, cudaStream_t st) {
    const int bn = swap_bn(M);
    // The automatic choice without a workspace splits as a cluster: the
    // splits' partials go through split 0's staging area, which holds three
    // 128 x 16 partials or one 128 x 32 one.
    p.csplit = 0;
    if (split_req == 0 && !ws) {
        const int s_max = bn == 16 ? 4 : 2;
        int s = swap_split(M, N, K, batch, 0, sm_count());
        s = s > s_max ? s_max : s;
        p.split = s;
        p.csplit = s > 1;
    } else {
        p.split = swap_split(M, N, K, batch, split_req, sm_count());
    }
    if (p.split == 0) return FP8_ERR_UNSUPPORTED;
    if (p.split > 1 && !p.csplit) {
        const int64_t tiles = ((N + BM - 1) / BM) * batch;
        if (!ws || ws_bytes < split_ws_bytes(tiles, 1, bn, p.split)) {
            if (split_req >= 2) return FP8_ERR_INVALID_ARG;
            p.split = 1;  // an automatic split that does not fit the workspace is dropped
        }
    }
    if (p.split > 1 && !p.csplit) {
        p.ws_cnt = static_cast<uint32_t*>(ws);
        p.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kSplitCntBytes);
    }
    // the kernel's problem: M' = N rows of A' = B, N' = M columns of B' = A
    p.M = int(N);
    p.N = int(M);
    p.a_bcast = stride_b == 0;
    p.b_bcast = stride_a == 0;
    p.tma_store = 0;
    p.vec_store = 0;
    CUtensorMap ta, tb;
    const bool ok_a = A_MN ? make_map(&ta, b8, N, K, batch, uint64_t(stride_b), 128, BK)
                           : make_map(&ta, b8, K, N, batch, uint64_t(stride_b), BK, BM);
    const bool ok_b = make_map(&tb, a8, K, M, batch, uint64_t(stride_a), BK, uint32_t(bn));
    if (!ok_a || !ok_b) return FP8_ERR_CUDA;
    const HostArgs h = {fb, fa, a8, batch, stride_a};
    if (bn == 16) return launch<16, A_MN, false, 10, 1, true>(ta, tb, p, h, st);
    return launch<32, A_MN, false, 9, 1, true>(ta, tb, p, h, st);
}

}  // namespace
}  // namespace fp8lite

using namespace fp8lite;

namespace fp8lite {
namespace {

// The FP8 output of fp8_mm_out8 (none for the bf16 entry points).
inline int choose_group_bn(const int64_t* M, const int64_t* N, const int64_t* kb, int count, int64_t sms);
inline int choose_narrow_tail(const int64_t* M, const int64_t* N, const int64_t* kb, int count, int64_t sms);
fp8_status mm_grouped_impl(const fp8_mm_problem* probs, int32_t count, void* stream);

struct Out8 {
    bool on;
    fp8_fmt fmt;
    fp8_ring* ring;
    float* amax;
    float* scale;
};

fp8_status mm_impl(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb, const float* sa, const float* sb,
                   fp8_layout layout, int64_t M, int64_t N, int64_t K, int64_t batch, int64_t stride_a,
                   int64_t stride_b, int64_t stride_c, const void* bias, const float* bias_scale, fp8_fmt bias_fmt,
                   void* out, void* workspace, size_t workspace_bytes, int32_t split_k, const Out8& o8,
                   void* stream) {
    if (split_k < 0 || split_k > kMaxSplit) return FP8_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return FP8_ERR_ALIGNMENT;
    if (!valid_fmt(fa) || !valid_fmt(fb)) return FP8_ERR_INVALID_ARG;
    if (layout != FP8_NT && layout != FP8_NN && layout != FP8_TN) return FP8_ERR_INVALID_ARG;
    if (!a8 || !b8 || !sa || !sb || !out) return FP8_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1 || batch < 1) return FP8_ERR_INVALID_ARG;
    if (stride_a < 0 || stride_b < 0 || stride_c < 0) return FP8_ERR_INVALID_ARG;
    if (bias_scale && !bias) return FP8_ERR_INVALID_ARG;
    if (bias && bias_scale && !valid_fmt(bias_fmt)) return FP8_ERR_INVALID_ARG;
    if (o8.on && (!valid_fmt(o8.fmt) || !o8.ring || !o8.scale)) return FP8_ERR_INVALID_ARG;
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
    if (!aligned(out, o8.on ? 1 : 4) || !aligned(sa, 4) || !aligned(sb, 4)) return FP8_ERR_ALIGNMENT;
    if (bias && !bias_scale && !aligned(bias, 2)) return FP8_ERR_ALIGNMENT;
    if (o8.on && (!aligned(o8.ring, 4) || !aligned(o8.scale, 4) || !aligned(o8.amax, 4))) return FP8_ERR_ALIGNMENT;
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
    p.split = 1;
    if (o8.on) {  // byte codes, 16-byte vector stores where rows allow
        p.out_fmt = int(o8.fmt);
        p.out_ring = o8.ring;
        p.out_amax = o8.amax;
        p.out_scale = o8.scale;
        p.vec_store = (N % 16 == 0) && (stride_c % 16 == 0) && aligned(out, 16);
        p.tma_store = 0;
    } else {
        p.vec_store = (N % 8 == 0) && (stride_c % 8 == 0) && aligned(out, 16);
        p.tma_store = p.vec_store;
    }
    cudaStream_t st = as_stream(stream);
    // One problem whose 128 x 256 tiles leave the persistent grid's last round
    // part-empty runs as a grouped launch of one, where its rightmost columns
    // can take 128-wide tiles (choose_narrow_tail); the result is the same.
    if (!o8.on && batch == 1 && split_k <= 1 && !swap_ab(M, N, layout)) {
        const TileChoice tc = choose_tile(M, N, K, 1, b_mn, sm_count(), split_k);
        const int64_t kb1 = (K + BK - 1) / BK;
        // only where it was measured to win: at least 8 k-blocks and at most
        // two rounds of 256-wide tiles (NT 2048 x 3072 x 1024: 11.52 -> 11.01 us);
        // with more rounds or fewer k-blocks the plain 128 x 256 launch was
        // faster (4096^2 x 1024 18.9 against 21.6 us, 2048^2 x 256 5.4 against 5.6)
        if (!tc.pair && tc.bn == 256 && tc.split == 1 && kb1 >= 8 &&
            tile_count(M, N, 1, false, 256) <= 2 * int64_t(sm_count()) &&
            choose_group_bn(&M, &N, &kb1, 1, sm_count()) == 256 && choose_narrow_tail(&M, &N, &kb1, 1, sm_count()) > 0) {
            const fp8_mm_problem one = {a8, b8, sa, sb, bias, bias_scale, out, M, N, K,
                                        int32_t(fa), int32_t(fb), int32_t(layout), int32_t(bias_fmt)};
            return mm_grouped_impl(&one, 1, stream);
        }
    }
    if (!o8.on && swap_ab(M, N, layout))
        return layout == FP8_NN ? dispatch_swap<true>(a8, fa, b8, fb, M, N, K, batch, stride_a, stride_b, p, workspace,
                                                      workspace_bytes, split_k, st)
                                : dispatch_swap<false>(a8, fa, b8, fb, M, N, K, batch, stride_a, stride_b, p,
                                                       workspace, workspace_bytes, split_k, st);

    CUtensorMap ta;
    bool ok = a_mn ? make_map(&ta, a8, M, K, batch, uint64_t(stride_a), 128, BK)
                   : make_map(&ta, a8, K, M, batch, uint64_t(stride_a), BK, BM);
    if (!ok) return FP8_ERR_CUDA;
    const HostArgs h = {int(fa), int(fb), b8, batch, stride_b};
    if (o8.on) {
        switch (layout) {
            case FP8_NT: return dispatch<false, false, true>(ta, p, h, nullptr, 0, 1, st);
            case FP8_NN: return dispatch<false, true, true>(ta, p, h, nullptr, 0, 1, st);
            default:     return dispatch<true, true, true>(ta, p, h, nullptr, 0, 1, st);
        }
    }
    switch (layout) {
        case FP8_NT: return dispatch<false, false>(ta, p, h, workspace, workspace_bytes, split_k, st);
        case FP8_NN: return dispatch<false, true>(ta, p, h, workspace, workspace_bytes, split_k, st);
        default:     return dispatch<true, true>(ta, p, h, workspace, workspace_bytes, split_k, st);
    }
}


// ------------------------------------------------------- grouped launch ---

template <int BN, int STAGES, bool HAS_BIAS>
fp8_status launch_group(const GroupTab<true>& g, int total_units, cudaStream_t st) {
    using L = Smem<BN, STAGES, 1>;
    auto kern = fp8_gemm_kernel<BN, false, false, STAGES, HAS_BIAS, 1, false, false, false, true>;
    static bool attr_set[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return FP8_ERR_CUDA;
        attr_set[dev] = true;
    }
    // the kernel-wide parameters a grouped launch still reads: the unit
    // count, the walk's group height, and valid scale pointers for the
    // epilogue's set-up (every unit reloads its own problem's scales)
    GemmParams p = {};
    p.total_units = total_units;
    p.total_tiles = total_units;
    p.split = 1;
    p.group_m = 16;
    p.a_bcast = 1;
    p.b_bcast = 1;
    p.sa = g.q[0].sa;
    p.sb = g.q[0].sb;
    const int units = total_units < sm_count() ? total_units : sm_count();
    const CUtensorMap none = {};
    return launch_pdl(kern, units, kThreads, L::kAlloc, st, 1, none, none, none, p, g);
}

// Tile width of a grouped launch: the persistent grid hands out the units in
// rounds of `grid`, alternating direction (unit_of), so the launch lasts as
// long as its busiest CTA; this is that CTA's k-blocks (times the per-k-block
// cost of the tile width) plus one exposed epilogue, the same cost model as a
// single problem's choice. Past a few thousand units the rounds even out and
// the estimate is rounds x the longest K.
inline int choose_group_bn(const int64_t* M, const int64_t* N, const int64_t* kb, int count, int64_t sms) {
    constexpr int64_t kMaxSlots = 1024, kSimUnits = 8192;
    int best_bn = 256;
    double best = 1e30;
    for (int bn : {256, 128}) {
        const double t_k = bn == 256 ? 0.48 : 0.40, t_epi = bn == 256 ? 2.0 : 1.0;
        int64_t total = 0, kb_max = 0;
        for (int i = 0; i < count; ++i) {
            total += ((M[i] + BM - 1) / BM) * ((N[i] + bn - 1) / bn);
            kb_max = kb[i] > kb_max ? kb[i] : kb_max;
        }
        const int64_t slots = sms < kMaxSlots ? sms : kMaxSlots;
        const int64_t grid = total < slots ? total : slots;
        int64_t worst = 0;
        if (total > kSimUnits) {
            worst = ((total + grid - 1) / grid) * kb_max;
        } else {
            int64_t load[kMaxSlots] = {0};
            int64_t u = 0;
            for (int i = 0; i < count; ++i) {
                const int64_t tiles = ((M[i] + BM - 1) / BM) * ((N[i] + bn - 1) / bn);
                for (int64_t k = 0; k < tiles; ++k, ++u) {
                    const int64_t round = u / grid, pos = u - round * grid;
                    load[(round & 1) ? grid - 1 - pos : pos] += kb[i];
                }
            }
            for (int64_t c = 0; c < grid; ++c) worst = load[c] > worst ? load[c] : worst;
        }
        const double c = double(worst) * t_k + t_epi;
        if (c < best) { best = c; best_bn = bn; }
    }
    return best_bn;
}

// How many of the last problem's 256-wide column tiles (counted from its
// right edge) to run as 128-wide tiles in a 256-wide grouped launch. The
// launch's last round often holds fewer tiles than there are CTAs; a 128-wide
// tile costs about 0.28 us per k-block against 0.45 us for a 256-wide one
// (measured on B200 with this kernel), so narrower tiles at the end shorten
// the busiest CTA. Each choice is evaluated on the exact unit-to-CTA
// assignment (unit_of); 0 keeps every tile 256 wide.
inline int choose_narrow_tail(const int64_t* M, const int64_t* N, const int64_t* kb, int count, int64_t sms) {
    constexpr int64_t kMaxSlots = 1024, kSimUnits = 8192;
    const int last = count - 1;
    const int64_t n256 = (N[last] + 255) / 256;
    int best_k = 0;
    double best = 1e30;
    for (int64_t k = 0; k <= n256; ++k) {
        const int64_t n1 = (n256 - k) * 256;  // columns left 256 wide
        int64_t units[kMaxEntries], cost[kMaxEntries];  // per entry: tiles, and their cost in 0.01 us
        int e = 0;
        for (int i = 0; i < last; ++i, ++e) {
            units[e] = ((M[i] + BM - 1) / BM) * ((N[i] + 255) / 256);
            cost[e] = kb[i] * 45;
        }
        const int64_t mt = (M[last] + BM - 1) / BM;
        units[e] = mt * (n1 / 256);
        cost[e++] = kb[last] * 45;
        units[e] = mt * ((N[last] - n1 + 127) / 128);
        cost[e++] = kb[last] * 28;
        int64_t total = 0;
        for (int i = 0; i < e; ++i) total += units[i];
        if (total > kSimUnits) return 0;
        const int64_t slots = sms < kMaxSlots ? sms : kMaxSlots;
        const int64_t grid = total < slots ? total : slots;
        int64_t load[kMaxSlots] = {0};
        int64_t u = 0;
        for (int i = 0; i < e; ++i)
            for (int64_t t = 0; t < units[i]; ++t, ++u) {
                const int64_t round = u / grid, pos = u - round * grid;
                load[(round & 1) ? grid - 1 - pos : pos] += cost[i];
            }
        int64_t worst = 0;
        for (int64_t c = 0; c < grid; ++c) worst = load[c] > worst ? load[c] : worst;
        if (double(worst) < best - 1e-9) { best = double(worst); best_k = int(k); }
    }
    return best_k;
}

fp8_status mm_grouped_impl(const fp8_mm_problem* probs, int32_t count, void* stream) {
    if (!probs || count < 1 || count > kMaxGroup) return FP8_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) {
        const fp8_mm_problem& q = probs[i];
        if (!valid_fmt(q.fmt_a) || !valid_fmt(q.fmt_b)) return FP8_ERR_INVALID_ARG;
        if (q.layout != FP8_NT && q.layout != FP8_NN && q.layout != FP8_TN) return FP8_ERR_INVALID_ARG;
        if (!q.a8 || !q.b8 || !q.sa || !q.sb || !q.out) return FP8_ERR_INVALID_ARG;
        if (q.M < 1 || q.N < 1 || q.K < 1) return FP8_ERR_INVALID_ARG;
        if (q.bias_scale && !q.bias) return FP8_ERR_INVALID_ARG;
        if (q.bias && q.bias_scale && !valid_fmt(q.bias_fmt)) return FP8_ERR_INVALID_ARG;
        if (q.M >= (int64_t(1) << 31) || q.N >= (int64_t(1) << 31) || q.K >= (int64_t(1) << 31))
            return FP8_ERR_UNSUPPORTED;
        const bool a_mn = q.layout == FP8_TN, b_mn = q.layout != FP8_NT;
        if ((a_mn ? q.M : q.K) % 16 != 0 || (b_mn ? q.N : q.K) % 16 != 0) return FP8_ERR_ALIGNMENT;
        if (!aligned(q.a8, 16) || !aligned(q.b8, 16)) return FP8_ERR_ALIGNMENT;
        if (!aligned(q.out, 4) || !aligned(q.sa, 4) || !aligned(q.sb, 4)) return FP8_ERR_ALIGNMENT;
        if (q.bias && !q.bias_scale && !aligned(q.bias, 2)) return FP8_ERR_ALIGNMENT;
    }
    // longest K first: the first wave of the persistent grid starts the
    // tiles that take longest, the shorter ones fill in behind them
    int order[kMaxGroup];
    for (int i = 0; i < count; ++i) order[i] = i;
    std::stable_sort(order, order + count, [&](int x, int y) { return probs[x].K > probs[y].K; });
    int64_t M[kMaxGroup], N[kMaxGroup], kb[kMaxGroup];
    for (int i = 0; i < count; ++i) {
        M[i] = probs[order[i]].M;
        N[i] = probs[order[i]].N;
        kb[i] = (probs[order[i]].K + BK - 1) / BK;
    }
    const int bn = choose_group_bn(M, N, kb, count, sm_count());
    // entries: every problem with bn-wide tiles; in a 256-wide launch the last
    // problem's rightmost columns may form one more entry with 128-wide tiles
    const int narrow = bn == 256 ? choose_narrow_tail(M, N, kb, count, sm_count()) : 0;
    GroupTab<true> g = {};
    int64_t units = 0;
    bool any_bias = false;
    int e = 0;
    for (int i = 0; i < count; ++i) {
        const fp8_mm_problem& q = probs[order[i]];
        const bool a_mn = q.layout == FP8_TN, b_mn = q.layout != FP8_NT;
        // column ranges of this problem: [0, n1) at bn, [n1, N) at 128
        const int64_t n1 = (i == count - 1 && narrow > 0) ? ((q.N + 255) / 256 - narrow) * 256 : q.N;
        for (int part = 0; part < 2; ++part) {
            const int64_t c0 = part == 0 ? 0 : n1, c1 = part == 0 ? n1 : q.N;
            if (c1 <= c0) continue;
            const int ebn = part == 0 ? bn : 128;
            GroupProblem& d = g.q[e++];
            const bool ok = (a_mn ? make_map(&d.ta, q.a8, q.M, q.K, 1, 0, 128, BK)
                                  : make_map(&d.ta, q.a8, q.K, q.M, 1, 0, BK, BM)) &&
                            (b_mn ? make_map(&d.tb, q.b8, q.N, q.K, 1, 0, 128, BK)
                                  : make_map(&d.tb, q.b8, q.K, q.N, 1, 0, BK, uint32_t(ebn)));
            if (!ok) return FP8_ERR_CUDA;
            d.M = int(q.M);
            d.N = int(q.N);
            d.k_blocks = int(kb[i]);
            d.m_tiles = int((q.M + BM - 1) / BM);
            d.n_tiles = int((c1 - c0 + ebn - 1) / ebn);
            d.bn = ebn;
            d.n_base = int(c0);
            units += int64_t(d.m_tiles) * d.n_tiles;
            if (units >= (int64_t(1) << 31)) return FP8_ERR_UNSUPPORTED;
            d.unit_end = int(units);
            d.a_mn = a_mn;
            d.b_mn = b_mn;
            d.idesc = sm100::instr_desc_f8(q.fmt_a, q.fmt_b, a_mn, b_mn, BM, ebn);
            d.bias_kind = q.bias ? (q.bias_scale ? 2 : 1) : 0;
            d.bias_fmt = q.bias_fmt;
            any_bias = any_bias || q.bias;
            d.vec_store = (q.N % 8 == 0) && aligned(q.out, 16);
            d.tma_store = d.vec_store;
            if (d.tma_store && !make_out_map(&d.tc, q.out, q.N, q.M, 1, 0)) return FP8_ERR_CUDA;
            d.sa = q.sa;
            d.sb = q.sb;
            d.bias = q.bias;
            d.bias_scale = q.bias_scale;
            d.out = static_cast<uint16_t*>(q.out);
        }
    }
    g.count = e;
    cudaStream_t st = as_stream(stream);
    if (bn == 256)
        return any_bias ? launch_group<256, 4, true>(g, int(units), st) : launch_group<256, 4, false>(g, int(units), st);
    return any_bias ? launch_group<128, 6, true>(g, int(units), st) : launch_group<128, 6, false>(g, int(units), st);
}
}  // namespace
}  // namespace fp8lite

extern "C" fp8_status fp8_mm_ws(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb, const float* sa,
                                const float* sb, fp8_layout layout, int64_t M, int64_t N, int64_t K, int64_t batch,
                                int64_t stride_a, int64_t stride_b, int64_t stride_c, const void* bias,
                                const float* bias_scale, fp8_fmt bias_fmt, void* out, void* workspace,
                                size_t workspace_bytes, int32_t split_k, void* stream) {
    const Out8 none = {false, FP8_E4M3, nullptr, nullptr, nullptr};
    return mm_impl(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias, bias_scale,
                   bias_fmt, out, workspace, workspace_bytes, split_k, none, stream);
}

extern "C" fp8_status fp8_mm_out8(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb, const float* sa,
                                  const float* sb, fp8_layout layout, int64_t M, int64_t N, int64_t K, int64_t batch,
                                  int64_t stride_a, int64_t stride_b, int64_t stride_c, const void* bias,
                                  const float* bias_scale, fp8_fmt bias_fmt, fp8_fmt out_fmt, fp8_ring* out_ring,
                                  uint8_t* out8, float* out_amax, float* out_scale, void* stream) {
    const Out8 o8 = {true, out_fmt, out_ring, out_amax, out_scale};
    return mm_impl(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias, bias_scale,
                   bias_fmt, out8, nullptr, 0, 1, o8, stream);
}

extern "C" fp8_status fp8_mm(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb, const float* sa,
                             const float* sb, fp8_layout layout, int64_t M, int64_t N, int64_t K, int64_t batch,
                             int64_t stride_a, int64_t stride_b, int64_t stride_c, const void* bias,
                             const float* bias_scale, fp8_fmt bias_fmt, void* out, void* stream) {
    return fp8_mm_ws(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias, bias_scale,
                     bias_fmt, out, nullptr, 0, 0, stream);
}

extern "C" size_t fp8_mm_workspace_size(int64_t M, int64_t N, int64_t K, int64_t batch, fp8_layout layout,
                                        int32_t split_k) {
    if (M < 1 || N < 1 || K < 1 || batch < 1 || split_k < 0 || split_k > kMaxSplit) return 0;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || batch >= (int64_t(1) << 31))
        return 0;
    if (layout != FP8_NT && layout != FP8_NN && layout != FP8_TN) return 0;
    if (swap_ab(M, N, layout)) {
        const int split = swap_split(M, N, K, batch, split_k, sm_count());
        if (split < 2) return 0;
        return split_ws_bytes(((N + BM - 1) / BM) * batch, 1, swap_bn(M), split);
    }
    const TileChoice tc = choose_tile(M, N, K, batch, layout != FP8_NT, sm_count(), split_k);
    if (tc.split < 2) return 0;
    return split_ws_bytes(tile_count(M, N, batch, tc.pair, tc.bn), tc.pair ? 2 : 1, tc.bn, tc.split);
}

// Library-owned split-K scratch for fp8_mm_splitk_static: the counter block
// (kSplitCntBytes) followed by the fp32 partial tiles. One array per device
// that loads the library, held until the process exits, shared by every call
// on that device. Host code may not use the symbol itself as a pointer: on
// the host it names a stand-in, not device memory, so the device address is
// looked up once per device (scratch_address) and passed to the kernel.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;
__device__ __align__(256) uint8_t g_splitk_scratch[kStaticScratchBytes];

namespace fp8lite {
namespace {

// The scratch's device address on the current device, looked up on the first
// call made with that device current and kept for later calls. The lookup may
// load the library's GEMM module on that device, which stream capture does not
// allow: the first call on a device must come before any capture.
void* scratch_address() {
    constexpr int kMaxDevices = 64;
    static void* addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_splitk_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace
}  // namespace fp8lite

extern "C" fp8_status fp8_mm_splitk_static(const uint8_t* a8, fp8_fmt fa, const uint8_t* b8, fp8_fmt fb,
                                           const float* sa, const float* sb, fp8_layout layout, int64_t M, int64_t N,
                                           int64_t K, int64_t batch, int64_t stride_a, int64_t stride_b,
                                           int64_t stride_c, const void* bias, const float* bias_scale,
                                           fp8_fmt bias_fmt, void* out, int32_t split_k, void* stream) {
    if (split_k < 2 || split_k > kMaxSplit) return FP8_ERR_INVALID_ARG;
    const size_t need = fp8_mm_workspace_size(M, N, K, batch, layout, split_k);
    if (need > kStaticScratchBytes) return FP8_ERR_UNSUPPORTED;
    void* scratch = scratch_address();
    if (!scratch) return FP8_ERR_CUDA;
    // The counters must be zero when the GEMM starts. A completed call leaves
    // them zero, but a call whose bounded wait gave up may not; clearing them
    // on the caller's stream makes every call start clean. The partial tiles
    // need no clearing: each is written before it is read.
    if (need > 0 && cudaMemsetAsync(scratch, 0, kSplitCntBytes, as_stream(stream)) != cudaSuccess)
        return FP8_ERR_CUDA;
    // fp8_mm_ws validates the rest (and reports a split the problem cannot take)
    return fp8_mm_ws(a8, fa, b8, fb, sa, sb, layout, M, N, K, batch, stride_a, stride_b, stride_c, bias, bias_scale,
                     bias_fmt, out, scratch, kStaticScratchBytes, split_k, stream);
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

extern "C" fp8_status fp8_mm_grouped(const fp8_mm_problem* problems, int32_t count, void* stream) {
    return mm_grouped_impl(problems, count, stream);
}
