// Low-precision linear-layer GEMM on B200 (sm_100a): Y = A W^T in bf16 from
// FP8 (e4m3, one dequantisation scale per tensor) or MXFP4 operands.
//
// The page "Accelerating Diffusers and xDiT Image Generation with MXFP4 using
// AMD Quark on AMD Instinct MI350 GPUs" (sections "MXFP4 Quantization" and
// "MXFP4 Kernel") runs the DiT's linear layers as FP4 x FP4 GEMMs on MXFP4
// operands; the page "How to Scale Diffusion Inference Across AMD RDNA 4 GPUs"
// (section "Make the Model Fit Before Tuning Latency") runs them in FP8.
// A is the activation [M, K] (K contiguous), W the weight [N, K] (K
// contiguous), Y [M, N] bf16.
//
// Design: a persistent kernel on CTA pairs (clusters of 2, tcgen05
// cta_group::2).  A pair owns a 256 x 256 output tile at a time: each CTA
// loads its own 128 rows of A and 128 of the tile's 256 rows of W per K
// stage (so each SM streams half of the W tile), and the leader issues every
// MMA once with M = N = 256.  The fp32 accumulator lives in TMEM, double
// buffered, so the epilogue of one tile (TMEM -> registers -> bf16 ->
// swizzled shared staging -> TMA store) overlaps the MMAs of the next.
//
// Warps (per CTA): 0 TMA producer, 1 TMEM owner and (leader) MMA issuer,
// 2-5 epilogue (warp w reads TMEM lanes 32 (w % 4) .. + 31).
//
// Every mbarrier wait is bounded by a time limit; on expiry the kernel
// records an error word, the roles leave their loops and the CTAs exit after
// draining what they issued.
#pragma once
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dit_gemm {

using namespace dit;

constexpr int kBM = 128;             // rows of A per CTA (256 per pair)
constexpr int kBN = 256;             // output columns per pair tile
constexpr int kBNh = kBN / 2;        // rows of W each CTA loads
constexpr int kBKB = 128;            // K bytes per stage (one 128-byte swizzle row)
constexpr int kStages = 5;
constexpr int kStageA = kBM * kBKB;  // 16 KB
constexpr int kStageB = kBNh * kBKB; // 16 KB
constexpr int kThreads = 192;
constexpr int kEpiWarp0 = 2;
constexpr int kOBox = 64;            // output columns per TMA store box (128 bytes of bf16)
constexpr int kOStage = kBM * 128;   // one staging box: 128 rows x 128 bytes
constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 accumulators

enum : uint32_t { kSiteFull = 1, kSiteEmpty = 2, kSiteTmemFull = 3, kSiteTmemEmpty = 4 };
constexpr uint32_t kErrTimeout = 7;

__device__ unsigned int g_gemm_error_word;

struct GemmParams {
    int M, N, K;                 // K in elements
    int kb;                      // K stages: ceil(K bytes / 128)
    int m_tiles, n_tiles;        // ceil(M / 256), ceil(N / 256)
    float out_scale;             // FP8: a_scale * w_scale; MXFP4: 1
    unsigned long long wait_limit_ns;
};

struct Bars {
    uint64_t full[kStages];      // leader: stage s of both CTAs landed
    uint64_t empty[kStages];     // each CTA: the MMAs reading stage s completed
    uint64_t tfull[2];           // each CTA: accumulator b holds a finished tile
    uint64_t tempty[2];          // leader: both CTAs' epilogues have read accumulator b
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

struct Smem {
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + kStages * kStageA;
    static constexpr int OFF_O = OFF_B + kStages * kStageB;
    static constexpr int OFF_BAR = OFF_O + 2 * kOStage;
    static constexpr int BYTES = OFF_BAR + 256 + 1024;   // + alignment slack
};
static_assert(Smem::BYTES <= 232448, "shared memory budget");

// ------------------------------------------------------------------ PTX not in the attention wrappers

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar, int c0, int c1,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, uint32_t src, int c0, int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}

// Wait until at most N bulk store groups are still reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
                                         unsigned long long limit, uint32_t site)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (*abort)
            return false;
        if (globaltimer_ns() - t0 > limit) {
            atomicCAS(&g_gemm_error_word, 0u, (site << 8) | kErrTimeout);
            *abort = 1u;
            return false;
        }
    }
}

__device__ __forceinline__ void named_bar(uint32_t id, uint32_t n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool bar_and(uint32_t id, uint32_t nthreads, bool pred)
{
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return out != 0;
}

// ------------------------------------------------------------------ FP8 operand configuration

struct Fp8Kind {
    static constexpr int KSTEP_BYTES = 32;             // K = 32 e4m3 per MMA
    static constexpr int MMAS_PER_STAGE = kBKB / KSTEP_BYTES;
    static constexpr uint32_t IDESC = make_idesc(kFmtE4M3, kFmtE4M3, 0, 2 * kBM, kBN);
};

// ------------------------------------------------------------------ roles

struct Ctx {
    Bars *bars;
    uint32_t base, tmem, rank;
    volatile uint32_t *abort;
    unsigned long long lim;
    __device__ uint32_t bar(const uint64_t &b) const { return smem_u32(&b); }
    __device__ uint32_t leader_bar(const uint64_t &b) const { return mapa_shared(smem_u32(&b), 0); }
};

// Tiles are walked with the N tiles of one 256-row block of A consecutive, so
// the pairs that run at the same time share that A block through L2.
__device__ __forceinline__ void tile_coords(const GemmParams &p, int t, int &m0, int &n0)
{
    m0 = (t / p.n_tiles) * 2 * kBM;
    n0 = (t % p.n_tiles) * kBN;
}

template <class Kind>
__device__ __forceinline__ void producer(const Ctx &x, const GemmParams &p, const CUtensorMap *tm_a,
                                         const CUtensorMap *tm_w)
{
    const uint64_t pol_a = l2_policy_evict_first();
    const uint64_t pol_w = l2_policy_evict_last();
    const bool leader = x.rank == 0;
    const int tiles = p.m_tiles * p.n_tiles;
    int it = 0;
    for (int t = blockIdx.x / 2; t < tiles; t += gridDim.x / 2) {
        int m0, n0;
        tile_coords(p, t, m0, n0);
        for (int k = 0; k < p.kb; ++k, ++it) {
            const int s = it % kStages;
            if (it >= kStages &&
                !wait_bar(x.bar(x.bars->empty[s]), ((it / kStages) - 1) & 1, x.abort, x.lim, kSiteEmpty))
                return;
            if (leader)
                mbar_arrive_expect_tx(x.bar(x.bars->full[s]), 2 * (kStageA + kStageB));
            const uint32_t full = x.leader_bar(x.bars->full[s]);
            tma_load_2d_pair(x.base + Smem::OFF_A + s * kStageA, tm_a, full, k * kBKB, m0 + (int)x.rank * kBM, pol_a);
            tma_load_2d_pair(x.base + Smem::OFF_B + s * kStageB, tm_w, full, k * kBKB, n0 + (int)x.rank * kBNh,
                             pol_w);
        }
    }
}

template <class Kind>
__device__ __forceinline__ void mma_issuer(const Ctx &x, const GemmParams &p)
{
    constexpr uint16_t kBoth = 0x3;
    const uint32_t base = __shfl_sync(0xffffffffu, x.base, 0);
    const uint32_t tmem = __shfl_sync(0xffffffffu, x.tmem, 0);
    const uint64_t a_desc = make_smem_desc(base + Smem::OFF_A, 16, 8 * 128, kSwizzle128B);
    const uint64_t b_desc = make_smem_desc(base + Smem::OFF_B, 16, 8 * 128, kSwizzle128B);
    const int tiles = p.m_tiles * p.n_tiles;
    bool ok = true;
    int it = 0, local = 0;
    for (int t = blockIdx.x / 2; t < tiles && ok; t += gridDim.x / 2, ++local) {
        const int b = local & 1;
        if (local >= 2)
            ok = __all_sync(0xffffffffu, wait_bar(x.bar(x.bars->tempty[b]), ((local >> 1) - 1) & 1, x.abort,
                                                  x.lim, kSiteTmemEmpty));
        if (!ok)
            break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(b * kBN);
        for (int k = 0; k < p.kb && ok; ++k, ++it) {
            const int s = it % kStages;
            ok = __all_sync(0xffffffffu,
                            wait_bar(x.bar(x.bars->full[s]), (it / kStages) & 1, x.abort, x.lim, kSiteFull));
            if (!ok)
                break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < Kind::MMAS_PER_STAGE; ++kk) {
                const uint64_t ad = a_desc + ((uint32_t)(s * kStageA + kk * Kind::KSTEP_BYTES) >> 4);
                const uint64_t bd = b_desc + ((uint32_t)(s * kStageB + kk * Kind::KSTEP_BYTES) >> 4);
                if (elect_one())
                    mma2_f8_ss(acc, ad, bd, Kind::IDESC, (k > 0 || kk > 0) ? 1u : 0u);
            }
            if (elect_one())
                mma2_commit_mc(x.bar(x.bars->empty[s]), kBoth);
            __syncwarp();
        }
        if (ok && elect_one())
            mma2_commit_mc(x.bar(x.bars->tfull[b]), kBoth);
        __syncwarp();
    }
    if (!ok) {
        if (elect_one())
            mma2_commit(x.bar(x.bars->drain));
        __syncwarp();
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(x.bar(x.bars->drain), 0) && globaltimer_ns() - t0 < 50000000ull) {
        }
    }
}

// Epilogue: 128 threads, thread r of this CTA's tile owns output row m0 + r
// and TMEM lane r.  Per 64-column box: 2 TMEM loads, scale, bf16, 128 bytes
// into the swizzled staging box, one TMA store (clipped at M and N).
__device__ __forceinline__ void epilogue(const Ctx &x, const GemmParams &p, const CUtensorMap *tm_y, int warp,
                                         int lane)
{
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool issuer = warp == kEpiWarp0 && lane == 0;
    const int tiles = p.m_tiles * p.n_tiles;
    const uint32_t tempty_leader[2] = {x.leader_bar(x.bars->tempty[0]), x.leader_bar(x.bars->tempty[1])};
    bool ok = true;
    int local = 0, box = 0;
    for (int t = blockIdx.x / 2; t < tiles && ok; t += gridDim.x / 2, ++local) {
        const int b = local & 1;
        int m0, n0;
        tile_coords(p, t, m0, n0);
        ok = __all_sync(0xffffffffu,
                        wait_bar(x.bar(x.bars->tfull[b]), (local >> 1) & 1, x.abort, x.lim, kSiteTmemFull));
        if (!bar_and(1, 128, ok)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const uint32_t acc = x.tmem + lane_off + (uint32_t)(b * kBN);
        const int row0 = m0 + (int)x.rank * kBM;
#pragma unroll 1
        for (int c = 0; c < kBN / kOBox; ++c, ++box) {
            if (n0 + c * kOBox >= p.N)
                break;                                   // uniform over the 128 threads
            uint32_t v0[32], v1[32];
            tmem_ld32(acc + c * kOBox, v0);
            tmem_ld32(acc + c * kOBox + 32, v1);
            // The staging box this store reuses was last read two stores ago.
            if (issuer)
                bulk_wait_group_read<1>();
            named_bar(1, 128);
            tmem_wait_ld_regs(v0);
            tmem_wait_ld_regs(v1);
            const uint32_t st = x.base + Smem::OFF_O + (box & 1) * kOStage;
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(v0[2 * i]) * p.out_scale,
                                                          __uint_as_float(v0[2 * i + 1]) * p.out_scale);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(v1[2 * i]) * p.out_scale,
                                                          __uint_as_float(v1[2 * i + 1]) * p.out_scale);
                pk[i] = *reinterpret_cast<uint32_t *>(&h0);
                pk[16 + i] = *reinterpret_cast<uint32_t *>(&h1);
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t off = (uint32_t)row * 128u + (uint32_t)ch * 16u;
                const uint32_t swz_off = off ^ ((off >> 3) & 0x70u);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(st + swz_off), "r"(pk[4 * ch]),
                             "r"(pk[4 * ch + 1]), "r"(pk[4 * ch + 2]), "r"(pk[4 * ch + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            named_bar(1, 128);
            if (issuer) {
                tma_store_2d(tm_y, st, n0 + c * kOBox, row0);
                bulk_commit_group();
            }
        }
        // Every TMEM load of accumulator b has completed (waited above): hand it back.
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive_cluster(tempty_leader[b]);
    }
    if (issuer)
        bulk_wait_group_all();
}

template <class Kind>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
            const __grid_constant__ CUtensorMap tm_y, const GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    Bars *bars = reinterpret_cast<Bars *>(smem_raw + (base - raw_addr) + Smem::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->tfull[b]), 1);
            mbar_init(smem_u32(&bars->tempty[b]), 8);   // 4 epilogue warps x 2 CTAs
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0u;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();

    Ctx x;
    x.bars = bars;
    x.base = base;
    x.tmem = bars->tmem_base;
    x.rank = rank;
    x.abort = &bars->abort;
    x.lim = p.wait_limit_ns;

    if (warp == 0) {
        if (lane == 0)
            producer<Kind>(x, p, &tm_a, &tm_w);
    } else if (warp == 1) {
        if (rank == 0)
            mma_issuer<Kind>(x, p);
    } else {
        epilogue(x, p, &tm_y, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(x.tmem, kTmemCols);
    }
}

} // namespace dit_gemm
