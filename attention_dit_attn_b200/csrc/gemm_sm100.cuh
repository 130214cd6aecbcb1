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

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int c0, int c1,
                                            uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
        : "memory");
}

// The output is written once and read by nobody in this kernel: it goes to L2
// with the evict-first policy, so it does not push out the operand tiles.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, uint32_t src, int c0, int c1)
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;"
                 ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(c0), "r"(c1), "l"(pol)
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

// Abort path of a producer (a wait ran out of time): give the tile loads it
// already issued 1 ms to land before the CTA leaves, far above a tile load's
// latency, so none writes into shared memory the SM has handed on.
__device__ __forceinline__ void pause_for_loads_in_flight()
{
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 1000000ull) {
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
    // A block: read by the n_tiles pairs that work on it side by side; W: by every pair.
    const uint64_t pol_a = l2_policy_evict_last();
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
                !wait_bar(x.bar(x.bars->empty[s]), ((it / kStages) - 1) & 1, x.abort, x.lim, kSiteEmpty)) {
                pause_for_loads_in_flight();
                return;
            }
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
            // One elected lane issues the stage's MMAs and its commit (one
            // election per stage: fewer issue slots taken from the epilogue
            // warps sharing this warp's sub-partition).
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < Kind::MMAS_PER_STAGE; ++kk) {
                    const uint64_t ad = a_desc + ((uint32_t)(s * kStageA + kk * Kind::KSTEP_BYTES) >> 4);
                    const uint64_t bd = b_desc + ((uint32_t)(s * kStageB + kk * Kind::KSTEP_BYTES) >> 4);
                    mma2_f8_ss(acc, ad, bd, Kind::IDESC, (k > 0 || kk > 0) ? 1u : 0u);
                }
                mma2_commit_mc(x.bar(x.bars->empty[s]), kBoth);
            }
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

// ================================================================== MXFP4 (block-scaled FP4)
//
// Operands are MXFP4 (OCP Microscaling): packed E2M1 codes, two per byte, the
// first element of a pair in the low nibble, and one E8M0 scale per 32
// consecutive K elements.  The tensor core applies the scales itself
// (tcgen05.mma kind::mxf4 block_scale scale_vec::2X: two scales per K = 64
// MMA), reading them from TMEM.  Scales are handed to the kernel in a tiled
// layout (dit_attn_mxfp4_tile_scales): for row r and K block b of a matrix
// with G = 2 ceil(K / 256) four-block groups per 128-row block,
//
//     tiled[((r / 128) G + b / 4) 512 + 16 (r % 32) + 4 ((r % 128) / 32) + b % 4]
//
// so each 512-byte atom (128 rows x 4 blocks) is one contiguous bulk copy and,
// copied to TMEM with tcgen05.cp 32x128b.warpx4 (replicated to the four lane
// quadrants), puts the scale of row m at lane m, column base + m / 32, byte
// b % 4, where the MMA reads it.
//
// The kernel (gemm_mxf4_pair_kernel, below) runs on CTA pairs.  Per K stage of
// 256 elements each CTA loads its share of A and W and their scale atoms,
// the leader copies the scales into a TMEM ring slot and issues four MMAs of
// K = 64.  When every pair can keep one N tile for the whole launch, K is at
// most 3328 and A fits in L2 (the host's choice), W's scales for all of K are
// copied into TMEM once per launch and only A's are copied per stage, two
// stages per run of copies.  The epilogue reads the whole fp32 accumulator into registers as
// bf16 and hands TMEM back before it stages and stores the tile, so the next
// tile's MMAs start while the stores drain.

constexpr int kF4BM = 128, kF4BN = 256;
constexpr uint32_t kF4SfCols = 32;                 // TMEM columns per ring slot (8 A + 16 B used)
constexpr uint32_t kF4TmemSf = 256;                // ring base column (accumulator: 0..255)

struct F4Params {
    int M, N, K;
    int kb;                      // K stages of 256 elements
    int m_tiles, n_tiles;        // ceil(M / 256), ceil(N / 256)
    int groups;                  // G: four-block groups per 128-row block (even)
    int w_row_blocks;            // ceil(N / 128)
    const uint8_t *sfa;          // tiled scales of A
    const uint8_t *sfw;          // tiled scales of W
    unsigned long long wait_limit_ns;
};

__host__ __device__ constexpr uint32_t idesc_mxf4(uint32_t M, uint32_t N, uint32_t sf_id)
{
    // [4,6) B scale id, [7,10) A format (E2M1 = 1), [10,13) B format, [17,23) N >> 3,
    // [23] scale format (1 = E8M0), [24,29) M >> 4, [29,31) A scale id; K-major A and B.
    return (sf_id << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) |
           (sf_id << 29);
}


// ------------------------------------------------------------------ MXFP4 on CTA pairs
//
// The same GEMM on CTA pairs (cta_group::2): a pair owns a 256 x 256 tile,
// each CTA loads its 128 rows of A and 128 of the tile's 256 rows of W per K
// stage, so each SM streams half the W tile through shared memory, and the
// leader issues M = N = 256 block-scaled MMAs.  Scales, measured with a
// probe: tcgen05.cp with cta_group::2 (issued once by the leader) copies each
// CTA's own shared memory into its own TMEM, and each CTA's half of the MMA
// reads A's scales for its own 128 rows and W's scales for all 256 columns
// from its own TMEM.  So each CTA loads the scale atoms of its A rows and of
// both 128-row blocks of the W tile.  The atoms come as plain 2-D TMA boxes
// (4 rows of 256 bytes = two 512-byte atoms) over the tiled array, so both
// CTAs' copies count on the leader's barrier; a W block past N is out of
// range and TMA fills it with zeros (finite scales).

constexpr int kP4Stages = 5;
constexpr int kP4StageA = kF4BM * kBKB;           // 16 KB: this CTA's 128 rows of A
constexpr int kP4StageB = (kF4BN / 2) * kBKB;     // 16 KB: this CTA's 128 rows of W
constexpr int kP4StageSFA = 1024, kP4StageSFB = 2048;
constexpr int kP4StageBytes = kP4StageA + kP4StageB + kP4StageSFA + kP4StageSFB;

// Resident W scales.  When each pair works on one 256-column tile of W for
// the whole launch (n_tiles <= pairs) and K is short enough, the W scale
// atoms for all of K are loaded once (one 2 KB block per K stage, as the
// per-stage path lays them out) and copied into TMEM once; each stage then
// copies only A's scales.  TMEM: accumulator 0..255, A scale ring
// 256 + 8 s, W scales from kF4ResSfb at 16 per K stage.
constexpr uint32_t kF4ResSfa = kF4TmemSf;                           // A scale slot s at + 8 s
constexpr uint32_t kF4ResSfb = kF4ResSfa + 8 * kP4Stages;          // 296: W scales of stage k at + 16 k
constexpr int kF4ResMaxStages = (int)(kTmemCols - kF4ResSfb) / 16; // 13: K <= 3328
constexpr int kP4StageBytesRes = kP4StageA + kP4StageB + kP4StageSFA;

struct P4Bars {
    uint64_t full[kP4Stages];   // leader: stage s of both CTAs landed
    uint64_t empty[kP4Stages];  // each CTA: the MMAs reading stage s completed
    uint64_t tfull;             // each CTA: the accumulator holds a finished tile
    uint64_t tempty;            // leader: both CTAs' epilogues have read it
    uint64_t sfb_full;          // leader: both CTAs' resident W scale atoms landed
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

struct P4Smem {
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + kP4Stages * kP4StageA;
    static constexpr int OFF_SFA = OFF_B + kP4Stages * kP4StageB;
    static constexpr int OFF_SFB = OFF_SFA + kP4Stages * kP4StageSFA;
    static constexpr int OFF_O = OFF_SFB + kP4Stages * kP4StageSFB;
    static constexpr int OFF_SFB_ALL = OFF_O + kOStage;            // resident W scales
    static constexpr int OFF_BAR = OFF_SFB_ALL + kF4ResMaxStages * kP4StageSFB;
    static constexpr int BYTES = OFF_BAR + 256 + 1024;
};
static_assert(P4Smem::BYTES <= 232448, "shared memory budget");
static_assert(kF4TmemSf + kP4Stages * kF4SfCols <= kTmemCols, "TMEM budget");
static_assert(kF4ResSfb + 16 * kF4ResMaxStages <= kTmemCols, "TMEM budget (resident W scales)");

// The k-th tile of this pair (false when it has no more).  Per-stage scales:
// tiles t = pair + k * pairs, the 12-ish N tiles of one A block consecutive.
// Resident W scales: pair p keeps N tile p % n_tiles, and the pairs sharing it
// take every c-th 256-row block of A.
template <bool RES>
__device__ __forceinline__ bool p4_tile(const F4Params &p, int k, int &m0, int &n0)
{
    const int pair = (int)blockIdx.x / 2, pairs = (int)gridDim.x / 2;
    if (RES) {
        const int n = pair % p.n_tiles, i = pair / p.n_tiles;
        const int c = pairs / p.n_tiles + (n < pairs % p.n_tiles ? 1 : 0);
        const long long m = i + (long long)k * c;
        if (m >= p.m_tiles)
            return false;
        m0 = (int)m * 2 * kF4BM;
        n0 = n * kF4BN;
        return true;
    }
    const long long t = pair + (long long)k * pairs;
    if (t >= (long long)p.m_tiles * p.n_tiles)
        return false;
    m0 = (int)(t / p.n_tiles) * 2 * kF4BM;
    n0 = (int)(t % p.n_tiles) * kF4BN;
    return true;
}

__device__ __forceinline__ void mma2_mxf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
                 : "memory");
}

// Each CTA's 32 x 128-bit shared-memory block into its own TMEM (issued by the leader).
__device__ __forceinline__ void tmem_cp2_32x128_x4(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

struct P4Ctx {
    P4Bars *bars;
    uint32_t base, tmem, rank;
    volatile uint32_t *abort;
    unsigned long long lim;
    __device__ uint32_t bar(const uint64_t &b) const { return smem_u32(&b); }
    __device__ uint32_t leader_bar(const uint64_t &b) const { return mapa_shared(smem_u32(&b), 0); }
};

template <bool RES>
__device__ __forceinline__ void p4_producer(const P4Ctx &x, const F4Params &p, const CUtensorMap *tm_a,
                                            const CUtensorMap *tm_w, const CUtensorMap *tm_sa,
                                            const CUtensorMap *tm_sw)
{
    const uint64_t pol_a = l2_policy_evict_last();
    const uint64_t pol_w = l2_policy_evict_last();
    const bool leader = x.rank == 0;
    int m0 = 0, n0 = 0;
    if (RES && p4_tile<RES>(p, 0, m0, n0)) {
        // This pair's W scale atoms for all of K, once (the N tile never changes).
        const uint32_t sfb_full = x.leader_bar(x.bars->sfb_full);
        if (leader)
            mbar_arrive_expect_tx(x.bar(x.bars->sfb_full), 2 * p.kb * kP4StageSFB);
        for (int k = 0; k < p.kb; ++k)
            for (int b = 0; b < 2; ++b)
                tma_load_2d_pair(x.base + P4Smem::OFF_SFB_ALL + k * kP4StageSFB + b * 1024, tm_sw, sfb_full, 0,
                                 ((n0 / 128 + b) * p.groups + 2 * k) * 2, pol_w);
    }
    int it = 0;
    for (int tk = 0; p4_tile<RES>(p, tk, m0, n0); ++tk) {
        const int rba = m0 / 128 + (int)x.rank, rbw = n0 / 128;
        for (int k = 0; k < p.kb; ++k, ++it) {
            const int s = it % kP4Stages;
            if (it >= kP4Stages &&
                !wait_bar(x.bar(x.bars->empty[s]), ((it / kP4Stages) - 1) & 1, x.abort, x.lim, kSiteEmpty)) {
                pause_for_loads_in_flight();
                return;
            }
            if (leader)
                mbar_arrive_expect_tx(x.bar(x.bars->full[s]), 2 * (RES ? kP4StageBytesRes : kP4StageBytes));
            const uint32_t full = x.leader_bar(x.bars->full[s]);
            tma_load_2d_pair(x.base + P4Smem::OFF_A + s * kP4StageA, tm_a, full, k * kBKB, m0 + (int)x.rank * kF4BM,
                             pol_a);
            tma_load_2d_pair(x.base + P4Smem::OFF_B + s * kP4StageB, tm_w, full, k * kBKB,
                             n0 + (int)x.rank * (kF4BN / 2), pol_w);
            // scale atoms of groups 2k, 2k+1: 4 rows of 256 bytes from (block * G + 2k) * 2
            tma_load_2d_pair(x.base + P4Smem::OFF_SFA + s * kP4StageSFA, tm_sa, full, 0, (rba * p.groups + 2 * k) * 2,
                             pol_a);
            if (!RES)
                for (int b = 0; b < 2; ++b)
                    tma_load_2d_pair(x.base + P4Smem::OFF_SFB + s * kP4StageSFB + b * 1024, tm_sw, full, 0,
                                     ((rbw + b) * p.groups + 2 * k) * 2, pol_w);
        }
    }
}

template <bool RES>
__device__ __forceinline__ void p4_mma(const P4Ctx &x, const F4Params &p)
{
    constexpr uint16_t kBoth = 0x3;
    const uint32_t base = __shfl_sync(0xffffffffu, x.base, 0);
    const uint32_t tmem = __shfl_sync(0xffffffffu, x.tmem, 0);
    const uint64_t a_desc = make_smem_desc(base + P4Smem::OFF_A, 16, 8 * 128, kSwizzle128B);
    const uint64_t b_desc = make_smem_desc(base + P4Smem::OFF_B, 16, 8 * 128, kSwizzle128B);
    const uint64_t sfa_desc = make_smem_desc(base + P4Smem::OFF_SFA, 2048, 128, kSwizzleNone);
    const uint64_t sfb_desc = make_smem_desc(base + P4Smem::OFF_SFB, 2048, 128, kSwizzleNone);
    bool ok = true;
    int it = 0, local = 0, m0 = 0, n0 = 0;
    if (RES && p4_tile<RES>(p, 0, m0, n0)) {
        // The resident W scales: stage k's 2 KB block (groups 2k, 2k+1; row blocks
        // 0, 1) into columns kF4ResSfb + 16 k + 8 g + 4 b, as the per-stage path does.
        const uint64_t all_desc = make_smem_desc(base + P4Smem::OFF_SFB_ALL, 2048, 128, kSwizzleNone);
        ok = __all_sync(0xffffffffu, wait_bar(x.bar(x.bars->sfb_full), 0, x.abort, x.lim, kSiteFull));
        if (ok) {
            tc_fence_after();
            if (elect_one()) {
                for (int k = 0; k < p.kb; ++k)
                    for (int g = 0; g < 2; ++g)
                        for (int b = 0; b < 2; ++b)
                            tmem_cp2_32x128_x4(tmem + kF4ResSfb + 16 * k + 8 * g + 4 * b,
                                               all_desc + ((uint32_t)(k * kP4StageSFB + b * 1024 + g * 512) >> 4));
            }
            __syncwarp();
        }
    }
    for (int tk = 0; ok && p4_tile<RES>(p, tk, m0, n0); ++tk, ++local) {
        if (local >= 1)
            ok = __all_sync(0xffffffffu,
                            wait_bar(x.bar(x.bars->tempty), (local - 1) & 1, x.abort, x.lim, kSiteTmemEmpty));
        if (!ok)
            break;
        tc_fence_after();
        for (int k = 0; k < p.kb && ok; ++k, ++it) {
            const int s = it % kP4Stages;
            const uint32_t sfa_t = RES ? tmem + kF4ResSfa + 8u * (uint32_t)s : tmem + kF4TmemSf + (uint32_t)s * kF4SfCols;
            const uint32_t sfb_t = RES ? tmem + kF4ResSfb + 16u * (uint32_t)k : sfa_t + 8;
            // A run of scale copies between MMAs costs about the same whatever its
            // length, so with resident W scales the A scales of two K stages are
            // copied together (at even k, once both stages have landed).
            if (!RES || (k & 1) == 0) {
                const bool pair_k = RES && k + 1 < p.kb;
                const int s2 = (it + 1) % kP4Stages;
                ok = __all_sync(0xffffffffu,
                                wait_bar(x.bar(x.bars->full[s]), (it / kP4Stages) & 1, x.abort, x.lim, kSiteFull) &&
                                    (!pair_k || wait_bar(x.bar(x.bars->full[s2]), ((it + 1) / kP4Stages) & 1,
                                                         x.abort, x.lim, kSiteFull)));
                if (!ok)
                    break;
                tc_fence_after();
                if (elect_one()) {
                    for (int g = 0; g < 2; ++g) {
                        tmem_cp2_32x128_x4(sfa_t + 4 * g, sfa_desc + ((uint32_t)(s * kP4StageSFA + g * 512) >> 4));
                        if (pair_k)
                            tmem_cp2_32x128_x4(tmem + kF4ResSfa + 8u * (uint32_t)s2 + 4 * g,
                                               sfa_desc + ((uint32_t)(s2 * kP4StageSFA + g * 512) >> 4));
                        if (!RES)
                            for (int b = 0; b < 2; ++b)
                                tmem_cp2_32x128_x4(sfb_t + 8 * g + 4 * b,
                                                   sfb_desc + ((uint32_t)(s * kP4StageSFB + b * 1024 + g * 512) >> 4));
                    }
                }
                __syncwarp();
            }
            // One elected lane issues the stage's MMAs and its commit.
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int g = kk >> 1;
                    const uint64_t ad = a_desc + ((uint32_t)(s * kP4StageA + kk * 32) >> 4);
                    const uint64_t bd = b_desc + ((uint32_t)(s * kP4StageB + kk * 32) >> 4);
                    mma2_mxf4(tmem, ad, bd, idesc_mxf4(2 * kF4BM, kF4BN, (uint32_t)(kk & 1) * 2u), sfa_t + 4 * g,
                              sfb_t + 8 * g, (k > 0 || kk > 0) ? 1u : 0u);
                }
                mma2_commit_mc(x.bar(x.bars->empty[s]), kBoth);
            }
            __syncwarp();
        }
        if (ok && elect_one())
            mma2_commit_mc(x.bar(x.bars->tfull), kBoth);
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

template <bool RES>
__device__ __forceinline__ void p4_epilogue(const P4Ctx &x, const F4Params &p, const CUtensorMap *tm_y, int warp,
                                            int lane)
{
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool issuer = warp == kEpiWarp0 && lane == 0;
    const uint32_t tempty_leader = x.leader_bar(x.bars->tempty);
    bool ok = true;
    int local = 0, mp = 0, n0 = 0;
    for (int tk = 0; ok && p4_tile<RES>(p, tk, mp, n0); ++tk, ++local) {
        const int m0 = mp + (int)x.rank * kF4BM;
        ok = __all_sync(0xffffffffu, wait_bar(x.bar(x.bars->tfull), local & 1, x.abort, x.lim, kSiteTmemFull));
        if (!bar_and(1, 128, ok)) {
            ok = false;
            break;
        }
        tc_fence_after();
        uint32_t pk[128];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld32(x.tmem + lane_off + 32 * c, v);
            tmem_wait_ld_regs(v);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                pk[16 * c + i] = *reinterpret_cast<uint32_t *>(&h);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive_cluster(tempty_leader);
#pragma unroll
        for (int c = 0; c < kF4BN / kOBox; ++c) {
            if (n0 + c * kOBox >= p.N)
                break;
            if (issuer)
                bulk_wait_group_read<0>();
            named_bar(1, 128);
            const uint32_t st = x.base + P4Smem::OFF_O;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t off = (uint32_t)row * 128u + (uint32_t)ch * 16u;
                const uint32_t swz_off = off ^ ((off >> 3) & 0x70u);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(st + swz_off), "r"(pk[32 * c + 4 * ch]),
                             "r"(pk[32 * c + 4 * ch + 1]), "r"(pk[32 * c + 4 * ch + 2]), "r"(pk[32 * c + 4 * ch + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            named_bar(1, 128);
            if (issuer) {
                tma_store_2d(tm_y, st, n0 + c * kOBox, m0);
                bulk_commit_group();
            }
        }
    }
    if (issuer)
        bulk_wait_group_all();
}

template <bool RES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_mxf4_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_sa,
                      const __grid_constant__ CUtensorMap tm_sw, const F4Params p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    P4Bars *bars = reinterpret_cast<P4Bars *>(smem_raw + (base - raw_addr) + P4Smem::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kP4Stages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->tfull), 1);
        mbar_init(smem_u32(&bars->tempty), 8);           // 4 epilogue warps x 2 CTAs
        mbar_init(smem_u32(&bars->sfb_full), 1);
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0u;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_w);
        tma_prefetch_desc(&tm_y);
        tma_prefetch_desc(&tm_sa);
        tma_prefetch_desc(&tm_sw);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();

    P4Ctx x;
    x.bars = bars;
    x.base = base;
    x.tmem = bars->tmem_base;
    x.rank = rank;
    x.abort = &bars->abort;
    x.lim = p.wait_limit_ns;

    if (warp == 0) {
        if (lane == 0)
            p4_producer<RES>(x, p, &tm_a, &tm_w, &tm_sa, &tm_sw);
    } else if (warp == 1) {
        if (rank == 0)
            p4_mma<RES>(x, p);
    } else {
        p4_epilogue<RES>(x, p, &tm_y, warp, lane);
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

// Scale tiling: plain [rows, K / 32] E8M0 bytes -> the tiled layout above
// (zero where the padded rows or blocks have no scale).  One thread per
// 16-byte chunk of the output: one row's 4 blocks for 4 rows 32 apart.
__global__ void tile_scales_kernel(const uint8_t *__restrict__ plain, uint32_t *__restrict__ tiled, int rows,
                                   int kblocks, int groups, long long chunks)
{
    for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < chunks;
         c += (long long)gridDim.x * blockDim.x) {
        const long long atom = c >> 5;                   // 32 chunks of 16 bytes per atom
        const int r32 = (int)(c & 31);
        const int g = (int)(atom % groups);
        const long long rb = atom / groups;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const long long r = rb * 128 + q * 32 + r32;
            uint32_t v = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int kb = g * 4 + b;
                if (r < rows && kb < kblocks)
                    v |= (uint32_t)plain[r * kblocks + kb] << (8 * b);
            }
            w[q] = v;
        }
        reinterpret_cast<uint4 *>(tiled)[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

} // namespace dit_gemm
