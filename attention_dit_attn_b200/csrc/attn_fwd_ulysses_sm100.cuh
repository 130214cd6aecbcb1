// Ulysses attention fused with its exchanges: the CTA-pair attention kernel
// reading Q/K/V from every rank's sequence shard and writing O/LSE back into
// every rank's shard.
//
// Page "How to Scale Diffusion Inference Across AMD RDNA 4 GPUs", section
// "Balance Transformer Work and Communication": Ulysses splits the tokens
// across GPUs and every attention layer exchanges data with an all-to-all
// (sequence shards -> head groups before attention, back after it).  Here rank
// `rank` of N owns head group [rank H/N, (rank + 1) H/N).  Instead of an
// all-to-all into a gathered [B, H/N, N Ls, D] tensor, its attention kernel
// loads every K/V/Q tile straight from the shard that holds it (shard c holds
// tokens [c Ls, (c + 1) Ls) of all heads, [B, H, Ls, D]; on several GPUs the
// shards are peers' memory mapped into this context), and its epilogue stores
// each O tile (and LSE row) into the shard its tokens came from.  So the two
// exchanges overlap the attention tile by tile, and no gathered copy exists.
//
// The arithmetic, the MMA issue, the softmax steps and (FP8) the V conversion
// are the CTA-pair kernel's own (attn_fwd_sm100.cuh).  What differs is where
// tiles come from: with Ls a multiple of 64, each 64-row box (a CTA's key
// half, a half of a Q, V or O tile) lies in one shard, so every tile is
// one or two TMA boxes, each addressed through its shard's tensor map.
// Loads are plain TMA loads (no cluster multicast), peers' memory included.
#pragma once
#include "attn_fwd_sm100.cuh"

namespace dit {

constexpr int kMaxUlyssesRanks = 8;
constexpr int kHalfRows = 64;          // rows per TMA box of Q, V and O (and K: KROWS)

struct UlyssesMaps {
    CUtensorMap q[kMaxUlyssesRanks];   // per shard: (D, Ls, B H), box (Q/K span, 64 rows)
    CUtensorMap k[kMaxUlyssesRanks];
    CUtensorMap v[kMaxUlyssesRanks];   // box (D/2, 64 rows)
    CUtensorMap o[kMaxUlyssesRanks];   // box (64 bf16, 64 rows), 128-byte swizzle
};

struct UlyssesParams {
    int n_ranks;
    int Ls;                            // tokens per shard (multiple of 64)
    int H;                             // heads of a shard (all heads)
    int Hn;                            // heads of this rank's group, H / n_ranks
    int head0;                         // first head of the group, rank * Hn
    float *lse[kMaxUlyssesRanks];      // per shard [B, H, Ls] fp32, or all null
};

// Global token g -> shard c and row r in it.  Tokens past the sequence map to
// rows >= Ls of the last shard, which TMA loads fill with zeros.
__device__ __forceinline__ void shard_of(const UlyssesParams &u, int g, int &c, int &r)
{
    c = g / u.Ls;
    if (c >= u.n_ranks)
        c = u.n_ranks - 1;
    r = g - c * u.Ls;
}

// (b, head of the group) as the kernel enumerates them -> b H + head0 + h, the
// head's index in every shard (and in the [B, H] FP8 scales).
__device__ __forceinline__ int shard_bh(const UlyssesParams &u, int bh_group)
{
    const int b = bh_group / u.Hn;
    return b * u.H + u.head0 + (bh_group - b * u.Hn);
}

// ------------------------------------------------------------------ producers (both CTAs)
// The CTA-pair producer's rings and barriers, with every box addressed
// through the tensor map of the shard that holds its rows.
template <class C>
__device__ __forceinline__ void ulysses_producer(const PairCtx<C> &x, const FwdParams &p, const UlyssesParams &u,
                                                 int lane, const UlyssesMaps &m)
{
    auto *bars = x.bars;
    const bool leader = x.rank == 0;
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    const int n = p.n_kv, n0 = n < 2 ? n : 2;
    const int bhs = shard_bh(u, x.bh);
    bool ok = true;
    auto load_k = [&](int j, uint32_t bar) {
        int c, r;
        shard_of(u, j * kBN + (int)x.rank * C::KROWS, c, r);
        for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d_pair(x.base + C::OFF_K + (j % 2) * align_up(C::KTILE, 1024) + b * C::KBOX_BYTES, &m.k[c],
                             bar, b * C::BOX_ELEMS, r, bhs, pol_kv);
    };
    if (lane == 0) {
        if (leader) {
            mbar_arrive_expect_tx(x.bar(bars->q_full), 2 * C::QTILE);
            mbar_arrive_expect_tx(x.bar(bars->k0_full), 2 * n0 * C::KTILE);
        }
        for (int hh = 0; hh < 2; ++hh) {
            int c, r;
            shard_of(u, x.q0 + hh * kHalfRows, c, r);
            for (int b = 0; b < C::NBOX; ++b)
                tma_load_3d_pair(x.base + C::OFF_Q + b * C::QBOX_BYTES + hh * kHalfRows * C::SWZ, &m.q[c],
                                 x.leader_bar(bars->q_full), b * C::BOX_ELEMS, r, bhs, pol_q);
        }
        for (int j = 0; j < n0; ++j)
            load_k(j, x.leader_bar(bars->k0_full));
        for (int j = 0; j < n && ok; ++j) {
            const int b2 = j % 2, mm = j + 2;           // load K(mm) for step j
            ok = wait_bar_cluster(x.bar(bars->s_full[b2]), (j / 2) & 1, x.abort, x.lim, kSiteKvEmpty);
            if (!ok)
                break;
            if (mm < n) {
                if (leader)
                    mbar_arrive_expect_tx(x.bar(bars->ready[b2]), 2 * C::KTILE);
                load_k(mm, x.leader_bar(bars->ready[b2]));
            } else if (leader) {
                mbar_arrive(x.bar(bars->ready[b2]));
            }
        }
    } else if (lane == 1) {
        for (int j = 0; j < n && ok; ++j) {
            const int st = j % 2;
            if (j >= 2)
                ok = wait_bar_cluster(x.bar(bars->pv_done[st]), ((j - 2) / 2) & 1, x.abort, x.lim, kSiteKvEmpty);
            if (!ok)
                break;
            const uint32_t dst = x.base + C::OFF_V + st * align_up(C::VRAW_TILE, 1024);
            if (C::FP8)
                mbar_arrive_expect_tx(x.bar(bars->v_full[st]), C::VRAW_TILE);
            else if (leader)
                mbar_arrive_expect_tx(x.bar(bars->ready[st]), 2 * C::VRAW_TILE);
            for (int hh = 0; hh < 2; ++hh) {
                int c, r;
                shard_of(u, j * kBN + hh * kHalfRows, c, r);
                const uint32_t d = dst + hh * kHalfRows * C::VRAW_ROW;
                if (C::FP8)
                    tma_load_3d(d, &m.v[c], x.bar(bars->v_full[st]), (int)x.rank * (C::D / 2), r, bhs, pol_kv);
                else
                    tma_load_3d_pair(d, &m.v[c], x.leader_bar(bars->ready[st]), (int)x.rank * (C::D / 2), r, bhs,
                                     pol_kv);
            }
        }
    }
    if (!ok) {
        // Give copies already in flight time to land before the cluster exits:
        // 1 ms, far above the latency of a tile load from this GPU's memory or
        // over NVLink from a peer's (a few microseconds).  Only the abort path
        // (after a wait has run out of time) pays it.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) {
        }
    }
}

// ------------------------------------------------------------------ softmax + epilogue
// The CTA-pair softmax (half_row_step) and its epilogue, with O and the LSE
// stored into the shards their rows belong to.
template <class C>
__device__ __forceinline__ void ulysses_softmax(const PairCtx<C> &x, const FwdParams &p, const UlyssesParams &u,
                                                const UlyssesMaps &m, int warp, int lane)
{
    constexpr int D = C::D;
    auto *bars = x.bars;
    const int h = warp >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;
    const int bhs = shard_bh(u, x.bh);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    float *red = reinterpret_cast<float *>(x.sm + C::OFF_RED);
    const uint32_t bar_id = 1 + wq;
    const uint32_t ready_leader[2] = {x.leader_bar(bars->ready[0]), x.leader_bar(bars->ready[1])};
    HalfRowState st;
    st.c2 = p.scale * kLog2e;
    float vs = 1.f;
    if (C::FP8) {
        st.c2 = p.scale * p.q_scale[bhs] * p.k_scale[bhs] * kLog2e;
        vs = p.v_scale[bhs];
    }
    st.m_use = -INFINITY;
    st.l = 0.f;
    st.alive = true;
    const int n = p.n_kv;
    for (int j = 0; j < n && st.alive; j += 2) {
        half_row_step<C>(x, p, j, h, lane, lane_off, ready_leader[0], st);
        if (j + 1 < n && st.alive)
            half_row_step<C>(x, p, j + 1, h, lane, lane_off, ready_leader[1], st);
    }
    bool alive = st.alive;
    // ---- epilogue: merge the two key halves through their log-sum-exp,
    // (a_0 O_0 + a_1 O_1) / l -> bf16 -> staging -> TMA stores into the shards; LSE.
    if (alive) {
        const int jl = n - 1;
        alive = __all_sync(0xffffffffu, wait_bar_cluster(x.bar(bars->pv_done[jl % 2]), (jl / 2) & 1, x.abort,
                                                          x.lim, kSiteOFull));
    }
    const float m2 = st.l > 0.f ? st.m_use * st.c2 : -INFINITY;
    red[h * kBM + row] = m2;
    red[(2 + h) * kBM + row] = st.l;
    alive = bar_and(bar_id, 64, alive);
    const float m2o = red[(1 - h) * kBM + row], lo = red[(3 - h) * kBM + row];
    const float mrow = fmaxf(m2, m2o);
    const float a_self = ex2_approx(m2 - mrow), a_other = ex2_approx(m2o - mrow);
    const float l_row = st.l * a_self + lo * a_other;
    const float a0 = h == 0 ? a_self : a_other, a1 = h == 0 ? a_other : a_self;
    const uint32_t ost = C::FP8 ? x.base + C::OFF_OST : x.base + C::OFF_Q;
    if (alive) {
        tc_fence_after();
        const float inv = (C::FP8 ? vs : 1.f) / l_row;
        const float w0 = a0 * inv, w1 = a1 * inv;
        const uint32_t tO0 = x.tmem + lane_off + C::TM_O + h * (D / 2);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
            uint32_t o0[32], o1[32];
            tmem_ld32(tO0 + 32 * cc, o0);
            tmem_ld32(tO0 + D + 32 * cc, o1);
            tmem_wait_ld_regs(o0);
            tmem_wait_ld_regs(o1);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_p(__uint_as_float(o0[2 * i]) * w0 + __uint_as_float(o1[2 * i]) * w1,
                               __uint_as_float(o0[2 * i + 1]) * w0 + __uint_as_float(o1[2 * i + 1]) * w1, false);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int chunk = h * (D / 16) + 4 * cc + k4;     // 16-byte chunk of the output row
                const uint32_t off = (chunk >> 3) * C::OBOX_BYTES +
                                     swz<128>((uint32_t)row * 128u + (uint32_t)(chunk & 7) * 16u);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ost + off),
                             "r"(pk[4 * k4]), "r"(pk[4 * k4 + 1]), "r"(pk[4 * k4 + 2]), "r"(pk[4 * k4 + 3])
                             : "memory");
            }
        }
        fence_proxy_async_smem();
    }
    alive = bar_and(5, 256, alive);
    if (alive) {
        const int qrow = x.q0 + row;
        if (h == 0 && u.lse[0] != nullptr && qrow < p.L) {
            int c, r;
            shard_of(u, qrow, c, r);
            u.lse[c][(long long)bhs * u.Ls + r] = (mrow + log2f(l_row)) * kLn2;
        }
        if (warp == 0 && lane == 0) {
            // Ls and L are multiples of 64: a 64-row half lies in one shard, wholly
            // inside the sequence or wholly past it.
            for (int hh = 0; hh < 2; ++hh) {
                const int g = x.q0 + hh * kHalfRows;
                if (g >= p.L)
                    break;
                int c, r;
                shard_of(u, g, c, r);
                for (int b = 0; b < C::OBOX; ++b)
                    tma_store_3d(&m.o[c], ost + b * C::OBOX_BYTES + hh * kHalfRows * 128, b * 64, r, bhs);
            }
            bulk_commit_group();
            bulk_wait_group_all();
        }
    }
}

// ------------------------------------------------------------------ the kernel
template <int D, bool FP8>
__global__ void __launch_bounds__(PCfg<D, FP8>::THREADS, 1)
attn_fwd_ulysses_kernel(const __grid_constant__ UlyssesMaps m, const FwdParams p, const __grid_constant__ UlyssesParams u)
{
    using C = PCfg<D, FP8>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    PairBars *bars = reinterpret_cast<PairBars *>(smem_raw + (base - raw_addr) + C::OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->q_full), 1);
        mbar_init(smem_u32(&bars->k0_full), 1);
        // ready: 16 softmax warps + the K producer + (bf16) the V producer or (FP8) two converters.
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars->ready[b]), FP8 ? 19 : 18);
            mbar_init(smem_u32(&bars->v_full[b]), 1);
            mbar_init(smem_u32(&bars->s_full[b]), 1);
            mbar_init(smem_u32(&bars->pv_done[b]), 1);
        }
        mbar_init(smem_u32(&bars->drain), 1);
        bars->abort = 0u;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc_pair(smem_u32(&bars->tmem_base), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();

    PairCtx<C> x;
    x.bars = bars;
    x.sm = smem_raw + (base - raw_addr);
    x.base = base;
    x.tmem = bars->tmem_base;
    x.rank = rank;
    x.abort = &bars->abort;
    x.lim = p.wait_limit_ns;
    const int cluster = blockIdx.x >> 1;
    x.bh = cluster / p.n_pairs;                        // (b, head of the group)
    x.q0 = (cluster % p.n_pairs) * 2 * kBM + (int)rank * kBM;

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        if (warp == C::TMA_WARP) {
            if (lane < 2)
                ulysses_producer<C>(x, p, u, lane, m);
        } else if (warp == C::MMA_WARP) {
            if (rank == 0)
                pair_mma<C>(x, p);
        } else if (FP8) {
            pair_convert_v<C>(x, p);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        ulysses_softmax<C>(x, p, u, m, warp, lane);
    }

    // Neither CTA leaves (or frees TMEM) while the pair's MMAs may still touch it.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == C::MMA_WARP) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(x.tmem, C::TMEM_COLS);
    }
}

} // namespace dit
