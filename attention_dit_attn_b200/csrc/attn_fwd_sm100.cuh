// Attention forward on a CTA pair (cluster of 2, tcgen05 cta_group::2).
//
// O = softmax(scale * Q K^T) V plus the row log-sum-exp (operation and
// sources: attn_common.cuh).  A cluster of two CTAs on two SMs processes 256 query
// rows of one (b, h); each CTA owns 128 of them.  Every MMA is issued once,
// by the leader CTA, with M = 256:
//
//   S = Q K^T   A = each CTA's own Q tile, B = K tile split by keys: each CTA
//               loads 64 of the tile's 128 keys;
//   O += P V    A = P from each CTA's TMEM, B = V tile split by columns: each
//               CTA loads D/2 of the D columns.
//
// So each SM streams only half of every K/V tile from L2 while the MMA sees
// the full tile, and no tile is copied between the two CTAs.
//
// Split keys: each query row is handled by two threads (warps w and w+4 share
// TMEM lanes 32(w%4)..+31).  Half h owns keys 64h..64h+63 of every K/V tile
// and keeps its own running max, running sum and output accumulator O_h
// (a flash-style split over keys); the two partial results are merged once,
// in the epilogue, through their log-sum-exp.  No per-tile exchange between
// the two threads is needed.  TMEM (per CTA, 512 columns): two S buffers of
// 128 columns, O_0 and O_1 of D columns each.  The MMA issues S(j+2) right
// after PV(j) into the same buffer, so the softmax of step j+1 overlaps
// PV(j) and S(j+2).
//
// Warps (per CTA):
//   0-3, 4-7  softmax + epilogue (half h = warp / 4)
//   8         TMA producers (lane 0: Q and K, lane 1: V; both CTAs load halves)
//   9         TMEM owner; in the leader also the MMA issuer (one elected lane)
//   10-11     FP8 only: e4m3 -> f16 conversion of this CTA's V half
//
// P of half h is written over S columns 64h..64h+31 of its buffer (values
// only that thread has read), and the PV MMA reads it from there.  O_h is
// rescaled lazily: a rescale at step j first waits for PV(j-1); per-buffer
// barriers keep every parity wait unambiguous (S(j) complete implies PV(j-2)
// complete, and S(j+2) / PV(j+2) cannot complete before this step's P).
#pragma once
#include <type_traits>

#include "attn_common.cuh"

namespace dit {

#ifndef DIT_EXP_EMU
#define DIT_EXP_EMU 2
#endif

template <int D_, bool FP8_>
struct PCfg {
    static constexpr int D = D_;
    static constexpr bool FP8 = FP8_;
    static constexpr int ELT = FP8 ? 1 : 2;
    static constexpr int ROW = D * ELT;                    // Q/K row bytes
    static constexpr int SWZ = ROW >= 128 ? 128 : 64;      // Q/K swizzle span
    static constexpr uint32_t SWZ_MODE = SWZ == 128 ? kSwizzle128B : kSwizzle64B;
    static constexpr int BOX_ELEMS = SWZ / ELT;
    static constexpr int NBOX = ROW / SWZ;
    static constexpr int QBOX_BYTES = kBM * SWZ;
    static constexpr int QTILE = kBM * ROW;
    static constexpr int KROWS = kBN / 2;                  // keys per CTA per tile
    static constexpr int KBOX_BYTES = KROWS * SWZ;
    static constexpr int KTILE = KROWS * ROW;
    static constexpr int KSTEP = 32;
    static constexpr int QK_STEPS = ROW / KSTEP;
    static constexpr int STEPS_PER_BOX = SWZ / KSTEP;
    // V half as loaded: 128 keys x D/2 elements (row = swizzle span).
    static constexpr int VRAW_ROW = (D / 2) * ELT;
    static constexpr int VRAW_TILE = kBN * VRAW_ROW;
    // 16-bit V operand of PV: 128 keys x D/2, MN-major, row = swizzle span.
    static constexpr int VROW = D;
    static constexpr uint32_t V_SWZ_MODE = VROW == 128 ? kSwizzle128B : kSwizzle64B;
    static constexpr int VTILE16 = kBN * VROW;
    static constexpr int NK = 2, NV = 2, NVH = 2;   // K(j), V(j) live in stage j % 2
    // O staging (bf16, 128 rows, SW128 boxes of 64 columns).
    static constexpr int OBOX = (D * 2) / 128, OBOX_BYTES = kBM * 128, OTILE = kBM * D * 2;
    // Shared memory (offsets from a 1024-aligned base).
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + align_up(QTILE, 1024);
    static constexpr int OFF_V = OFF_K + NK * align_up(KTILE, 1024);
    static constexpr int OFF_VH = OFF_V + NV * align_up(VRAW_TILE, 1024);
    static constexpr int OFF_OST = OFF_VH + (FP8 ? NVH * align_up(VTILE16, 1024) : 0);
    static constexpr int OFF_RED = OFF_OST + (FP8 ? OTILE : 0);
    static constexpr int RED_BYTES = 2 * 2 * kBM * 4;      // [m|l][half][row] floats (epilogue merge)
    static constexpr int OFF_BAR = OFF_RED + RED_BYTES;
    static constexpr int BAR_BYTES = 512;
    // At least 116 KB so two CTAs never share an SM (each holds all 512 TMEM columns).
    static constexpr int SMEM_RAW = OFF_BAR + BAR_BYTES + 1024;
    static constexpr int SMEM_BYTES = SMEM_RAW > 118784 ? SMEM_RAW : 118784;
    // TMEM columns.
    static constexpr uint32_t TM_S = 0;                    // buffer b at 128 b (b = 0, 1)
    static constexpr uint32_t TM_O = 256;                  // O_h at TM_O + h * D
    static constexpr uint32_t TMEM_COLS = 512;
    // Warp roles / registers.
    static constexpr int TMA_WARP = 8, MMA_WARP = 9, CONV_WARP0 = 10, CONV_THREADS = 64;
    static constexpr int THREADS = 384;
    static constexpr int REGS_SOFTMAX = 192, REGS_OTHER = 120;   // 2 x 192 + 120 = 3 x 168
    static constexpr int EXP_EMU = DIT_EXP_EMU;
    static_assert(EXP_EMU >= 1 && 8 % EXP_EMU == 0, "polynomial pairs: 1, 2, 4 or 8 of every 8");
    static constexpr uint32_t IDESC_QK = FP8 ? make_idesc(kFmtE4M3, kFmtE4M3, 0, 2 * kBM, kBN)
                                             : make_idesc(kFmtBF16, kFmtBF16, 0, 2 * kBM, kBN);
    static constexpr uint32_t IDESC_PV = FP8 ? make_idesc(kFmtF16, kFmtF16, 1, 2 * kBM, D)
                                             : make_idesc(kFmtBF16, kFmtBF16, 1, 2 * kBM, D);

    static_assert(D == 64 || D == 128, "head dim");
    static_assert(NBOX * QBOX_BYTES == QTILE && NBOX * KBOX_BYTES == KTILE, "whole boxes");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(TM_O + 2 * D <= TMEM_COLS, "TMEM budget");
};

struct PairBars {
    uint64_t q_full;          // leader: both CTAs' Q tiles landed
    uint64_t k0_full;         // leader: K(0..1), both halves, landed
    uint64_t ready[2];        // leader: everything step j needs (b = j % 2): P(j) from
                              // the 16 softmax warps, V(j), K(j+2)
    uint64_t v_full[2];       // fp8: this CTA's raw V(j) half landed (converter input)
    uint64_t s_full[2];       // each CTA: S buffer b holds S(j); frees K stage b
    uint64_t pv_done[2];      // each CTA: PV(j) complete; frees V stage b
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

template <class C>
struct PairCtx {
    PairBars *bars;
    uint8_t *sm;              // generic pointer to the aligned shared-memory base
    uint32_t base, tmem, rank;
    volatile uint32_t *abort;
    unsigned long long lim;
    int bh, q0;               // q0: first query row of this CTA's tile
    __device__ uint32_t bar(const uint64_t &b) const { return smem_u32(&b); }
    __device__ uint32_t leader_bar(const uint64_t &b) const { return mapa_shared(smem_u32(&b), 0); }
};

__device__ __forceinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
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
            atomicCAS(&g_error_word, 0u, (site << 8) | kErrTimeout);
            *abort = 1u;
            return false;
        }
    }
}

// ------------------------------------------------------------------ producers (both CTAs)
// Two threads of the TMA warp, one per ring.  K(j) and V(j) live in stage
// j % 2.  Lane 0 loads Q, K(0..1) (barrier k0_full), then K(j+2) once S(j)
// has completed (s_full), counted on the leader's ready[j % 2]; for the last
// two steps it only arrives there.  Lane 1 loads V(j) once PV(j-2) has
// completed (pv_done), counted on ready[j % 2] (bf16) or on this CTA's
// v_full[j % 2] (FP8: converted first).  s_full / pv_done phases cannot run
// two ahead of these waits (S(j+2) needs K(j+2), PV(j) needs V(j)).
template <class C>
__device__ __forceinline__ void pair_producer(const PairCtx<C> &x, const FwdParams &p, int lane,
                                              const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                              const CUtensorMap *tm_v)
{
    auto *bars = x.bars;
    const bool leader = x.rank == 0;
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    const int n = p.n_kv, n0 = n < 2 ? n : 2;
    bool ok = true;
    auto k_dst = [&](int j, int b) {
        return x.base + C::OFF_K + (j % 2) * align_up(C::KTILE, 1024) + b * C::KBOX_BYTES;
    };
    if (lane == 0) {
        if (leader) {
            mbar_arrive_expect_tx(x.bar(bars->q_full), 2 * C::QTILE);
            mbar_arrive_expect_tx(x.bar(bars->k0_full), 2 * n0 * C::KTILE);
        }
        for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d_pair(x.base + C::OFF_Q + b * C::QBOX_BYTES, tm_q, x.leader_bar(bars->q_full),
                             b * C::BOX_ELEMS, x.q0, x.bh, pol_q);
        for (int j = 0; j < n0; ++j)
            for (int b = 0; b < C::NBOX; ++b)
                tma_load_3d_pair(k_dst(j, b), tm_k, x.leader_bar(bars->k0_full), b * C::BOX_ELEMS,
                                 j * kBN + (int)x.rank * C::KROWS, x.bh, pol_kv);
        for (int j = 0; j < n && ok; ++j) {
            const int b2 = j % 2, m = j + 2;            // load K(m) for step j
            ok = wait_bar_cluster(x.bar(bars->s_full[b2]), (j / 2) & 1, x.abort, x.lim, kSiteKvEmpty);
            if (!ok)
                break;
            if (m < n) {
                if (leader)
                    mbar_arrive_expect_tx(x.bar(bars->ready[b2]), 2 * C::KTILE);
                for (int b = 0; b < C::NBOX; ++b)
                    tma_load_3d_pair(k_dst(m, b), tm_k, x.leader_bar(bars->ready[b2]), b * C::BOX_ELEMS,
                                     m * kBN + (int)x.rank * C::KROWS, x.bh, pol_kv);
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
            if (C::FP8) {
                mbar_arrive_expect_tx(x.bar(bars->v_full[st]), C::VRAW_TILE);
                tma_load_3d(dst, tm_v, x.bar(bars->v_full[st]), (int)x.rank * (C::D / 2), j * kBN, x.bh, pol_kv);
            } else {
                if (leader)
                    mbar_arrive_expect_tx(x.bar(bars->ready[st]), 2 * C::VRAW_TILE);
                tma_load_3d_pair(dst, tm_v, x.leader_bar(bars->ready[st]), (int)x.rank * (C::D / 2),
                                 j * kBN, x.bh, pol_kv);
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

// ------------------------------------------------------------------ MMA issuer (leader, one warp)
// The whole warp runs the loop and its waits; one elected lane issues all of a
// step's MMAs and commits inside a single branch.  The issuing warp shares
// its SM sub-partition with two softmax warps, and every instruction it
// issues is taken from theirs: an election per MMA cost 1-4 % of the whole
// kernel against one per step.  All shared-memory descriptors of one operand
// differ only in the start-address field (bits 0..13, address >> 4;
// addresses stay below 2^18 so the field never carries), so each is a base
// descriptor plus a compile-time constant, and the loop is unrolled over the
// two S buffers so that every TMEM address and descriptor offset is an
// immediate.
template <class C>
__device__ __forceinline__ void pair_mma(const PairCtx<C> &x, const FwdParams &p)
{
    auto *bars = x.bars;
    constexpr uint16_t kBoth = 0x3;
    constexpr uint32_t K_STAGE = align_up(C::KTILE, 1024);
    constexpr uint32_t V_STAGE = C::FP8 ? align_up(C::VTILE16, 1024) : align_up(C::VRAW_TILE, 1024);
    const uint32_t base = __shfl_sync(0xffffffffu, x.base, 0);
    const uint32_t tmem = __shfl_sync(0xffffffffu, x.tmem, 0);
    const uint64_t q_desc = make_smem_desc(base + C::OFF_Q, 16, 8 * C::SWZ, C::SWZ_MODE);
    const uint64_t k_desc = make_smem_desc(base + C::OFF_K, 16, 8 * C::SWZ, C::SWZ_MODE);
    const uint64_t v_desc =
        make_smem_desc(base + (C::FP8 ? C::OFF_VH : C::OFF_V), 16, 8 * C::VROW, C::V_SWZ_MODE);
    // S(j) into buffer BUF = j % 2 from K stage BUF.
    auto issue_s = [&](auto buf_c) {
        constexpr int BUF = decltype(buf_c)::value;
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk) {
            const uint32_t b = kk / C::STEPS_PER_BOX, w = (kk % C::STEPS_PER_BOX) * C::KSTEP;
            const uint64_t ad = q_desc + ((b * C::QBOX_BYTES + w) >> 4);
            const uint64_t bd = k_desc + ((BUF * K_STAGE + b * C::KBOX_BYTES + w) >> 4);
            if (C::FP8)
                mma2_f8_ss(tmem + C::TM_S + 128u * BUF, ad, bd, C::IDESC_QK, kk > 0);
            else
                mma2_f16_ss(tmem + C::TM_S + 128u * BUF, ad, bd, C::IDESC_QK, kk > 0);
        }
    };
    // PV(j) from buffer BUF: key half h (P_h, V rows 64h..64h+63) into O_h.
    auto issue_pv = [&](auto buf_c, bool first) {
        constexpr int BUF = decltype(buf_c)::value;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int h = m >> 2, kk = m & 3;
            const uint64_t bd = v_desc + ((BUF * V_STAGE + (64 * h + 16 * kk) * C::VROW) >> 4);
            mma2_f16_ts(tmem + C::TM_O + h * C::D, tmem + C::TM_S + 128u * BUF + 64 * h + 8 * kk, bd,
                        C::IDESC_PV, (kk == 0 && first) ? 0u : 1u);
        }
    };
    bool ok = true;
    const int n = p.n_kv;
    // Step j: once P(j), V(j) and K(j+2) are in (ready[j % 2]), PV(j) and then
    // S(j+2) into the same buffer.  S(j+2) depends on nothing of step j+1, so
    // the softmax of step j+1 overlaps both.
    auto step = [&](auto buf_c, int j) {
        constexpr int BUF = decltype(buf_c)::value;
        ok = __all_sync(0xffffffffu,
                        wait_bar_cluster(x.bar(bars->ready[BUF]), (j >> 1) & 1, x.abort, x.lim, kSitePFull));
        if (!ok)
            return;
        tc_fence_after();
        if (elect_one()) {
            issue_pv(buf_c, j == 0);
            mma2_commit_mc(x.bar(bars->pv_done[BUF]), kBoth);
            if (j + 2 < n) {
                issue_s(buf_c);
                mma2_commit_mc(x.bar(bars->s_full[BUF]), kBoth);
            }
        }
        __syncwarp();
    };
    using B0 = std::integral_constant<int, 0>;
    using B1 = std::integral_constant<int, 1>;
    ok = __all_sync(0xffffffffu, wait_bar_cluster(x.bar(bars->q_full), 0, x.abort, x.lim, kSiteQFull) &&
                                     wait_bar_cluster(x.bar(bars->k0_full), 0, x.abort, x.lim, kSiteKFull));
    if (ok) {
        tc_fence_after();
        if (elect_one()) {
            issue_s(B0{});
            mma2_commit_mc(x.bar(bars->s_full[0]), kBoth);
            if (n > 1) {
                issue_s(B1{});
                mma2_commit_mc(x.bar(bars->s_full[1]), kBoth);
            }
        }
        __syncwarp();
    }
    for (int j = 0; j < n && ok; j += 2) {
        step(B0{}, j);
        if (j + 1 < n && ok)
            step(B1{}, j + 1);
    }
    if (!ok) {
        if (elect_one())
            mma2_commit(x.bar(bars->drain));
        __syncwarp();
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(x.bar(bars->drain), 0) && globaltimer_ns() - t0 < 50000000ull) {
        }
    }
}

// ------------------------------------------------------------------ FP8: V half e4m3 -> f16
template <class C>
__device__ __forceinline__ void pair_convert_v(const PairCtx<C> &x, const FwdParams &p)
{
    auto *bars = x.bars;
    const int ct = threadIdx.x - C::CONV_WARP0 * 32;
    constexpr int CPR = C::VRAW_ROW / 16;               // raw 16-byte chunks per key row
    constexpr int CHUNKS = kBN * CPR;
    const uint32_t ready_leader[2] = {x.leader_bar(bars->ready[0]), x.leader_bar(bars->ready[1])};
    for (int j = 0; j < p.n_kv; ++j) {
        const int st = j % 2;
        bool ok = wait_bar(x.bar(bars->v_full[st]), (j / 2) & 1, x.abort, x.lim, kSiteConvFull);
        // f16 buffer j & 1 was last read by PV(j-2).
        if (j >= 2)
            ok = ok && wait_bar_cluster(x.bar(bars->pv_done[st]), ((j - 2) / 2) & 1, x.abort, x.lim,
                                        kSiteVhEmpty);
        if (!bar_and(6, C::CONV_THREADS, ok))
            break;
        const uint32_t src = x.base + C::OFF_V + st * align_up(C::VRAW_TILE, 1024);
        const uint32_t dst = x.base + C::OFF_VH + (j & 1) * align_up(C::VTILE16, 1024);
        for (int idx = ct; idx < CHUNKS; idx += C::CONV_THREADS) {
            const int r = idx / CPR, d0 = (idx % CPR) * 16;
            uint32_t w[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(src + swz<C::VRAW_ROW>((uint32_t)(r * C::VRAW_ROW + d0))));
            uint32_t hv[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                hv[2 * i] = cvt_e4m3x2_to_f16x2(w[i] & 0xFFFFu);
                hv[2 * i + 1] = cvt_e4m3x2_to_f16x2(w[i] >> 16);
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t off = swz<C::VROW>((uint32_t)(r * C::VROW + (d0 + 8 * half) * 2));
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + off),
                             "r"(hv[4 * half]), "r"(hv[4 * half + 1]), "r"(hv[4 * half + 2]),
                             "r"(hv[4 * half + 3])
                             : "memory");
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(6, C::CONV_THREADS);
        if (ct == 0)
            mbar_arrive_cluster(ready_leader[j % 2]);
    }
}

// ------------------------------------------------------------------ softmax (two threads per row)

// Max of this thread's 64 S values (keys >= valid count as -inf).
template <bool MASK>
__device__ __forceinline__ float half_row_max(const uint32_t (&s)[2][32], int kbase, int valid)
{
    auto val = [&](int i, int c) {
        const float v = __uint_as_float(s[i][c]);
        return (!MASK || kbase + 32 * i + c < valid) ? v : -INFINITY;
    };
    float m8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        m8[k] = fmaxf(val(0, 2 * k), val(0, 2 * k + 1));
#pragma unroll
    for (int e = 16; e < 64; e += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k)
            m8[k] = max3f(m8[k], val(e >> 5, (e & 31) + 2 * k), val(e >> 5, (e & 31) + 2 * k + 1));
    return max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
}

// p = 2^(s*c2 - mc) for this thread's 64 values, packed to 16 bits and stored
// as 32 TMEM columns at tS (over S values only this thread has read).
// Returns the sum of the p.  Of every 8 pairs, EMU use the FMA-pipe exp2.
// bf16 P (bf16 path) and f16 P (FP8 path) are rounded to nearest even; f16 P
// (FP8 path) is rounded to nearest.
// The second 32 values may still be in flight from TMEM: the loop waits for
// them (a no-op when they have landed) before their chunk.
template <class C, bool MASK, int EMU>
__device__ __forceinline__ float half_row_exp_store(uint32_t (&s)[2][32], uint32_t tS, int kbase, int valid,
                                                    float c2, float mc)
{
    const float2 c2c2 = make_float2(c2, c2), nmc = make_float2(-mc, -mc);
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        if (i == 1)
            tmem_wait_ld_regs(s[1]);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
            const int pi = (32 * i + c) >> 1;
            const float2 xv = __ffma2_rn(make_float2(__uint_as_float(s[i][c]), __uint_as_float(s[i][c + 1])),
                                         c2c2, nmc);
            float2 e;
            // Which EMU of every 8 pairs take the polynomial: the last ones on
            // the bf16 path, every (8/EMU)-th one on the FP8 path (each measured
            // faster on its own path).
            const bool poly = C::FP8 ? (pi % (8 / EMU)) == (8 / EMU) - 1 : (pi & 7) >= 8 - EMU;
            if (poly) {
                e = exp2_poly2(xv);
            } else {
                e.x = ex2_approx(xv.x);
                e.y = ex2_approx(xv.y);
            }
            if (MASK) {
                e.x = (kbase + 32 * i + c < valid) ? e.x : 0.f;
                e.y = (kbase + 32 * i + c + 1 < valid) ? e.y : 0.f;
            }
            acc[pi & 3] = __fadd2_rn(acc[pi & 3], e);
            pk[c / 2] = pack_p(e.x, e.y, C::FP8);
        }
        tmem_st16(tS + 16 * i, pk);
    }
    const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return a.x + a.y;
}

// Per-thread softmax state: running max (raw S units, lazily raised), running
// sum of this thread's key half, log2(e) * scale (with the FP8 dequant scales).
struct HalfRowState {
    float m_use, l, c2;
    bool alive;
};

// One step j for one thread: its 64 values of S(j) -> P(j) (in place in TMEM),
// running max / sum, lazy rescale of O_h; hands P(j) to the MMA through the
// leader's ready[j % 2].
template <class C>
__device__ __forceinline__ void half_row_step(const PairCtx<C> &x, const FwdParams &p, int j, int h,
                                              int lane, uint32_t lane_off, uint32_t ready_leader,
                                              HalfRowState &st)
{
    constexpr int D = C::D;
    auto *bars = x.bars;
    const int n = p.n_kv, buf = j % 2;
    st.alive = __all_sync(0xffffffffu, st.alive && wait_bar_cluster(x.bar(bars->s_full[buf]), (j / 2) & 1,
                                                                     x.abort, x.lim, kSiteSFull));
    if (!st.alive)
        return;
    tc_fence_after();
    const uint32_t tS = x.tmem + lane_off + C::TM_S + 128u * buf + 64 * h;
    // The first 32 values are waited for here; the second 32 load while the
    // exponentials of the first run (the first tile needs all 64 for its max).
    uint32_t s[2][32];
    tmem_ld32(tS, s[0]);
    tmem_wait_ld_regs(s[0]);
    tmem_ld32(tS + 32, s[1]);
    if (j == 0)
        tmem_wait_ld_regs(s[1]);
    const bool masked = j == n - 1 && p.kv_tail < kBN;
    auto tile_max = [&]() {
        return masked ? half_row_max<true>(s, 64 * h, p.kv_tail) : half_row_max<false>(s, 64 * h, kBN);
    };
    auto exp_store = [&]() {
        const float mc = st.m_use * st.c2;
        return masked ? half_row_exp_store<C, true, C::EXP_EMU>(s, tS, 64 * h, p.kv_tail, st.c2, mc)
                      : half_row_exp_store<C, false, C::EXP_EMU>(s, tS, 64 * h, kBN, st.c2, mc);
    };
    float alpha = 1.f;
    float sum;
    // The first tile sets the running max; later tiles use it as it stands, and
    // only the guard on their sum of p sends a warp back through the max
    // (attn_common.cuh).  tcgen05.st is warp-wide, so the whole warp recomputes
    // and stores P; lanes whose max did not move store the same values again.
    if (j == 0)
        st.m_use = tile_max();
    sum = exp_store();
    bool rescale = false;                    // warp-uniform: only the guard's path changes alpha
    if (j > 0) {
        const bool over = !(sum < (C::FP8 ? kPGuardF16 : kPGuardBF16));
        if (__any_sync(0xffffffffu, over)) {
            rescale = true;
            if (over) {
                const float mx = tile_max();
                if (mx > st.m_use) {
                    alpha = ex2_approx((st.m_use - mx) * st.c2);
                    st.m_use = mx;
                }
            }
            sum = exp_store();
        }
    }
    st.l = st.l * alpha + sum;
    if (rescale) {
        // Rescale this thread's row of O_h once PV(j-1) has finished with it.
        const int jp = j - 1;
        st.alive = __all_sync(0xffffffffu, wait_bar_cluster(x.bar(bars->pv_done[jp % 2]), (jp / 2) & 1,
                                                             x.abort, x.lim, kSiteOFull));
        if (!st.alive)
            return;
        tc_fence_after();
        const uint32_t tO = x.tmem + lane_off + C::TM_O + h * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld_regs(o);
#pragma unroll
            for (int c = 0; c < 32; ++c)
                o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + 32 * cc, o);
        }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0)
        mbar_arrive_cluster(ready_leader);
}

template <class C>
__device__ __forceinline__ void pair_softmax(const PairCtx<C> &x, const FwdParams &p,
                                             const CUtensorMap *tm_o, int warp, int lane)
{
    constexpr int D = C::D;
    auto *bars = x.bars;
    const int h = warp >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    float *red = reinterpret_cast<float *>(x.sm + C::OFF_RED);
    const uint32_t bar_id = 1 + wq;
    const uint32_t ready_leader[2] = {x.leader_bar(bars->ready[0]), x.leader_bar(bars->ready[1])};
    HalfRowState st;
    st.c2 = p.scale * kLog2e;
    float vs = 1.f;
    if (C::FP8) {
        st.c2 = p.scale * p.q_scale[x.bh] * p.k_scale[x.bh] * kLog2e;
        vs = p.v_scale[x.bh];
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
    // (a_0 O_0 + a_1 O_1) / l -> bf16 -> staging -> TMA store; LSE.
    if (alive) {
        const int jl = n - 1;
        alive = __all_sync(0xffffffffu, wait_bar_cluster(x.bar(bars->pv_done[jl % 2]), (jl / 2) & 1, x.abort,
                                                          x.lim, kSiteOFull));
    }
    // A half with no valid key (L < 64) has l = 0 and takes no part.
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
        // This thread writes output columns h*D/2 .. h*D/2 + D/2 of its row.
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
        if (h == 0 && p.lse != nullptr && qrow < p.L)
            p.lse[(long long)x.bh * p.L + qrow] = (mrow + log2f(l_row)) * kLn2;
        if (warp == 0 && lane == 0) {
            for (int b = 0; b < C::OBOX; ++b)
                tma_store_3d(tm_o, ost + b * C::OBOX_BYTES, b * 64, x.q0, x.bh);
            bulk_commit_group();
            bulk_wait_group_all();
        }
    }
}

// ------------------------------------------------------------------ the kernel
template <int D, bool FP8>
__global__ void __launch_bounds__(PCfg<D, FP8>::THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const FwdParams p)
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
    if (warp == C::TMA_WARP && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
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
    x.bh = cluster / p.n_pairs;
    x.q0 = (cluster % p.n_pairs) * 2 * kBM + (int)rank * kBM;

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        if (warp == C::TMA_WARP) {
            if (lane < 2)
                pair_producer<C>(x, p, lane, &tm_q, &tm_k, &tm_v);
        } else if (warp == C::MMA_WARP) {
            if (rank == 0)
                pair_mma<C>(x, p);
        } else if (FP8) {
            pair_convert_v<C>(x, p);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        pair_softmax<C>(x, p, &tm_o, warp, lane);
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
