// Flash-style attention forward for B200 (sm_100a): TMA-staged Q/K/V tiles,
// tcgen05 MMAs with TMEM accumulators, online fp32 softmax, warp-specialised
// roles, bf16 and FP8-E4M3 inputs.
//
// Operation: O = softmax(scale * Q K^T) V per (batch, head) with the fp32
// log-sum-exp of each row, the attention core of a DiT block (page "How to
// Scale Diffusion Inference Across AMD RDNA 4 GPUs", sections "Understanding
// the Inference Pipeline" and "Select an Attention Backend and Compile the
// Transformer").  The tiling with a running max and running sum is the
// FlashAttention-2 scheme the pages cite (page "xDiT: an Inference Engine for
// Diffusion Transformers (DiTs) with Massive Parallelism", reference list),
// re-designed here for tcgen05 / TMEM.
//
// One CTA owns a pair of 128-row query tiles of one (b, h) and streams all
// K/V tiles of that head through a shared-memory ring:
//
//   warps 0-3   softmax + epilogue of query tile 0 (one thread per row)
//   warps 4-7   softmax + epilogue of query tile 1
//   warp  8     TMA producer (Q once, then K_j, V_j into the ring)
//   warp  9     MMA issuer (one thread) and TMEM owner
//   warps 10-11 FP8 only: convert each e4m3 V tile to f16 in shared memory
//
// TMEM (512 columns x 128 lanes of 32 bit): S0 | S1 | O0 | O1.  S_g holds the
// fp32 logits of tile g; the softmax overwrites its first 64 (bf16/f16 P)
// columns with P, which the PV MMA reads straight from TMEM.  MMA issue order
//   S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) S0(2) ...
// lets one tile's softmax overlap the other tile's MMAs (ping-pong).  The
// MMAs of one thread run in issue order, so S_g(j+1) (which overwrites P_g(j))
// starts after PV_g(j), and when S_g(j+1) is complete O_g is stable, which is
// when the softmax rescales it.
//
// Rescaling is lazy: a row keeps its running max m while the new tile's max
// exceeds it by at most kRescaleLog2 (in log2 units), so p <= 2^kRescaleLog2;
// O and l are only rescaled when the max grows further.  The result is exact
// because O and l always share the same max.
//
// Every wait is bounded by a time limit; on expiry the kernel records an
// error word, the roles drain their in-flight copies/MMAs and the CTA exits.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

namespace dit {

constexpr int kBM = 128;             // query rows per tile (MMA M)
constexpr int kBN = 128;             // keys per K/V tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f; // lazy-rescale threshold (p <= 256)

// Wait sites recorded in the error word (bits 8..15).
enum : uint32_t {
    kSiteQFull = 1, kSiteKFull = 2, kSitePFull = 3, kSiteVhFull = 4, kSiteKvEmpty = 5,
    kSiteSFull = 6, kSiteOFull = 7, kSiteConvFull = 8, kSiteVhEmpty = 9, kSiteDrain = 10,
    kSiteSelftest = 11
};
constexpr uint32_t kErrTimeout = 7;  // same value as DIT_ATTN_ERR_TIMEOUT

__device__ unsigned int g_error_word;

struct FwdParams {
    int L;
    int n_kv;          // ceil(L / kBN)
    int n_pairs;       // ceil(ceil(L / kBM) / 2)
    int kv_tail;       // valid keys in the last K/V tile, 1..128
    float scale;       // softmax scale
    const float *q_scale;  // FP8: [B*H] dequant scales
    const float *k_scale;
    const float *v_scale;
    float *lse;        // [B*H*L] or null
    unsigned long long wait_limit_ns;
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <int D_, bool FP8_>
struct KCfg {
    static constexpr int D = D_;
    static constexpr bool FP8 = FP8_;
    static constexpr int ELT = FP8 ? 1 : 2;              // bytes per input element
    static constexpr int ROW = D * ELT;                  // bytes per Q/K/V row
    static constexpr int SWZ = ROW >= 128 ? 128 : 64;    // swizzle span of Q/K/V tiles
    static constexpr uint32_t SWZ_MODE = SWZ == 128 ? kSwizzle128B : kSwizzle64B;
    static constexpr int BOX_ELEMS = SWZ / ELT;          // elements per TMA box row
    static constexpr int NBOX = D / BOX_ELEMS;           // TMA boxes per tile
    static constexpr int BOX_BYTES = kBM * SWZ;
    static constexpr int TILE = kBM * ROW;               // one Q/K/V tile in smem
    static constexpr int KSTEP = 32;                     // bytes of K per MMA: 16 x 16-bit or 32 x 8-bit
    static constexpr int QK_STEPS = ROW / KSTEP;
    static constexpr int STEPS_PER_BOX = SWZ / KSTEP;
    // 16-bit V operand of the PV MMA (bf16 or f16), MN-major, 128B swizzle.
    static constexpr int VROW = D * 2;
    static constexpr int VBOX_BYTES = kBN * 128;
    static constexpr int VTILE = kBN * VROW;
    static constexpr int PV_STEPS = kBN / 16;
    // 16-bit O staging tile for the TMA store, 128B swizzle, 64 columns per box.
    static constexpr int OBOX = (D * 2) / 128;
    static constexpr int OBOX_BYTES = kBM * 128;
    static constexpr int OTILE = kBM * D * 2;
    static constexpr int NSTAGE = FP8 ? (D == 64 ? 8 : 4) : (D == 64 ? 8 : 4);
    // Shared-memory layout (offsets from a 1024-byte aligned base).
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = OFF_Q + 2 * align_up(TILE, 1024);
    static constexpr int OFF_VH = OFF_KV + NSTAGE * align_up(TILE, 1024);
    static constexpr int OFF_OST = OFF_VH + (FP8 ? 2 * VTILE : 0);
    static constexpr int OFF_BAR = OFF_OST + (FP8 ? 2 * OTILE : 0);
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
    // TMEM columns.
    static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O0 = 256, TM_O1 = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
    // Warp roles.
    static constexpr int TMA_WARP = 8, MMA_WARP = 9, CONV_WARP0 = 10;
    static constexpr int CONV_THREADS = FP8 ? 64 : 0;
    // Three full warpgroups for every variant, so setmaxnreg can move registers
    // from warpgroup 2 (TMA, MMA, converter) to the two softmax warpgroups:
    // 12 warps x 168 launch registers = (2 x 208 + 88) x 128 threads.  The
    // wait helpers are all inlined: a real call across warpgroups with
    // different register budgets does not allocate.
    static constexpr int THREADS = 384;
    static constexpr int REGS_SOFTMAX = 208, REGS_OTHER = 88;
    // Element pairs (of every 8) whose exponential runs on the FMA pipe.
#ifndef DIT_EXP_EMU
#define DIT_EXP_EMU 2
#endif
    static constexpr int EXP_EMU = DIT_EXP_EMU;
    static_assert(2 * REGS_SOFTMAX + REGS_OTHER == 3 * 168, "register split = launch budget");
    // Instruction descriptors (M = 128 rows).
    static constexpr uint32_t IDESC_QK =
        FP8 ? make_idesc(kFmtE4M3, kFmtE4M3, 0, kBM, kBN) : make_idesc(kFmtBF16, kFmtBF16, 0, kBM, kBN);
    static constexpr uint32_t IDESC_PV =
        FP8 ? make_idesc(kFmtF16, kFmtF16, 1, kBM, D) : make_idesc(kFmtBF16, kFmtBF16, 1, kBM, D);

    static_assert(D == 64 || D == 128, "head dim");
    static_assert(NBOX * BOX_BYTES == TILE, "tile = whole boxes");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(TM_O1 + D <= TMEM_COLS, "TMEM budget");
};

// Barrier block in shared memory.
template <int NS>
struct Bars {
    uint64_t q_full;
    uint64_t kv_full[NS];
    uint64_t kv_empty[NS];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_full[2];
    uint64_t vh_full[2];
    uint64_t vh_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

// ------------------------------------------------------------------ bounded waits

__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
                                       unsigned long long limit, uint32_t site)
{
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

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t *abort,
                                         unsigned long long limit, uint32_t site)
{
    if (mbar_try_wait(bar, parity))
        return true;
    return wait_slow(bar, parity, abort, limit, site);
}

// Named barrier with an AND-reduction: every participant learns whether all
// of them are still healthy (keeps later decisions uniform).
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

__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_p(float lo, float hi, bool f16)
{
    if (f16) {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&h);
    }
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&b);
}

__device__ __forceinline__ uint32_t cvt_e4m3x2_to_f16x2(uint32_t two_codes)
{
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(r)
        : "r"(two_codes));
    return r;
}

// Byte offset of a 16-byte chunk inside a swizzled tile: the swizzle XORs
// the chunk bits [4, 4+log2(span/16)) with the row bits [7, ...).
template <int SPAN>
__device__ __forceinline__ uint32_t swz(uint32_t off)
{
    constexpr uint32_t mask = SPAN == 128 ? 0x70u : (SPAN == 64 ? 0x30u : 0x10u);
    return off ^ ((off >> 3) & mask);
}

// ------------------------------------------------------------------ softmax of one S tile

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for a pair, on the FMA/ALU pipes instead of MUFU.  x = n + f with
// n = rint(x) (adding 1.5*2^23 leaves rint(x) in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f is a cubic fitted for minimum max relative error on
// [-1/2, 1/2] (max rel. error 7.5e-5, below the half-ulp of bf16 and f16 P);
// 2^n is added to the exponent field.  x is clamped to >= -126 so the
// exponent never underflows; the callers guarantee x <= 9.
constexpr float kPolyC0 = 0.9999281167984009f, kPolyC1 = 0.6932609677314758f,
                kPolyC2 = 0.24261052906513214f, kPolyC3 = 0.05517127364873886f;
constexpr float kRintMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ float2 exp2_poly2(float2 x)
{
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    const float2 t = __fadd2_rn(x, make_float2(kRintMagic, kRintMagic));
    const float2 n = __fadd2_rn(t, make_float2(-kRintMagic, -kRintMagic));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 q = __ffma2_rn(f, make_float2(kPolyC3, kPolyC3), make_float2(kPolyC2, kPolyC2));
    q = __ffma2_rn(q, f, make_float2(kPolyC1, kPolyC1));
    q = __ffma2_rn(q, f, make_float2(kPolyC0, kPolyC0));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

// Loads this thread's row of S (128 fp32), updates the running max / sum,
// writes P (16-bit) over the S columns and rescales O when needed.  P chunk
// i (S columns 32i..32i+31) goes to columns 16i..16i+15, which hold S values
// already consumed, so P can be stored chunk by chunk.  Of every 8 element
// pairs, EMU pairs take 2^x from exp2_poly2 (FMA pipe), the rest from MUFU,
// which balances the two pipes.
template <class C, bool MASK, int EMU>
__device__ __forceinline__ void softmax_tile(uint32_t tS, uint32_t tO, int valid, bool first,
                                             float c2, float &m_use, float &l)
{
    uint32_t s[4][32];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        tmem_ld32(tS + 32 * i, s[i]);
    tmem_wait_ld();

    if (MASK) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (32 * i + c >= valid)
                    s[i][c] = __float_as_uint(-INFINITY);
    }
    // Row max: 8 independent chains of 3-input max, then a short tree.
    float m8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        m8[k] = fmaxf(__uint_as_float(s[0][2 * k]), __uint_as_float(s[0][2 * k + 1]));
#pragma unroll
    for (int e = 16; e < 128; e += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k)
            m8[k] = max3f(m8[k], __uint_as_float(s[e >> 5][(e & 31) + 2 * k]),
                          __uint_as_float(s[e >> 5][(e & 31) + 2 * k + 1]));
    const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));

    float alpha = 1.f;
    if (first) {
        m_use = mx;
    } else if ((mx - m_use) * c2 > kRescaleLog2) {
        alpha = ex2_approx((m_use - mx) * c2);
        m_use = mx;
    }
    const float mc = m_use * c2;
    const float2 c2c2 = make_float2(c2, c2), nmc = make_float2(-mc, -mc);

    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                     make_float2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
            const int pi = (32 * i + c) >> 1;     // pair index 0..63
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[i][c]), __uint_as_float(s[i][c + 1])),
                                        c2c2, nmc);
            float2 e;
            if ((pi & 7) >= 8 - EMU) {
                e = exp2_poly2(x);
            } else {
                e.x = ex2_approx(x.x);
                e.y = ex2_approx(x.y);
            }
            if (MASK) {
                e.x = (32 * i + c < valid) ? e.x : 0.f;
                e.y = (32 * i + c + 1 < valid) ? e.y : 0.f;
            }
            acc[pi & 3] = __fadd2_rn(acc[pi & 3], e);
            pk[c / 2] = pack_p(e.x, e.y, C::FP8);
        }
        tmem_st16(tS + 16 * i, pk);
    }
    const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
    const float2 a = __fadd2_rn(a01, a23);
    l = l * alpha + (a.x + a.y);

    // After the exponentials (S registers dead).  O is stable here: S_g(j)
    // complete implies PV_g(j-1) complete.
    if (!first && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int cc = 0; cc < C::D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c)
                o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + 32 * cc, o);
        }
    }
    tmem_wait_st();
}

// ------------------------------------------------------------------ roles
// Shared state every role sees.
template <class C>
struct Ctx {
    Bars<C::NSTAGE> *bars;
    uint32_t base;                 // 1024-aligned shared-memory base address
    uint32_t tmem;                 // TMEM base address
    volatile uint32_t *abort;      // CTA-wide abort flag
    unsigned long long lim;        // wait limit, ns
    int bh, q0;                    // (b, h) index and first query row of the pair
    __device__ uint32_t bar(const uint64_t &b) const { return smem_u32(&b); }
};

// TMA producer (one thread): both Q tiles once, then K_j, V_j into the ring.
template <class C>
__device__ __forceinline__ void producer_role(const Ctx<C> &x, const FwdParams &p,
                                              const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                              const CUtensorMap *tm_v)
{
    constexpr int NS = C::NSTAGE;
    auto *bars = x.bars;
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    mbar_arrive_expect_tx(x.bar(bars->q_full), 2 * C::TILE);
    for (int g = 0; g < 2; ++g)
        for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(x.base + C::OFF_Q + g * C::TILE + b * C::BOX_BYTES, tm_q, x.bar(bars->q_full),
                        b * C::BOX_ELEMS, x.q0 + g * kBM, x.bh, pol_q);
    int last_round[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s)
        last_round[s] = -1;
    const int n_loads = 2 * p.n_kv;
    for (int t = 0; t < n_loads; ++t) {
        const int st = t % NS, rd = t / NS;
        if (!wait_bar(x.bar(bars->kv_empty[st]), (rd & 1) ^ 1, x.abort, x.lim, kSiteKvEmpty))
            break;
        const uint32_t fb = x.bar(bars->kv_full[st]);
        mbar_arrive_expect_tx(fb, C::TILE);
        const CUtensorMap *m = (t & 1) ? tm_v : tm_k;
        for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d(x.base + C::OFF_KV + st * C::TILE + b * C::BOX_BYTES, m, fb, b * C::BOX_ELEMS,
                        (t >> 1) * kBN, x.bh, pol_kv);
#pragma unroll
        for (int s = 0; s < NS; ++s)
            if (s == st)
                last_round[s] = rd;
    }
    if (*x.abort) {
        // Let copies already in flight land before the CTA exits (bounded).
        constexpr unsigned long long kDrainNs = 50000000ull;
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            if (last_round[s] < 0)
                continue;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(x.bar(bars->kv_full[s]), last_round[s] & 1) &&
                   globaltimer_ns() - t0 < kDrainNs) {
            }
        }
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(x.bar(bars->q_full), 0) && globaltimer_ns() - t0 < kDrainNs) {
        }
    }
}

// MMA issuer (one thread).  Issue order per K/V tile j:
//   PV0(j), S0(j+1), PV1(j), S1(j+1)   after the prologue S0(0), S1(0).
template <class C>
__device__ __forceinline__ void mma_role(const Ctx<C> &x, const FwdParams &p)
{
    constexpr int NS = C::NSTAGE;
    auto *bars = x.bars;
    auto issue_s = [&](int g, uint32_t k_addr) {
        const uint32_t q_addr = x.base + C::OFF_Q + g * C::TILE;
        const uint32_t tS = x.tmem + (g ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < C::QK_STEPS; ++kk) {
            const uint32_t off =
                (kk / C::STEPS_PER_BOX) * C::BOX_BYTES + (kk % C::STEPS_PER_BOX) * C::KSTEP;
            const uint64_t ad = make_smem_desc(q_addr + off, 16, 8 * C::SWZ, C::SWZ_MODE);
            const uint64_t bd = make_smem_desc(k_addr + off, 16, 8 * C::SWZ, C::SWZ_MODE);
            if (C::FP8)
                mma_f8_ss(tS, ad, bd, C::IDESC_QK, kk > 0);
            else
                mma_f16_ss(tS, ad, bd, C::IDESC_QK, kk > 0);
        }
    };
    auto issue_pv = [&](int g, uint32_t v_addr, bool acc) {
        const uint32_t tS = x.tmem + (g ? C::TM_S1 : C::TM_S0);
        const uint32_t tO = x.tmem + (g ? C::TM_O1 : C::TM_O0);
#pragma unroll
        for (int kk = 0; kk < C::PV_STEPS; ++kk) {
            const uint64_t bd =
                make_smem_desc(v_addr + kk * 16 * 128, C::VBOX_BYTES, 1024, kSwizzle128B);
            mma_f16_ts(tO, tS + kk * 8, bd, C::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
    };

    bool ok = wait_bar(x.bar(bars->q_full), 0, x.abort, x.lim, kSiteQFull) &&
              wait_bar(x.bar(bars->kv_full[0]), 0, x.abort, x.lim, kSiteKFull);
    if (ok) {
        tc_fence_after();
        const uint32_t k_addr = x.base + C::OFF_KV;
        issue_s(0, k_addr);
        mma_commit(x.bar(bars->s_full[0]));
        issue_s(1, k_addr);
        mma_commit(x.bar(bars->s_full[1]));
        mma_commit(x.bar(bars->kv_empty[0]));
    }
    for (int j = 0; ok && j < p.n_kv; ++j) {
        const bool has_next = j + 1 < p.n_kv;
        uint32_t v_addr;
        int sv = 0;
        if (C::FP8) {
            ok = wait_bar(x.bar(bars->vh_full[j & 1]), (j >> 1) & 1, x.abort, x.lim, kSiteVhFull);
            v_addr = x.base + C::OFF_VH + (j & 1) * C::VTILE;
        } else {
            const int t = 2 * j + 1;
            sv = t % NS;
            ok = wait_bar(x.bar(bars->kv_full[sv]), (t / NS) & 1, x.abort, x.lim, kSiteKFull);
            v_addr = x.base + C::OFF_KV + sv * C::TILE;
        }
        int sk = 0;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            ok = ok && wait_bar(x.bar(bars->p_full[g]), j & 1, x.abort, x.lim, kSitePFull);
            if (!ok)
                break;
            tc_fence_after();
            issue_pv(g, v_addr, j > 0);
            if (!has_next)
                mma_commit(x.bar(bars->o_full[g]));
            if (g == 1)
                mma_commit(C::FP8 ? x.bar(bars->vh_empty[j & 1]) : x.bar(bars->kv_empty[sv]));
            if (has_next) {
                if (g == 0) {
                    const int t = 2 * (j + 1);
                    sk = t % NS;
                    ok = wait_bar(x.bar(bars->kv_full[sk]), (t / NS) & 1, x.abort, x.lim, kSiteKFull);
                    if (!ok)
                        break;
                    tc_fence_after();
                }
                issue_s(g, x.base + C::OFF_KV + sk * C::TILE);
                mma_commit(x.bar(bars->s_full[g]));
                if (g == 1)
                    mma_commit(x.bar(bars->kv_empty[sk]));
            }
        }
    }
    if (!ok) {
        // Wait (bounded) until every MMA issued so far has finished.
        mma_commit(x.bar(bars->drain));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(x.bar(bars->drain), 0) && globaltimer_ns() - t0 < 50000000ull) {
        }
    }
}

// FP8 path (warps 10-11): converts each e4m3 V tile of the ring into a
// 16-bit (f16) MN-major 128B-swizzled tile for the PV MMA, then releases the
// ring stage.  e4m3 values are exact in f16.
template <class C>
__device__ __forceinline__ void convert_v_role(const Ctx<C> &x, const FwdParams &p)
{
    constexpr int NS = C::NSTAGE;
    auto *bars = x.bars;
    const int ct = threadIdx.x - C::CONV_WARP0 * 32;   // 0..63
    constexpr int CHUNKS = kBN * C::ROW / 16;          // raw 16-byte chunks per V tile
    for (int j = 0; j < p.n_kv; ++j) {
        const int t = 2 * j + 1, st = t % NS;
        bool ok = wait_bar(x.bar(bars->kv_full[st]), (t / NS) & 1, x.abort, x.lim, kSiteConvFull);
        ok = ok && wait_bar(x.bar(bars->vh_empty[j & 1]), ((j >> 1) & 1) ^ 1, x.abort, x.lim,
                            kSiteVhEmpty);
        if (!bar_and(3, C::CONV_THREADS, ok))
            break;
        const uint32_t src = x.base + C::OFF_KV + st * C::TILE;
        const uint32_t dst = x.base + C::OFF_VH + (j & 1) * C::VTILE;
        for (int idx = ct; idx < CHUNKS; idx += C::CONV_THREADS) {
            const int r = idx / (C::ROW / 16);      // key row
            const int d0 = (idx % (C::ROW / 16)) * 16;  // first of 16 elements
            const uint32_t roff = (d0 / C::BOX_ELEMS) * C::BOX_BYTES +
                                  swz<C::SWZ>((uint32_t)r * C::SWZ + (uint32_t)(d0 % C::BOX_ELEMS));
            uint32_t w[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(src + roff));
            uint32_t h[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                h[2 * i] = cvt_e4m3x2_to_f16x2(w[i] & 0xFFFFu);
                h[2 * i + 1] = cvt_e4m3x2_to_f16x2(w[i] >> 16);
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int d = d0 + 8 * half;        // 8 f16 = one 16-byte chunk
                const uint32_t doff =
                    (d / 64) * C::VBOX_BYTES + swz<128>((uint32_t)r * 128u + (uint32_t)(d % 64) * 2u);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + doff),
                             "r"(h[4 * half]), "r"(h[4 * half + 1]), "r"(h[4 * half + 2]),
                             "r"(h[4 * half + 3])
                             : "memory");
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(3, C::CONV_THREADS);
        if (ct == 0) {
            mbar_arrive(x.bar(bars->vh_full[j & 1]));
            mbar_arrive(x.bar(bars->kv_empty[st]));
        }
    }
}

// Softmax + epilogue of query tile g (warps 4g..4g+3, one thread per row).
template <class C>
__device__ __forceinline__ void softmax_role(const Ctx<C> &x, const FwdParams &p,
                                             const CUtensorMap *tm_o, int warp, int lane)
{
    constexpr int D = C::D;
    auto *bars = x.bars;
    const int g = warp >> 2;
    const int wq = warp & 3;             // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;      // row inside query tile g
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = x.tmem + lane_off + (g ? C::TM_S1 : C::TM_S0);
    const uint32_t tO = x.tmem + lane_off + (g ? C::TM_O1 : C::TM_O0);
    float c2 = p.scale * kLog2e;         // logit scale in log2 units
    float vs = 1.f;
    if (C::FP8) {
        c2 = p.scale * p.q_scale[x.bh] * p.k_scale[x.bh] * kLog2e;
        vs = p.v_scale[x.bh];
    }
    float m_use = -INFINITY, l = 0.f;
    bool alive = true;
    for (int j = 0; j < p.n_kv; ++j) {
        const bool ok = wait_bar(x.bar(bars->s_full[g]), j & 1, x.abort, x.lim, kSiteSFull);
        if (!__all_sync(0xffffffffu, ok)) {
            alive = false;
            break;
        }
        tc_fence_after();
        if (j + 1 < p.n_kv || p.kv_tail == kBN)
            softmax_tile<C, false, C::EXP_EMU>(tS, tO, kBN, j == 0, c2, m_use, l);
        else
            softmax_tile<C, true, C::EXP_EMU>(tS, tO, p.kv_tail, j == 0, c2, m_use, l);
        tc_fence_before();
        mbar_arrive(x.bar(bars->p_full[g]));
    }
    // ---- epilogue: O / l -> bf16 -> swizzled staging smem -> TMA store; LSE.
    if (alive)
        alive = __all_sync(0xffffffffu,
                           wait_bar(x.bar(bars->o_full[g]), 0, x.abort, x.lim, kSiteOFull));
    const uint32_t ost =
        C::FP8 ? x.base + C::OFF_OST + g * C::OTILE : x.base + C::OFF_Q + g * C::TILE;
    if (alive) {
        tc_fence_after();
        const float inv = vs / l;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pack_p(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv,
                               false);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int chunk = 4 * cc + k4;   // 16-byte chunk of this row
                const uint32_t off = (chunk >> 3) * C::OBOX_BYTES +
                                     swz<128>((uint32_t)row * 128u + (uint32_t)(chunk & 7) * 16u);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ost + off),
                             "r"(pk[4 * k4]), "r"(pk[4 * k4 + 1]), "r"(pk[4 * k4 + 2]),
                             "r"(pk[4 * k4 + 3])
                             : "memory");
            }
        }
        fence_proxy_async_smem();
    }
    alive = bar_and(1 + g, 128, alive);
    if (alive) {
        const int qrow = x.q0 + g * kBM + row;
        if (p.lse != nullptr && qrow < p.L)
            p.lse[(long long)x.bh * p.L + qrow] = (m_use * c2 + log2f(l)) * kLn2;
        if (row == 0) {
            for (int b = 0; b < C::OBOX; ++b)
                tma_store_3d(tm_o, ost + b * C::OBOX_BYTES, b * 64, x.q0 + g * kBM, x.bh);
            bulk_commit_group();
            bulk_wait_group_all();
        }
    }
}

// ------------------------------------------------------------------ the kernel

template <int D, bool FP8>
__global__ void __launch_bounds__(KCfg<D, FP8>::THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const FwdParams p)
{
    using C = KCfg<D, FP8>;
    constexpr int NS = C::NSTAGE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    Bars<NS> *bars = reinterpret_cast<Bars<NS> *>(smem_raw + (base - raw_addr) + C::OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- set-up: barriers (one thread), TMEM (MMA warp)
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars->q_full), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&bars->kv_full[s]), 1);
            mbar_init(smem_u32(&bars->kv_empty[s]), 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(smem_u32(&bars->s_full[g]), 1);
            mbar_init(smem_u32(&bars->p_full[g]), kBM);
            mbar_init(smem_u32(&bars->o_full[g]), 1);
            mbar_init(smem_u32(&bars->vh_full[g]), 1);
            mbar_init(smem_u32(&bars->vh_empty[g]), 1);
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
        tmem_alloc(smem_u32(&bars->tmem_base), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    Ctx<C> x;
    x.bars = bars;
    x.base = base;
    x.tmem = bars->tmem_base;
    x.abort = &bars->abort;
    x.lim = p.wait_limit_ns;
    x.bh = blockIdx.x / p.n_pairs;
    x.q0 = (blockIdx.x % p.n_pairs) * 2 * kBM;

    if (warp >= 8) {
        // Warpgroup 2: producer, MMA issuer, converter.  Each warpgroup sets
        // its register budget at the top of its own branch.
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_OTHER));
        if (warp == C::TMA_WARP) {
            if (lane == 0)
                producer_role<C>(x, p, &tm_q, &tm_k, &tm_v);
        } else if (warp == C::MMA_WARP) {
            if (lane == 0)
                mma_role<C>(x, p);
        } else if (FP8) {
            convert_v_role<C>(x, p);
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFTMAX));
        softmax_role<C>(x, p, &tm_o, warp, lane);
    }

    // ---- tear-down
    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(x.tmem, C::TMEM_COLS);
    }
}

// Self-test of the bounded wait: one thread waits on an mbarrier nothing completes.
__global__ void selftest_wait_kernel(unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t abort;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        wait_bar(smem_u32(&bar), 0, reinterpret_cast<volatile uint32_t *>(&abort), limit_ns,
                 kSiteSelftest);
    __syncthreads();
}

} // namespace dit
