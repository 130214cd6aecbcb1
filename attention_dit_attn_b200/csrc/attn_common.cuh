// Shared pieces of the attention forward kernel for B200 (sm_100a): tile
// sizes, kernel parameters, the device error word, bounded mbarrier waits and
// the small arithmetic helpers of the softmax.
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
// Every wait is bounded by a time limit; on expiry the kernel records an
// error word, the roles drain their in-flight copies/MMAs and the CTAs exit.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100_ptx.cuh"

namespace dit {

constexpr int kBM = 128;             // query rows per tile (MMA M)
constexpr int kBN = 128;             // keys per K/V tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Lazy rescaling without a per-tile max: a half-row keeps the running max of
// its first key tile, so a later tile's p = 2^(x - m) may exceed 1.  The sum
// of the thread's p over a tile bounds each of them; when that sum reaches the
// guard (or is not finite) the warp takes the rescale path: the tile's max,
// O and l scaled down, P recomputed.  f16 P (FP8 path) must stay below 65504;
// bf16 P and the fp32 accumulators (O, l) have room for 2^64 per p.
constexpr float kPGuardF16 = 32768.0f;                   // 2^15
constexpr float kPGuardBF16 = 18446744073709551616.0f;   // 2^64


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
// 2^n is added to the exponent field.  x is clamped to [-126, 127], so the
// exponent field neither underflows nor wraps: a larger x (x is not bounded by
// a per-tile max) gives 2^127, which the caller's guard on the sum of p
// catches as it catches MUFU's +inf.
constexpr float kPolyC0 = 0.9999281167984009f, kPolyC1 = 0.6932609677314758f,
                kPolyC2 = 0.24261052906513214f, kPolyC3 = 0.05517127364873886f;
constexpr float kRintMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ float2 exp2_poly2(float2 x)
{
    x.x = fminf(fmaxf(x.x, -126.f), 127.f);
    x.y = fminf(fmaxf(x.y, -126.f), 127.f);
    const float2 t = __fadd2_rn(x, make_float2(kRintMagic, kRintMagic));
    const float2 n = __fadd2_rn(t, make_float2(-kRintMagic, -kRintMagic));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 q = __ffma2_rn(f, make_float2(kPolyC3, kPolyC3), make_float2(kPolyC2, kPolyC2));
    q = __ffma2_rn(q, f, make_float2(kPolyC1, kPolyC1));
    q = __ffma2_rn(q, f, make_float2(kPolyC0, kPolyC0));
    return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

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
