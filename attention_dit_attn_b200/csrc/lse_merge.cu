// LSE merge of partial attentions (the combine step of ring attention / USP,
// which the xDiT paper cites in its reference list and whose `ring degree`
// setting appears in the 2-GPU script of the page "Accelerating Diffusers and
// xDiT Image Generation with MXFP4 using AMD Quark on AMD Instinct MI350
// GPUs").  For n partial results over disjoint key chunks,
//
//     lse = M + log sum_c exp(lse_c - M),   M = max_c lse_c,
//     o   = sum_c exp(lse_c - lse) o_c,
//
// per row; a row whose parts all have lse = -inf gives o = 0, lse = -inf.
//
// Memory-bound: each row is read once from every part and written once, with
// 16-byte streaming loads (no L1 allocation) and stores.  A row of D bf16 is
// handled by D/8 consecutive lanes of one warp, 8 elements per lane; only the
// row's first lane reads the parts' LSE, computes the weights and writes the
// merged LSE, and shuffles the weights to the other lanes, so the merged
// output may overwrite part 0 (o and lse) in place.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "abi_util.h"
#include "dit_attn.h"

namespace {

constexpr int kMaxParts = DIT_ATTN_MERGE_MAX_PARTS;

struct MergeParams {
    const uint4 *o[kMaxParts];
    const float *lse[kMaxParts];
    uint4 *out;
    float *lse_out;
    long long n_vec;          // rows * D / 8
};

// Plain (coherent) loads: the output may overwrite part 0 within this kernel,
// so the read-only .nc path is not used.  Each element is read once.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream(uint4 *p, uint4 v)
{
    asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float ex2f(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t f2_to_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// The loop runs over groups of 32 vectors (32 / VPR rows) per warp and is
// warp-uniform, so every shuffle has the whole warp converged; lanes past the
// last row only skip their loads and stores.  Each iteration handles U groups
// (U * N 16-byte loads in flight per lane before any of them is used).
template <int N, int VPR, int U>
__global__ void __launch_bounds__(256) lse_merge_kernel(const MergeParams p)
{
    constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
    const int lane = threadIdx.x & 31;
    const bool row_lead = (lane & (VPR - 1)) == 0;
    const long long n_groups = (p.n_vec + 31) >> 5;
    const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long g0 = warp0; g0 < n_groups; g0 += U * n_warps) {
        long long i[U];
        bool valid[U];
        uint4 x[U][N];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            i[u] = ((g0 + u * n_warps) << 5) + lane;
            valid[u] = i[u] < p.n_vec;
            if (valid[u]) {
#pragma unroll
                for (int c = 0; c < N; ++c)
                    x[u][c] = ld_stream(p.o[c] + i[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long row = i[u] / VPR;
            // Weights w_c = exp(lse_c - lse), computed by the row's first lane.
            float w[N];
#pragma unroll
            for (int c = 0; c < N; ++c)
                w[c] = 0.f;
            if (valid[u] && row_lead) {
                float l[N], m = -INFINITY;
#pragma unroll
                for (int c = 0; c < N; ++c) {
                    l[c] = p.lse[c][row];
                    m = fmaxf(m, l[c]);
                }
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < N; ++c) {
                    w[c] = m == -INFINITY ? 0.f : ex2f((l[c] - m) * kLog2e);
                    s += w[c];
                }
                const float inv = s > 0.f ? 1.f / s : 0.f;
#pragma unroll
                for (int c = 0; c < N; ++c)
                    w[c] *= inv;
                if (p.lse_out != nullptr)
                    p.lse_out[row] = s > 0.f ? m + __log2f(s) * kLn2 : -INFINITY;
            }
#pragma unroll
            for (int c = 0; c < N; ++c)
                w[c] = __shfl_sync(0xffffffffu, w[c], 0, VPR);
            if (!valid[u])
                continue;
            float acc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                acc[e] = 0.f;
#pragma unroll
            for (int c = 0; c < N; ++c) {
                const uint32_t v4[4] = {x[u][c].x, x[u][c].y, x[u][c].z, x[u][c].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = bf16x2_to_f2(v4[q]);
                    acc[2 * q] = fmaf(w[c], f.x, acc[2 * q]);
                    acc[2 * q + 1] = fmaf(w[c], f.y, acc[2 * q + 1]);
                }
            }
            uint4 r;
            r.x = f2_to_bf16x2(acc[0], acc[1]);
            r.y = f2_to_bf16x2(acc[2], acc[3]);
            r.z = f2_to_bf16x2(acc[4], acc[5]);
            r.w = f2_to_bf16x2(acc[6], acc[7]);
            st_stream(p.out + i[u], r);
        }
    }
}

// Grid: as many 256-thread blocks as are resident at once on every SM (from
// the occupancy of this instantiation), fewer for small inputs.
template <int N, int VPR>
cudaError_t launch_nv(const MergeParams &p, int sms, cudaStream_t stream)
{
    constexpr int U = N <= 4 ? 2 : 1;
    auto kern = lse_merge_kernel<N, VPR, U>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
    if (e != cudaSuccess)
        return e;
    const long long want = (p.n_vec + 255) / 256;
    const long long full = (long long)(per_sm > 0 ? per_sm : 1) * sms;
    kern<<<(int)(want < full ? want : full), 256, 0, stream>>>(p);
    return cudaGetLastError();
}

template <int N>
cudaError_t launch_n(const MergeParams &p, int vpr, int sms, cudaStream_t stream)
{
    return vpr == 16 ? launch_nv<N, 16>(p, sms, stream) : launch_nv<N, 8>(p, sms, stream);
}

// SM count per device, looked up once per device.
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

} // namespace

extern "C" int dit_attn_lse_merge(const void *const *o_parts, const float *const *lse_parts, int n_parts,
                                  void *o, float *lse, long long rows, int D, cudaStream_t stream)
{
    if (o_parts == nullptr || lse_parts == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (n_parts < 1 || n_parts > kMaxParts || rows < 0 || (D != 64 && D != 128))
        return DIT_ATTN_ERR_SHAPE;
    if (rows * (long long)D >= (1ll << 40))
        return DIT_ATTN_ERR_SHAPE;
    if (rows == 0)
        return DIT_ATTN_OK;             // nothing to read or write: device pointers unused
    if (o == nullptr)
        return DIT_ATTN_ERR_NULL;
    for (int c = 0; c < n_parts; ++c) {
        if (o_parts[c] == nullptr || lse_parts[c] == nullptr)
            return DIT_ATTN_ERR_NULL;
        if (!aligned(o_parts[c], 16) || !aligned(lse_parts[c], 4))
            return DIT_ATTN_ERR_ALIGN;
    }
    if (!aligned(o, 16) || (lse != nullptr && !aligned(lse, 4)))
        return DIT_ATTN_ERR_ALIGN;
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess)
        return DIT_ATTN_ERR_ARCH;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess ||
        major != 10 || minor != 0)
        return DIT_ATTN_ERR_ARCH;
    if (device >= kMaxDevices)
        return DIT_ATTN_ERR_ARCH;
    if (!dit_abi::device_buffers(device, {o, lse}))
        return DIT_ATTN_ERR_DEVICE;
    for (int c = 0; c < n_parts; ++c)
        if (!dit_abi::device_buffers(device, {o_parts[c], lse_parts[c]}))
            return DIT_ATTN_ERR_DEVICE;
    int sms = g_sm_count[device].load(std::memory_order_relaxed);
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        g_sm_count[device].store(sms, std::memory_order_relaxed);
    }
    MergeParams p{};
    for (int c = 0; c < n_parts; ++c) {
        p.o[c] = static_cast<const uint4 *>(o_parts[c]);
        p.lse[c] = lse_parts[c];
    }
    p.out = static_cast<uint4 *>(o);
    p.lse_out = lse;
    p.n_vec = rows * (long long)(D / 8);
    const int vpr = D / 8;
    cudaError_t e;
    switch (n_parts) {
    case 1: e = launch_n<1>(p, vpr, sms, stream); break;
    case 2: e = launch_n<2>(p, vpr, sms, stream); break;
    case 3: e = launch_n<3>(p, vpr, sms, stream); break;
    case 4: e = launch_n<4>(p, vpr, sms, stream); break;
    case 5: e = launch_n<5>(p, vpr, sms, stream); break;
    case 6: e = launch_n<6>(p, vpr, sms, stream); break;
    case 7: e = launch_n<7>(p, vpr, sms, stream); break;
    default: e = launch_n<8>(p, vpr, sms, stream); break;
    }
    return e == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}
