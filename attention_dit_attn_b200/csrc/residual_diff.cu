// Step-cache reuse decision (DBCache: page "How to Scale Diffusion Inference
// Across AMD RDNA 4 GPUs", section "Skip Transformer Work Only When the Model
// Has Enough Steps"): the relative L1 change of the first blocks' residual
// between consecutive denoising steps,
//
//     diff = sum_i |r_i - r'_i| / sum_i |r'_i|,    reuse <=> diff < threshold,
//
// (0 if both sums are 0, +inf if only the denominator is).  The page names
// the threshold (0.12 in the published setting) but no formula; this is the
// plainest reading.
//
// One HBM-bound pass over both bf16 residuals with 16-byte loads.  Each
// thread accumulates in fp32 over its few elements; each block reduces to two
// fp64 partial sums in the workspace.  The last block to finish (an atomic
// ticket) adds the partials in a fixed order in fp64, takes the decision,
// writes diff and the flag, and resets the ticket, so the result is
// bit-reproducible and the workspace is left ready for the next call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "abi_util.h"
#include "dit_attn.h"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxBlocks = 1184;            // 8 blocks x 148 SMs
constexpr size_t kHeaderBytes = 16;         // ticket (u32), padded

struct DiffParams {
    const uint4 *cur;
    const uint4 *prev;
    long long n;             // elements
    float threshold;
    unsigned int *ticket;    // workspace + 0
    double2 *partials;       // workspace + kHeaderBytes: (num, den) per block
    float *diff_out;
    int *reuse_out;
};

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void acc_pair(uint32_t c, uint32_t p, float &num, float &den)
{
    const float c0 = __uint_as_float(c << 16), c1 = __uint_as_float(c & 0xFFFF0000u);
    const float p0 = __uint_as_float(p << 16), p1 = __uint_as_float(p & 0xFFFF0000u);
    num += fabsf(c0 - p0) + fabsf(c1 - p1);
    den += fabsf(p0) + fabsf(p1);
}

__device__ __forceinline__ void acc_vec(uint4 c, uint4 p, float &num, float &den)
{
    acc_pair(c.x, p.x, num, den);
    acc_pair(c.y, p.y, num, den);
    acc_pair(c.z, p.z, num, den);
    acc_pair(c.w, p.w, num, den);
}

// Sum of v over the block in fp64, in a fixed order; the result is valid in thread 0.
__device__ __forceinline__ double block_sum(double v, double *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_down_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0)
        for (int w = 0; w < kThreads / 32; ++w)
            s += red[w];
    return s;
}

__global__ void __launch_bounds__(kThreads) residual_diff_kernel(const DiffParams p)
{
    __shared__ double red[kThreads / 32];
    __shared__ bool last;
    const long long n_vec = p.n >> 3;
    const long long stride = (long long)gridDim.x * kThreads;
    float num = 0.f, den = 0.f;
    long long i = (long long)blockIdx.x * kThreads + threadIdx.x;
    // Four vector pairs (128 bytes) in flight per thread before any is used.
    for (; i + 3 * stride < n_vec; i += 4 * stride) {
        uint4 c[4], q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            c[u] = ld_stream(p.cur + i + u * stride);
            q[u] = ld_stream(p.prev + i + u * stride);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            acc_vec(c[u], q[u], num, den);
    }
    for (; i < n_vec; i += stride)
        acc_vec(ld_stream(p.cur + i), ld_stream(p.prev + i), num, den);
    // Elements past the last whole 16-byte vector (n % 8 of them): block 0.
    if (blockIdx.x == 0 && threadIdx.x < (int)(p.n & 7)) {
        const uint16_t *c = reinterpret_cast<const uint16_t *>(p.cur) + (n_vec << 3) + threadIdx.x;
        const uint16_t *q = reinterpret_cast<const uint16_t *>(p.prev) + (n_vec << 3) + threadIdx.x;
        const float cv = __uint_as_float((uint32_t)*c << 16), pv = __uint_as_float((uint32_t)*q << 16);
        num += fabsf(cv - pv);
        den += fabsf(pv);
    }
    const double bnum = block_sum((double)num, red);
    const double bden = block_sum((double)den, red);
    if (threadIdx.x == 0) {
        p.partials[blockIdx.x] = make_double2(bnum, bden);
        __threadfence();
        last = atomicAdd(p.ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!last)
        return;
    // Last block: fixed-order fp64 sum of all partials.
    __threadfence();
    double tnum = 0.0, tden = 0.0;
    for (int b = threadIdx.x; b < (int)gridDim.x; b += kThreads) {
        const double2 v = __ldcg(p.partials + b);
        tnum += v.x;
        tden += v.y;
    }
    const double snum = block_sum(tnum, red);
    const double sden = block_sum(tden, red);
    if (threadIdx.x == 0) {
        const double diff = sden > 0.0 ? snum / sden : (snum > 0.0 ? INFINITY : 0.0);
        if (p.diff_out != nullptr)
            *p.diff_out = (float)diff;
        if (p.reuse_out != nullptr)
            *p.reuse_out = diff < (double)p.threshold ? 1 : 0;
        *p.ticket = 0u;               // ready for the next call
    }
}

// Blocks for n elements: enough for 4 vectors per thread, at most the blocks
// resident at once on the device (from occupancy) and at most kMaxBlocks,
// which bounds the workspace independently of the device.
int blocks_for(long long n, int resident)
{
    const long long want = ((n >> 3) + 4ll * kThreads - 1) / (4ll * kThreads);
    const long long cap = resident < kMaxBlocks ? resident : kMaxBlocks;
    return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

// Resident blocks per device (occupancy x SM count), looked up once per device.
constexpr int kMaxDevices = 64;
std::atomic<int> g_resident[kMaxDevices];

// Scratch of the no-allocation entry point: the largest workspace any n needs,
// in the module's own device memory (zero at load; every call leaves it zero).
constexpr size_t kScratchBytes = kHeaderBytes + sizeof(double2) * kMaxBlocks;
static __device__ __align__(256) unsigned char g_diff_scratch[kScratchBytes];

// Its address per device, looked up once per CUDA context: a context made
// after cudaDeviceReset loads the module again, at a new address.  Contexts
// are told apart by their process-unique id (cuCtxGetId), never reused.
struct ScratchAddr {
    unsigned long long ctx_id;
    void *addr;
};
std::mutex g_scratch_mu;
ScratchAddr g_scratch_addr[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
template <class Fn>
Fn driver_fn(const char *name)
{
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(ptr);
    return nullptr;
}

// Id of the context current on this thread (0 when none can be had).
unsigned long long current_ctx_id()
{
    static std::once_flag once;
    static CtxGetCurrentFn get_ctx = nullptr;
    static CtxGetIdFn get_id = nullptr;
    std::call_once(once, [] {
        get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    // cudaFree(0) makes the device's primary context current if none is yet.
    if (get_ctx == nullptr || get_id == nullptr || cudaFree(0) != cudaSuccess || get_ctx(&ctx) != CUDA_SUCCESS ||
        ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id + 1;   // 0 stays "none"
}

bool aligned(const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; }

} // namespace

extern "C" size_t dit_attn_residual_diff_workspace_bytes(long long n)
{
    if (n < 1)
        return 0;
    return kHeaderBytes + sizeof(double2) * (size_t)blocks_for(n, kMaxBlocks);
}

extern "C" int dit_attn_residual_diff(const void *cur, const void *prev, long long n, float threshold,
                                      void *workspace, size_t workspace_bytes, float *diff_out, int *reuse_out,
                                      cudaStream_t stream)
{
    if (cur == nullptr || prev == nullptr || workspace == nullptr || (diff_out == nullptr && reuse_out == nullptr))
        return DIT_ATTN_ERR_NULL;
    if (n < 1 || n >= (1ll << 40))
        return DIT_ATTN_ERR_SHAPE;
    if (!aligned(cur, 16) || !aligned(prev, 16) || !aligned(workspace, 16) ||
        (diff_out != nullptr && !aligned(diff_out, 4)) || (reuse_out != nullptr && !aligned(reuse_out, 4)))
        return DIT_ATTN_ERR_ALIGN;
    if (std::isnan(threshold))
        return DIT_ATTN_ERR_VALUE;
    if (workspace_bytes < dit_attn_residual_diff_workspace_bytes(n))
        return DIT_ATTN_ERR_SHAPE;
    int device = 0, major = 0, minor = 0;
    if (cudaGetDevice(&device) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess ||
        major != 10 || minor != 0)
        return DIT_ATTN_ERR_ARCH;
    if (device >= kMaxDevices)
        return DIT_ATTN_ERR_ARCH;
    if (!dit_abi::device_buffers(device, {cur, prev, workspace, diff_out, reuse_out}))
        return DIT_ATTN_ERR_DEVICE;
    int resident = g_resident[device].load(std::memory_order_relaxed);
    if (resident == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, residual_diff_kernel, kThreads, 0) !=
                cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        resident = (per_sm > 0 ? per_sm : 1) * sms;
        g_resident[device].store(resident, std::memory_order_relaxed);
    }
    DiffParams p{};
    p.cur = static_cast<const uint4 *>(cur);
    p.prev = static_cast<const uint4 *>(prev);
    p.n = n;
    p.threshold = threshold;
    p.ticket = static_cast<unsigned int *>(workspace);
    p.partials = reinterpret_cast<double2 *>(static_cast<char *>(workspace) + kHeaderBytes);
    p.diff_out = diff_out;
    p.reuse_out = reuse_out;
    residual_diff_kernel<<<blocks_for(n, resident), kThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

extern "C" int dit_attn_residual_diff_noalloc(const void *cur, const void *prev, long long n, float threshold,
                                              float *diff_out, int *reuse_out, cudaStream_t stream)
{
    if (n < 1 || n >= (1ll << 40) || dit_attn_residual_diff_workspace_bytes(n) > kScratchBytes)
        return DIT_ATTN_ERR_SHAPE;
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices)
        return DIT_ATTN_ERR_ARCH;
    const unsigned long long ctx_id = current_ctx_id();
    if (ctx_id == 0)
        return DIT_ATTN_ERR_ARCH;
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        ScratchAddr &slot = g_scratch_addr[device];
        if (slot.ctx_id != ctx_id || slot.addr == nullptr) {
            if (cudaGetSymbolAddress(&slot.addr, g_diff_scratch) != cudaSuccess) {
                slot.addr = nullptr;
                slot.ctx_id = 0;
                return DIT_ATTN_ERR_ARCH;
            }
            slot.ctx_id = ctx_id;
        }
        scratch = slot.addr;
    }
    return dit_attn_residual_diff(cur, prev, n, threshold, scratch, kScratchBytes, diff_out, reuse_out, stream);
}
