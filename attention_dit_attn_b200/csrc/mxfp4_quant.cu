// MXFP4 1x32 activation quantiser (page "Accelerating Diffusers and xDiT
// Image Generation with MXFP4 using AMD Quark on AMD Instinct MI350 GPUs",
// sections "MXFP4 Quantization" and "MXFP4 Kernel": activations of the linear
// layers are quantised on the fly to the OCP Microscaling MXFP4 format the
// page cites).  For every 32 consecutive values of a row:
//
//     s   = clamp(floor(log2(max |v|)) - 2, -127, 127)    (-127 for a zero block)
//     q_i = E2M1(v_i / 2^s), round to nearest even, saturate at +-6
//
// stored as the E8M0 byte s + 127 and 16 bytes of codes (first element of each
// pair in the low 4 bits).  The page does not restate the rule; this is the OCP
// MX definition it points to.
//
// Memory-bound: four lanes per 32-value block, each with one 16-byte load of 8
// bf16, so a warp reads 512 contiguous bytes and writes 128 contiguous bytes of
// codes.  The block max is combined with two shuffles; the exponent comes from
// the max's float bits; the scaling by 2^-s is exact; the rounding and packing
// use cvt.rn.satfinite.e2m1x2.f32.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "abi_util.h"
#include "dit_attn.h"

namespace {

constexpr int kThreads = 256;

struct QuantParams {
    const uint4 *x;           // bf16, 8 per uint4
    uint32_t *q;              // 8 codes per uint32
    uint8_t *scales;          // one per 32 values
    long long n_vec;          // rows * K / 8
};

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Two values -> one byte of E2M1 codes: `lo` in bits 0..3, `hi` in bits 4..7.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// One 16-byte vector (8 values, a quarter block) -> 4 bytes of codes; the
// block max is combined across the block's four lanes.  Every lane of the
// warp calls this (the shuffles need all of them); `valid` lanes store.
__device__ __forceinline__ void quant_vec(const QuantParams &p, long long i, bool valid, uint4 w, int lane)
{
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(u[k] << 16);
        v[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k)
        amax = fmaxf(amax, fabsf(v[k]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    if (!valid)
        return;
    // floor(log2(amax)) from the exponent field (a subnormal or zero max gives
    // the clamp -127 below).
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
    int s = e - 2;
    s = s < -127 ? -127 : (s > 127 ? 127 : s);
    const float inv = __uint_as_float((uint32_t)(127 - s) << 23);     // 2^-s, exact
    uint32_t packed = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        packed |= e2m1x2(v[2 * k] * inv, v[2 * k + 1] * inv) << (8 * k);
    p.q[i] = packed;
    if ((lane & 3) == 0)
        p.scales[i >> 2] = (uint8_t)(s + 127);
}

__global__ void __launch_bounds__(kThreads) mxfp4_quant_kernel(const QuantParams p)
{
    // Warp-uniform loop over groups of 32 vectors (8 blocks), kUnroll groups per
    // iteration with all their loads issued first (four 16-byte loads in flight
    // per thread measured 2-3 % faster than two; eight, slower); lanes past the
    // end skip their loads and stores.  A block's four lanes are valid or
    // invalid together (n_vec % 4 == 0).
    constexpr int kUnroll = 4;
    const int lane = threadIdx.x & 31;
    const long long n_groups = (p.n_vec + 31) >> 5;
    const long long warp0 = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const long long n_warps = ((long long)gridDim.x * kThreads) >> 5;
    for (long long g = warp0; g < n_groups; g += kUnroll * n_warps) {
        long long idx[kUnroll];
        bool valid[kUnroll];
        uint4 w[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            idx[u] = ((g + u * n_warps) << 5) + lane;
            valid[u] = idx[u] < p.n_vec;
            w[u] = make_uint4(0u, 0u, 0u, 0u);
            if (valid[u])
                w[u] = ld_stream(p.x + idx[u]);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            quant_vec(p, idx[u], valid[u], w[u], lane);
    }
}

// Resident blocks per device (occupancy x SM count), looked up once per device.
constexpr int kMaxDevices = 64;
std::atomic<int> g_resident[kMaxDevices];

bool aligned(const void *q, uintptr_t a) { return (reinterpret_cast<uintptr_t>(q) & (a - 1)) == 0; }

} // namespace

extern "C" int dit_attn_mxfp4_quantize(const void *x, void *q, void *scales, long long rows, int K,
                                       cudaStream_t stream)
{
    if (rows < 0 || K < 32 || K % 32 != 0 || (rows > 0 && rows * (long long)K >= (1ll << 40)))
        return DIT_ATTN_ERR_SHAPE;
    if (rows == 0)
        return DIT_ATTN_OK;             // nothing to read or write: pointers unused
    if (x == nullptr || q == nullptr || scales == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16))
        return DIT_ATTN_ERR_ALIGN;
    int device = 0, major = 0, minor = 0;
    if (cudaGetDevice(&device) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess ||
        major != 10 || minor != 0)
        return DIT_ATTN_ERR_ARCH;
    if (device >= kMaxDevices)
        return DIT_ATTN_ERR_ARCH;
    if (!dit_abi::device_buffers(device, {x, q, scales}))
        return DIT_ATTN_ERR_DEVICE;
    int resident = g_resident[device].load(std::memory_order_relaxed);
    if (resident == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mxfp4_quant_kernel, kThreads, 0) !=
                cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        resident = (per_sm > 0 ? per_sm : 1) * sms;
        g_resident[device].store(resident, std::memory_order_relaxed);
    }
    QuantParams p{};
    p.x = static_cast<const uint4 *>(x);
    p.q = static_cast<uint32_t *>(q);
    p.scales = static_cast<uint8_t *>(scales);
    p.n_vec = rows * (long long)(K / 8);
    const long long want = (p.n_vec + 2 * kThreads - 1) / (2 * kThreads);   // two vectors per thread
    const int grid = (int)(want < resident ? want : resident);
    mxfp4_quant_kernel<<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}
