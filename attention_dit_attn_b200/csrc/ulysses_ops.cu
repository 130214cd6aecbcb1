// Local data movement of Ulysses sequence parallelism (page "How to Scale
// Diffusion Inference Across AMD RDNA 4 GPUs", section "Balance Transformer
// Work and Communication": attention's tokens are divided across GPUs and
// every attention layer exchanges data with an all-to-all; `--use fp8 comms`
// sends that exchange in FP8).
//
//  * dit_attn_block_transpose: out[c][r] = in[r][c] over contiguous blocks.
//    Every layout move of the exchange is one of these: heads grouped by
//    destination before the all-to-all, sequence chunks concatenated after it,
//    and the same two moves backwards for O.
//  * dit_attn_absmax_rows: max |x| of each row (one (b, h) of a shard).
//  * dit_attn_quantize_e4m3_rows: e4m3(x / s) per row with s = amax / 448 (1
//    for amax = 0), rounded to nearest even and saturated, plus the per-row
//    dequantisation scale s.  With the all-reduced (global) amax of each head,
//    every rank quantises its shard with the same per-head scale, so the
//    received FP8 tensors are exactly the inputs of the FP8 attention path.
//
// All three are memory-bound: 16-byte loads and stores, no waits.  A row is
// one head of a shard, so there are few rows (B H) of up to millions of
// values: every kernel splits each row over many CTAs (grid.x = chunks of a
// row, grid.y = rows), and the absmax CTAs combine their partial maxima with
// an atomic max on the (order-preserving) bit patterns of non-negative floats.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "abi_util.h"
#include "dit_attn.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;                               // units in flight per thread
constexpr long long kUnitsPerCta = (long long)kUnroll * kThreads;
constexpr float kE4M3Max = 448.f;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// One CTA row (blockIdx.y, grid-strided) per block pair (r, c); the CTAs of a
// row (blockIdx.x) split the block's 16-byte (or 4-byte) words.
template <class W>
__global__ void __launch_bounds__(kThreads) block_transpose_kernel(const W *in, W *out, long long R, long long C,
                                                                    long long words)
{
    for (long long blk = blockIdx.y; blk < R * C; blk += gridDim.y) {
        const long long r = blk / C, c = blk - r * C;
        const W *src = in + blk * words;
        W *dst = out + (c * R + r) * words;
        for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < words; i += (long long)gridDim.x * kThreads)
            dst[i] = src[i];
    }
}

// Per row: max |x| over row_len bf16 (row_len % 8 == 0).  CTA (x, y) covers
// vectors [x U, x U + U) (U = kUnitsPerCta, kUnroll per thread, all loads
// issued before use) of rows y, y + gridDim.y, ...; amax_bits holds 0 on
// entry and receives max(|bf16| bits) << 16, the float bits of the maximum.
__global__ void __launch_bounds__(kThreads) absmax_rows_kernel(const uint4 *x, unsigned int *amax_bits,
                                                               long long rows, long long vec_per_row)
{
    __shared__ uint32_t red[kThreads / 32];
    const long long beg = (long long)blockIdx.x * kUnitsPerCta + threadIdx.x;
    for (long long row = blockIdx.y; row < rows; row += gridDim.y) {
        const uint4 *src = x + row * vec_per_row;
        uint4 w[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const long long i = beg + (long long)k * kThreads;
            w[k] = i < vec_per_row ? ld_stream(src + i) : make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t m = 0;                                  // max of |bf16| bit patterns (order-preserving)
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const uint32_t u[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                m = max(m, u[e] & 0x7FFFu);
                m = max(m, (u[e] >> 16) & 0x7FFFu);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == 0)
            red[threadIdx.x >> 5] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t r = 0;
            for (int w = 0; w < kThreads / 32; ++w)
                r = max(r, red[w]);
            atomicMax(amax_bits + row, r << 16);
        }
        __syncthreads();
    }
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Per row: q = e4m3(x / s), s = amax / 448 (1 if amax == 0); 16 values per
// unit (two 16-byte loads, one 16-byte store).  CTA (x, y) covers units
// [x U, x U + U) (kUnroll per thread, all loads issued before use) of rows
// y, y + gridDim.y, ...; the CTAs with x = 0 write the row's scale.
__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const uint4 *x, uint4 *q, const float *amax,
                                                                 float *scale_out, long long rows,
                                                                 long long vec16_per_row)
{
    const long long beg = (long long)blockIdx.x * kUnitsPerCta + threadIdx.x;
    for (long long row = blockIdx.y; row < rows; row += gridDim.y) {
        const float a = amax[row];
        const float s = a > 0.f ? __fdiv_rn(a, kE4M3Max) : 1.f;
        if (blockIdx.x == 0 && threadIdx.x == 0 && scale_out != nullptr)
            scale_out[row] = s;
        const uint4 *src = x + row * vec16_per_row * 2;
        uint4 *dst = q + row * vec16_per_row;
        uint4 w[2 * kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const long long i = beg + (long long)k * kThreads;
            if (i < vec16_per_row) {
                w[2 * k] = ld_stream(src + 2 * i);
                w[2 * k + 1] = ld_stream(src + 2 * i + 1);
            }
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const long long i = beg + (long long)k * kThreads;
            if (i >= vec16_per_row)
                break;
            const uint4 w0 = w[2 * k], w1 = w[2 * k + 1];
            const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t out[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float v0 = __fdiv_rn(__uint_as_float(u[2 * e] << 16), s);
                const float v1 = __fdiv_rn(__uint_as_float(u[2 * e] & 0xFFFF0000u), s);
                const float v2 = __fdiv_rn(__uint_as_float(u[2 * e + 1] << 16), s);
                const float v3 = __fdiv_rn(__uint_as_float(u[2 * e + 1] & 0xFFFF0000u), s);
                out[e] = e4m3x2(v0, v1) | (e4m3x2(v2, v3) << 16);
            }
            dst[i] = make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The current device is a B200 and every buffer is its device memory.
int check_arch(std::initializer_list<const void *> buffers)
{
    int device = 0, major = 0, minor = 0;
    if (cudaGetDevice(&device) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess ||
        major != 10 || minor != 0)
        return DIT_ATTN_ERR_ARCH;
    return dit_abi::device_buffers(device, buffers) ? DIT_ATTN_OK : DIT_ATTN_ERR_DEVICE;
}

// Grid of a row-chunked kernel: chunks of `per_cta` units per row in x, rows
// in y (capped; the kernels stride over the remaining rows).
dim3 grid_rows(long long rows, long long units_per_row, long long per_cta)
{
    const long long chunks = (units_per_row + per_cta - 1) / per_cta;
    return dim3((unsigned)chunks, (unsigned)(rows < 65535 ? rows : 65535));
}

} // namespace

extern "C" int dit_attn_block_transpose(const void *in, void *out, long long R, long long C, long long block_bytes,
                                        cudaStream_t stream)
{
    if (R < 0 || C < 0 || block_bytes < 0 || block_bytes % 4 != 0 ||
        (R > 0 && C > 0 && block_bytes > 0 && R * C > (1ll << 40) / block_bytes))
        return DIT_ATTN_ERR_SHAPE;
    if (R == 0 || C == 0 || block_bytes == 0)
        return DIT_ATTN_OK;
    if (in == nullptr || out == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!aligned(in, 4) || !aligned(out, 4))
        return DIT_ATTN_ERR_ALIGN;
    const int rc = check_arch({in, out});
    if (rc != DIT_ATTN_OK)
        return rc;
    const bool wide = block_bytes % 16 == 0 && aligned(in, 16) && aligned(out, 16);
    const long long words = block_bytes / (wide ? 16 : 4);
    const long long blocks = R * C;
    const long long per_block_ctas = (words + kThreads * 4 - 1) / (kThreads * 4);
    dim3 grid((unsigned)(per_block_ctas < 1184 ? per_block_ctas : 1184),
              (unsigned)(blocks < 65535 ? blocks : 65535));
    if (wide)
        block_transpose_kernel<uint4><<<grid, kThreads, 0, stream>>>(static_cast<const uint4 *>(in),
                                                                     static_cast<uint4 *>(out), R, C, words);
    else
        block_transpose_kernel<uint32_t><<<grid, kThreads, 0, stream>>>(static_cast<const uint32_t *>(in),
                                                                        static_cast<uint32_t *>(out), R, C, words);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

extern "C" int dit_attn_absmax_rows(const void *x, float *amax, long long rows, long long row_len, cudaStream_t stream)
{
    if (rows < 0 || row_len < 8 || row_len % 8 != 0 || (rows > 0 && rows * row_len >= (1ll << 40)))
        return DIT_ATTN_ERR_SHAPE;
    if (rows == 0)
        return DIT_ATTN_OK;
    if (x == nullptr || amax == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!aligned(x, 16) || !aligned(amax, 4))
        return DIT_ATTN_ERR_ALIGN;
    const int rc = check_arch({x, amax});
    if (rc != DIT_ATTN_OK)
        return rc;
    if (cudaMemsetAsync(amax, 0, (size_t)rows * sizeof(float), stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    absmax_rows_kernel<<<grid_rows(rows, row_len / 8, kUnitsPerCta), kThreads, 0, stream>>>(
        static_cast<const uint4 *>(x), reinterpret_cast<unsigned int *>(amax), rows, row_len / 8);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

extern "C" int dit_attn_quantize_e4m3_rows(const void *x, const float *amax, void *q, float *scale_out, long long rows,
                                           long long row_len, cudaStream_t stream)
{
    if (rows < 0 || row_len < 16 || row_len % 16 != 0 || (rows > 0 && rows * row_len >= (1ll << 40)))
        return DIT_ATTN_ERR_SHAPE;
    if (rows == 0)
        return DIT_ATTN_OK;
    if (x == nullptr || amax == nullptr || q == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(amax, 4) || (scale_out != nullptr && !aligned(scale_out, 4)))
        return DIT_ATTN_ERR_ALIGN;
    const int rc = check_arch({x, amax, q, scale_out});
    if (rc != DIT_ATTN_OK)
        return rc;
    quantize_rows_kernel<<<grid_rows(rows, row_len / 16, kUnitsPerCta), kThreads, 0, stream>>>(
        static_cast<const uint4 *>(x), static_cast<uint4 *>(q), amax, scale_out, rows, row_len / 16);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}
