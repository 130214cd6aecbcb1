// C ABI of the low-precision linear-layer GEMMs (Y = A W^T, bf16 out):
// argument validation, TMA tensor maps, persistent launch on CTA pairs.
// Kernel and sources: gemm_sm100.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "abi_util.h"
#include "dit_attn.h"
#include "gemm_sm100.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 4000000000ull;
constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_attr_set[kMaxDevices];
std::atomic<int> g_attr_set_f4[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D map over a row-major [rows, row_bytes] byte matrix (or bf16 with elt 2):
// dims (cols, rows), box (box_cols, box_rows), 128-byte swizzle unless told otherwise.
bool make_map_2d(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, long long cols, long long rows,
                 long long row_bytes, int box_cols, int box_rows,
                 CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B)
{
    auto enc = encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_device(int *device)
{
    int major = 0, minor = 0;
    if (cudaGetDevice(device) != cudaSuccess || *device < 0 || *device >= kMaxDevices ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *device) != cudaSuccess ||
        major != 10 || minor != 0)
        return DIT_ATTN_ERR_ARCH;
    return DIT_ATTN_OK;
}

template <class Kind>
int launch(const CUtensorMap &ta, const CUtensorMap &tw, const CUtensorMap &ty, const dit_gemm::GemmParams &p,
           int device, cudaStream_t stream)
{
    auto kern = dit_gemm::gemm_kernel<Kind>;
    if (g_attr_set[device].load(std::memory_order_acquire) == 0) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dit_gemm::Smem::BYTES) !=
            cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        g_attr_set[device].store(1, std::memory_order_release);
    }
    int sms = g_sms[device].load(std::memory_order_relaxed);
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        g_sms[device].store(sms, std::memory_order_relaxed);
    }
    // One cluster (CTA pair) per two SMs, never more clusters than tiles.
    const long long tiles = (long long)p.m_tiles * p.n_tiles;
    const long long clusters = tiles < sms / 2 ? tiles : sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(dit_gemm::kThreads);
    cfg.dynamicSmemBytes = dit_gemm::Smem::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tw, ty, p) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

} // namespace

extern "C" {

int dit_attn_gemm_fp8(const void *a, const void *w, void *y, long long M, int N, int K, float a_scale,
                      float w_scale, cudaStream_t stream)
{
    if (M < 0 || N < 1 || K < 16 || K % 16 != 0 || N % 8 != 0 || M > 0x7FFFFFFFll)
        return DIT_ATTN_ERR_SHAPE;
    if (M == 0)
        return DIT_ATTN_OK;
    if (a == nullptr || w == nullptr || y == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!dit_abi::aligned(a, 16) || !dit_abi::aligned(w, 16) || !dit_abi::aligned(y, 16))
        return DIT_ATTN_ERR_ALIGN;
    if (!std::isfinite(a_scale) || !std::isfinite(w_scale))
        return DIT_ATTN_ERR_VALUE;
    int device = 0;
    const int rc = check_device(&device);
    if (rc != DIT_ATTN_OK)
        return rc;
    if (!dit_abi::device_buffers(device, {a, w, y}))
        return DIT_ATTN_ERR_DEVICE;
    CUtensorMap ta, tw, ty;
    if (!make_map_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, dit_gemm::kBKB, dit_gemm::kBM) ||
        !make_map_2d(&tw, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, dit_gemm::kBKB, dit_gemm::kBNh) ||
        !make_map_2d(&ty, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, 2ll * N, dit_gemm::kOBox, dit_gemm::kBM))
        return DIT_ATTN_ERR_LAUNCH;
    dit_gemm::GemmParams p{};
    p.M = (int)M;
    p.N = N;
    p.K = K;
    p.kb = (K + dit_gemm::kBKB - 1) / dit_gemm::kBKB;
    p.m_tiles = (int)((M + 2 * dit_gemm::kBM - 1) / (2 * dit_gemm::kBM));
    p.n_tiles = (N + dit_gemm::kBN - 1) / dit_gemm::kBN;
    p.out_scale = a_scale * w_scale;
    p.wait_limit_ns = kWaitLimitNs;
    return launch<dit_gemm::Fp8Kind>(ta, tw, ty, p, device, stream);
}

long long dit_attn_mxfp4_tiled_scale_bytes(long long rows, int K)
{
    if (rows < 1 || K < 32 || K % 32 != 0)
        return 0;
    const long long row_blocks = (rows + 127) / 128;
    const long long groups = 2 * ((K + 255) / 256);
    return row_blocks * groups * 512;
}

int dit_attn_mxfp4_tile_scales(const void *plain, void *tiled, long long rows, int K, cudaStream_t stream)
{
    if (rows < 0 || K < 32 || K % 32 != 0 || rows > 0x7FFFFFFFll)
        return DIT_ATTN_ERR_SHAPE;
    if (rows == 0)
        return DIT_ATTN_OK;
    if (plain == nullptr || tiled == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!dit_abi::aligned(tiled, 16))
        return DIT_ATTN_ERR_ALIGN;
    int device = 0;
    const int rc = check_device(&device);
    if (rc != DIT_ATTN_OK)
        return rc;
    if (!dit_abi::device_buffers(device, {plain, tiled}))
        return DIT_ATTN_ERR_DEVICE;
    const long long chunks = dit_attn_mxfp4_tiled_scale_bytes(rows, K) / 16;
    const int groups = 2 * ((K + 255) / 256);
    const long long blocks = (chunks + 255) / 256;
    dit_gemm::tile_scales_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(
        static_cast<const uint8_t *>(plain), static_cast<uint32_t *>(tiled), (int)rows, K / 32, groups, chunks);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

int dit_attn_gemm_mxfp4(const void *a, const void *a_scales, const void *w, const void *w_scales, void *y,
                        long long M, int N, int K, cudaStream_t stream)
{
    if (M < 0 || N < 8 || N % 8 != 0 || K < 32 || K % 32 != 0 || M > 0x7FFFFFFFll)
        return DIT_ATTN_ERR_SHAPE;
    if (M == 0)
        return DIT_ATTN_OK;
    if (a == nullptr || w == nullptr || y == nullptr || a_scales == nullptr || w_scales == nullptr)
        return DIT_ATTN_ERR_NULL;
    if (!dit_abi::aligned(a, 16) || !dit_abi::aligned(w, 16) || !dit_abi::aligned(y, 16) ||
        !dit_abi::aligned(a_scales, 16) || !dit_abi::aligned(w_scales, 16))
        return DIT_ATTN_ERR_ALIGN;
    int device = 0;
    const int rc = check_device(&device);
    if (rc != DIT_ATTN_OK)
        return rc;
    if (!dit_abi::device_buffers(device, {a, w, y, a_scales, w_scales}))
        return DIT_ATTN_ERR_DEVICE;
    if (g_attr_set_f4[device].load(std::memory_order_acquire) == 0) {
        if (cudaFuncSetAttribute(dit_gemm::gemm_mxf4_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dit_gemm::P4Smem::BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(dit_gemm::gemm_mxf4_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 dit_gemm::P4Smem::BYTES) != cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        g_attr_set_f4[device].store(1, std::memory_order_release);
    }
    int sms = g_sms[device].load(std::memory_order_relaxed);
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        g_sms[device].store(sms, std::memory_order_relaxed);
    }
    dit_gemm::F4Params p{};
    p.M = (int)M;
    p.N = N;
    p.K = K;
    p.groups = 2 * ((K + 255) / 256);
    p.kb = p.groups / 2;
    p.m_tiles = (int)((M + 2 * dit_gemm::kF4BM - 1) / (2 * dit_gemm::kF4BM));
    p.n_tiles = (N + dit_gemm::kF4BN - 1) / dit_gemm::kF4BN;
    p.w_row_blocks = (N + 127) / 128;
    p.sfa = static_cast<const uint8_t *>(a_scales);
    p.sfw = static_cast<const uint8_t *>(w_scales);
    p.wait_limit_ns = kWaitLimitNs;
    // Scale atoms as 256-byte rows: two rows per 512-byte atom.
    const long long sa_rows = dit_attn_mxfp4_tiled_scale_bytes(M, K) / 256;
    const long long sw_rows = dit_attn_mxfp4_tiled_scale_bytes(N, K) / 256;
    CUtensorMap ta, tw, ty, tsa, tsw;
    if (!make_map_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, M, K / 2, dit_gemm::kBKB, dit_gemm::kF4BM) ||
        !make_map_2d(&tw, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, dit_gemm::kBKB, dit_gemm::kF4BN / 2) ||
        !make_map_2d(&ty, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, 2ll * N, dit_gemm::kOBox, dit_gemm::kF4BM) ||
        !make_map_2d(&tsa, a_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, sa_rows, 256, 256, 4,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&tsw, w_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, sw_rows, 256, 256, 4,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return DIT_ATTN_ERR_LAUNCH;
    const long long tiles = (long long)p.m_tiles * p.n_tiles;
    const long long clusters = tiles < sms / 2 ? tiles : sms / 2;
    // W scales resident in TMEM when every pair keeps one N tile and K fits.  That
    // walk has the pairs of different N tiles reach a block of A at different
    // times, which only costs nothing while all of A stays in L2 (126 MB): at most
    // 64 MB of A codes.
    const bool resident = p.n_tiles <= clusters && p.kb <= dit_gemm::kF4ResMaxStages &&
                          M * (long long)(K / 2) <= (64ll << 20);
    auto kern = resident ? dit_gemm::gemm_mxf4_pair_kernel<true> : dit_gemm::gemm_mxf4_pair_kernel<false>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(dit_gemm::kThreads);
    cfg.dynamicSmemBytes = dit_gemm::P4Smem::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tw, ty, tsa, tsw, p) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

int dit_attn_gemm_check_device_error(cudaStream_t stream, uint32_t *detail)
{
    unsigned int word = 0;
    if (cudaMemcpyFromSymbolAsync(&word, dit_gemm::g_gemm_error_word, sizeof word, 0, cudaMemcpyDeviceToHost,
                                  stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    if (detail)
        *detail = word;
    if (word == 0)
        return DIT_ATTN_OK;
    static const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(dit_gemm::g_gemm_error_word, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return DIT_ATTN_ERR_TIMEOUT;
}

} // extern "C"
