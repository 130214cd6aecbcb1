// C ABI of the fused Ulysses attention (attn_fwd_ulysses_sm100.cuh): argument
// validation, one tensor map per shard and tensor, launch.  See
// include/dit_attn.h for the contract.
//
// This translation unit compiles the attention kernel's headers a second time
// (dit_attn.cu holds the first).  The headers' two non-template definitions,
// the device error word and the wait self-test kernel, take other names here so
// that both units link into one library; this unit's error word is read by
// dit_attn_ulysses_check_device_error.
#define g_error_word g_error_word_ulysses
#define selftest_wait_kernel selftest_wait_kernel_ulysses

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "abi_util.h"
#include "dit_attn.h"
#include "attn_fwd_ulysses_sm100.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 4000000000ull;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
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

// 3-D map over one shard [BH, Ls, D]: dims (D, Ls, BH), box (box_x, 64, 1).
bool shard_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elt, int D, int Ls, long long BH,
               int box_x, CUtensorMapSwizzle swz)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Ls, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * elt, (cuuint64_t)Ls * D * elt};
    const cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)dit::kHalfRows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for(int bytes)
{
    return bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : (bytes >= 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_attr_set[4][kMaxDevices];

template <int D, bool FP8>
int launch(const void *const *q, const void *const *k, const void *const *v, void *const *o,
           const dit::FwdParams &prm, const dit::UlyssesParams &u, long long B, int device, cudaStream_t stream)
{
    using C = dit::PCfg<D, FP8>;
    constexpr int variant = (D == 128 ? 1 : 0) + (FP8 ? 2 : 0);
    auto kern = dit::attn_fwd_ulysses_kernel<D, FP8>;
    if (device >= kMaxDevices || g_attr_set[variant][device].load(std::memory_order_acquire) == 0) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        // The 8 softmax warps' and 4 other warps' setmaxnreg shares must fit in what
        // the CTA is launched with (8-register granules), or the increase never returns.
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
            8 * C::REGS_SOFTMAX + 4 * C::REGS_OTHER > 12 * ((fa.numRegs + 7) & ~7))
            return DIT_ATTN_ERR_LAUNCH;
        if (device < kMaxDevices)
            g_attr_set[variant][device].store(1, std::memory_order_release);
    }
    const CUtensorMapDataType in_t = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const long long BH = B * u.H;
    dit::UlyssesMaps maps;
    for (int c = 0; c < u.n_ranks; ++c) {
        if (!shard_map(&maps.q[c], q[c], in_t, C::ELT, D, u.Ls, BH, C::BOX_ELEMS, swizzle_for(C::SWZ)) ||
            !shard_map(&maps.k[c], k[c], in_t, C::ELT, D, u.Ls, BH, C::BOX_ELEMS, swizzle_for(C::SWZ)) ||
            !shard_map(&maps.v[c], v[c], in_t, C::ELT, D, u.Ls, BH, D / 2, swizzle_for(C::VRAW_ROW)) ||
            !shard_map(&maps.o[c], o[c], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, u.Ls, BH, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return DIT_ATTN_ERR_LAUNCH;
    }
    for (int c = u.n_ranks; c < dit::kMaxUlyssesRanks; ++c)
        maps.q[c] = maps.k[c] = maps.v[c] = maps.o[c] = maps.q[0];   // never addressed
    const long long blocks = 2 * B * u.Hn * (long long)prm.n_pairs;
    if (blocks > 0x7FFFFFFFll)
        return DIT_ATTN_ERR_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, maps, prm, u) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

} // namespace

extern "C" {

int dit_attn_fwd_ulysses(const void *const *q_shards, const void *const *k_shards, const void *const *v_shards,
                         void *const *o_shards, float *const *lse_shards, int n_ranks, int rank, int B, int H,
                         int Ls, int D, float scale, int dtype, const float *q_scale, const float *k_scale,
                         const float *v_scale, cudaStream_t stream)
{
    if (!q_shards || !k_shards || !v_shards || !o_shards)
        return DIT_ATTN_ERR_NULL;
    if (n_ranks < 1 || n_ranks > dit::kMaxUlyssesRanks || rank < 0 || rank >= n_ranks)
        return DIT_ATTN_ERR_SHAPE;
    if (dtype != DIT_ATTN_BF16 && dtype != DIT_ATTN_FP8_E4M3)
        return DIT_ATTN_ERR_DTYPE;
    const bool fp8 = dtype == DIT_ATTN_FP8_E4M3;
    if (fp8 && (!q_scale || !k_scale || !v_scale))
        return DIT_ATTN_ERR_NULL;
    if (!fp8 && (q_scale || k_scale || v_scale))
        return DIT_ATTN_ERR_DTYPE;
    if (B < 1 || H < 1 || Ls < 1 || (D != 64 && D != 128) || H % n_ranks != 0 || Ls % dit::kHalfRows != 0)
        return DIT_ATTN_ERR_SHAPE;
    const long long L = (long long)n_ranks * Ls;
    if (L > 0x7FFFFFFFll || (long long)B * H * L * D >= (1ll << 40) || (long long)B * H > 0x7FFFFFFFll)
        return DIT_ATTN_ERR_SHAPE;
    const bool with_lse = lse_shards != nullptr && lse_shards[0] != nullptr;
    for (int c = 0; c < n_ranks; ++c) {
        if (!q_shards[c] || !k_shards[c] || !v_shards[c] || !o_shards[c] || (with_lse && !lse_shards[c]) ||
            (!with_lse && lse_shards != nullptr && lse_shards[c] != nullptr))
            return DIT_ATTN_ERR_NULL;
        if (!aligned(q_shards[c], 16) || !aligned(k_shards[c], 16) || !aligned(v_shards[c], 16) ||
            !aligned(o_shards[c], 16) || (with_lse && !aligned(lse_shards[c], 4)))
            return DIT_ATTN_ERR_ALIGN;
    }
    if (fp8 && (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4)))
        return DIT_ATTN_ERR_ALIGN;
    if (!std::isfinite(scale) || scale < 0.f)
        return DIT_ATTN_ERR_VALUE;
    int device = 0, major = 0, minor = 0;
    if (cudaGetDevice(&device) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess ||
        major != 10 || minor != 0)
        return DIT_ATTN_ERR_ARCH;
    // Shards may be peers' memory mapped into this context; the scales are
    // read by this device only.
    for (int c = 0; c < n_ranks; ++c)
        if (!dit_abi::device_buffers(device, {q_shards[c], k_shards[c], v_shards[c], o_shards[c],
                                              with_lse ? lse_shards[c] : nullptr},
                                     /*peers_ok=*/true))
            return DIT_ATTN_ERR_DEVICE;
    if (!dit_abi::device_buffers(device, {q_scale, k_scale, v_scale}))
        return DIT_ATTN_ERR_DEVICE;

    dit::FwdParams prm{};
    prm.L = (int)L;
    prm.n_kv = (int)((L + dit::kBN - 1) / dit::kBN);
    prm.n_pairs = (int)(((L + dit::kBM - 1) / dit::kBM + 1) / 2);
    prm.kv_tail = (int)(L - (long long)(prm.n_kv - 1) * dit::kBN);
    prm.scale = scale;
    prm.q_scale = q_scale;
    prm.k_scale = k_scale;
    prm.v_scale = v_scale;
    prm.lse = nullptr;                                 // the LSE goes through the shard pointers
    prm.wait_limit_ns = kWaitLimitNs;
    dit::UlyssesParams u{};
    u.n_ranks = n_ranks;
    u.Ls = Ls;
    u.H = H;
    u.Hn = H / n_ranks;
    u.head0 = rank * u.Hn;
    for (int c = 0; c < dit::kMaxUlyssesRanks; ++c)
        u.lse[c] = (with_lse && c < n_ranks) ? lse_shards[c] : nullptr;

    if (!fp8 && D == 128)
        return launch<128, false>(q_shards, k_shards, v_shards, o_shards, prm, u, B, device, stream);
    if (!fp8 && D == 64)
        return launch<64, false>(q_shards, k_shards, v_shards, o_shards, prm, u, B, device, stream);
    if (fp8 && D == 128)
        return launch<128, true>(q_shards, k_shards, v_shards, o_shards, prm, u, B, device, stream);
    return launch<64, true>(q_shards, k_shards, v_shards, o_shards, prm, u, B, device, stream);
}

int dit_attn_ulysses_check_device_error(cudaStream_t stream, uint32_t *detail)
{
    unsigned int word = 0;
    if (cudaMemcpyFromSymbolAsync(&word, dit::g_error_word, sizeof word, 0, cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    if (detail)
        *detail = word;
    if (word == 0)
        return DIT_ATTN_OK;
    static const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(dit::g_error_word, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return DIT_ATTN_ERR_TIMEOUT;
}

} // extern "C"
