// C ABI of the DiT joint-attention forward: argument validation, TMA tensor
// maps, launch.  See include/dit_attn.h for the contract of each entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "abi_util.h"
#include "dit_attn.h"
#include "attn_fwd_sm100.cuh"

namespace {

constexpr unsigned long long kDefaultWaitLimitNs = 4000000000ull;
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D map over a contiguous [BH, L, D] tensor: dims (D, L, BH), box (box_x, box_rows, 1).
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elt, int D, int L,
              long long BH, int box_x, CUtensorMapSwizzle swz, int box_rows = dit::kBM)
{
    auto enc = tensor_map_encoder();
    if (!enc)
        return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)D * elt, (cuuint64_t)L * D * elt};
    const cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swizzle_for(int bytes)
{
    return bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : (bytes >= 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// Per-device "max dynamic smem attribute set" flags, one per kernel instantiation.
constexpr int kMaxDevices = 64;
std::atomic<int> g_attr_set[4][kMaxDevices];

// The four tensor maps of a call depend only on (device, q, k, v, o, B*H, L,
// variant): a small cache lets a repeated call (every layer and denoising step
// of a DiT) skip the four cuTensorMapEncodeTiled calls.  A map holds nothing
// but the address, shape and strides, so an entry stays valid for any buffer
// at the same address with the same shape.
struct MapKey {
    int device, variant, L;
    long long BH;
    const void *q, *k, *v, *o;
    bool operator==(const MapKey &b) const
    {
        return device == b.device && variant == b.variant && L == b.L && BH == b.BH && q == b.q && k == b.k &&
               v == b.v && o == b.o;
    }
};
struct MapEntry {
    MapKey key;
    CUtensorMap tq, tk, tv, to;
    unsigned long long used;
    bool valid;
};
constexpr int kMapCache = 16;
std::mutex g_map_mu;
MapEntry g_maps[kMapCache];
unsigned long long g_map_clock = 0;

// Clusters of 2 CTAs, one 128-row query tile per CTA.
template <int D, bool FP8>
int launch(const void *q, const void *k, const void *v, void *o, const dit::FwdParams &prm,
                long long BH, int L, int device, cudaStream_t stream)
{
    using C = dit::PCfg<D, FP8>;
    constexpr int variant = (D == 128 ? 1 : 0) + (FP8 ? 2 : 0);
    auto kern = dit::attn_fwd_kernel<D, FP8>;
    if (device >= kMaxDevices || g_attr_set[variant][device].load(std::memory_order_acquire) == 0) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
            cudaSuccess)
            return DIT_ATTN_ERR_LAUNCH;
        if (device < kMaxDevices)
            g_attr_set[variant][device].store(1, std::memory_order_release);
    }
    const MapKey key{device, variant, L, BH, q, k, v, o};
    CUtensorMap tq, tk, tv, to;
    bool hit = false;
    {
        std::lock_guard<std::mutex> lock(g_map_mu);
        for (MapEntry &e : g_maps)
            if (e.valid && e.key == key) {
                tq = e.tq, tk = e.tk, tv = e.tv, to = e.to;
                e.used = ++g_map_clock;
                hit = true;
                break;
            }
    }
    if (!hit) {
        const CUtensorMapDataType in_t = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        if (!make_map(&tq, q, in_t, C::ELT, D, L, BH, C::BOX_ELEMS, swizzle_for(C::SWZ), dit::kBM) ||
            !make_map(&tk, k, in_t, C::ELT, D, L, BH, C::BOX_ELEMS, swizzle_for(C::SWZ), C::KROWS) ||
            !make_map(&tv, v, in_t, C::ELT, D, L, BH, D / 2, swizzle_for(C::VRAW_ROW), dit::kBN) ||
            !make_map(&to, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, L, BH, 64, CU_TENSOR_MAP_SWIZZLE_128B,
                      dit::kBM))
            return DIT_ATTN_ERR_LAUNCH;
        std::lock_guard<std::mutex> lock(g_map_mu);
        MapEntry *slot = &g_maps[0];
        for (MapEntry &e : g_maps)
            if (!e.valid || e.used < slot->used) {
                slot = &e;
                if (!e.valid)
                    break;
            }
        *slot = MapEntry{key, tq, tk, tv, to, ++g_map_clock, true};
    }
    const long long blocks = 2 * BH * (long long)prm.n_pairs;
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
    if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, prm) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_device(int *device)
{
    if (cudaGetDevice(device) != cudaSuccess)
        return DIT_ATTN_ERR_ARCH;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *device) != cudaSuccess)
        return DIT_ATTN_ERR_ARCH;
    return (major == 10 && minor == 0) ? DIT_ATTN_OK : DIT_ATTN_ERR_ARCH;
}

} // namespace

extern "C" {

int dit_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                 int L, int D, float scale, int dtype, const float *q_scale, const float *k_scale,
                 const float *v_scale, cudaStream_t stream)
{
    if (!q || !k || !v || !o)
        return DIT_ATTN_ERR_NULL;
    if (dtype != DIT_ATTN_BF16 && dtype != DIT_ATTN_FP8_E4M3)
        return DIT_ATTN_ERR_DTYPE;
    const bool fp8 = dtype == DIT_ATTN_FP8_E4M3;
    if (fp8 && (!q_scale || !k_scale || !v_scale))
        return DIT_ATTN_ERR_NULL;
    if (!fp8 && (q_scale || k_scale || v_scale))
        return DIT_ATTN_ERR_DTYPE;
    if (B < 1 || H < 1 || L < 1 || (D != 64 && D != 128))
        return DIT_ATTN_ERR_SHAPE;
    const long long BH = (long long)B * H;
    if (BH > 0x7FFFFFFFll || BH * (long long)L * D >= (1ll << 40))
        return DIT_ATTN_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        (lse && !aligned(lse, 4)) ||
        (fp8 && (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4))))
        return DIT_ATTN_ERR_ALIGN;
    if (!std::isfinite(scale) || scale < 0.f)
        return DIT_ATTN_ERR_VALUE;
    int device = 0;
    const int dev_rc = check_device(&device);
    if (dev_rc != DIT_ATTN_OK)
        return dev_rc;
    if (!dit_abi::device_buffers(device, {q, k, v, o, lse, q_scale, k_scale, v_scale}))
        return DIT_ATTN_ERR_DEVICE;

    dit::FwdParams prm{};
    prm.L = L;
    prm.n_kv = (L + dit::kBN - 1) / dit::kBN;
    prm.n_pairs = ((L + dit::kBM - 1) / dit::kBM + 1) / 2;
    prm.kv_tail = L - (prm.n_kv - 1) * dit::kBN;
    prm.scale = scale;
    prm.q_scale = q_scale;
    prm.k_scale = k_scale;
    prm.v_scale = v_scale;
    prm.lse = lse;
    prm.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);

    if (!fp8 && D == 128)
        return launch<128, false>(q, k, v, o, prm, BH, L, device, stream);
    if (!fp8 && D == 64)
        return launch<64, false>(q, k, v, o, prm, BH, L, device, stream);
    if (fp8 && D == 128)
        return launch<128, true>(q, k, v, o, prm, BH, L, device, stream);
    return launch<64, true>(q, k, v, o, prm, BH, L, device, stream);
}

const char *dit_attn_status_string(int status)
{
    switch (status) {
    case DIT_ATTN_OK: return "ok";
    case DIT_ATTN_ERR_NULL: return "a required pointer is NULL";
    case DIT_ATTN_ERR_SHAPE: return "unsupported shape (need B,H,L >= 1, D in {64,128}, B*H*L*D < 2^40)";
    case DIT_ATTN_ERR_DTYPE: return "unknown dtype, or scales passed for bf16";
    case DIT_ATTN_ERR_ALIGN: return "q/k/v/o must be 16-byte aligned, lse and scales 4-byte aligned";
    case DIT_ATTN_ERR_ARCH: return "no CUDA device, or the current device is not sm_100 (B200)";
    case DIT_ATTN_ERR_LAUNCH: return "a CUDA runtime call or the kernel launch failed";
    case DIT_ATTN_ERR_TIMEOUT: return "a device-side wait exceeded its time limit";
    case DIT_ATTN_ERR_VALUE: return "scale must be finite and >= 0";
    case DIT_ATTN_ERR_DEVICE:
        return "a buffer is not device memory of the current device (host memory, another GPU's, or unallocated)";
    default: return "unknown status";
    }
}

int dit_attn_check_device_error(cudaStream_t stream, uint32_t *detail)
{
    unsigned int word = 0;
    if (cudaMemcpyFromSymbolAsync(&word, dit::g_error_word, sizeof word, 0, cudaMemcpyDeviceToHost,
                                  stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    if (detail)
        *detail = word;
    if (word == 0)
        return DIT_ATTN_OK;
    static const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(dit::g_error_word, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DIT_ATTN_ERR_LAUNCH;
    return DIT_ATTN_ERR_TIMEOUT;
}

void dit_attn_set_wait_limit_ns(uint64_t ns)
{
    g_wait_limit_ns.store(ns ? (unsigned long long)ns : kDefaultWaitLimitNs, std::memory_order_relaxed);
}

int dit_attn_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream)
{
    int device = 0;
    const int dev_rc = check_device(&device);
    if (dev_rc != DIT_ATTN_OK)
        return dev_rc;
    dit::selftest_wait_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_ns);
    return cudaGetLastError() == cudaSuccess ? DIT_ATTN_OK : DIT_ATTN_ERR_LAUNCH;
}

int dit_attn_launches_per_call(int B, int H, int L, int D, int dtype)
{
    (void)B; (void)H; (void)L; (void)D; (void)dtype;
    return 1;
}

} // extern "C"
