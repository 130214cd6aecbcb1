// Host-side argument checks shared by the C-ABI entry points.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>
#include <initializer_list>

namespace dit_abi {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// True when every non-NULL pointer is device memory that the current device's
// kernels may read and write: memory of `device` itself or managed memory,
// and, with peers_ok, another GPU's memory mapped into this context.  Host
// memory, pointers no CUDA allocation covers, and (without peers_ok) another
// GPU's memory are refused: a kernel given them would fault or reach across
// the link.
inline bool device_buffers(int device, std::initializer_list<const void *> ptrs, bool peers_ok = false)
{
    for (const void *p : ptrs) {
        if (p == nullptr)
            continue;
        cudaPointerAttributes a{};
        if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
            (void)cudaGetLastError();   // not sticky: clear it for the caller
            return false;
        }
        if (a.type == cudaMemoryTypeManaged)
            continue;
        if (a.type != cudaMemoryTypeDevice || (!peers_ok && a.device != device))
            return false;
    }
    return true;
}

} // namespace dit_abi
