// Byte copy by a kernel between any two addresses the GPU can reach (device memory, or pinned
// host memory through unified addressing).  A decode step's inputs (tens of KiB) staged from
// pinned host memory this way cost one PCIe round trip inside the kernel chain instead of a
// copy-engine operation between kernels.
#pragma once

#include "common.cuh"

namespace dsa {

__global__ void __launch_bounds__(256) copy_kernel(uint8_t *__restrict__ dst, const uint8_t *__restrict__ src,
                                                   size_t bytes)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x, nt = (size_t)gridDim.x * blockDim.x;
    const bool vec = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) == 0;
    size_t done = 0;
    if (vec) {
        const size_t n16 = bytes / 16;
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
        for (size_t i = tid; i < n16; i += nt) d4[i] = s4[i];
        done = n16 * 16;
    }
    for (size_t i = done + tid; i < bytes; i += nt) dst[i] = src[i];
}

}  // namespace dsa
