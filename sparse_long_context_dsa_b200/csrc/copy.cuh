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
        // up to four 16-byte loads of a thread in flight before its stores: from pinned host
        // memory every dependent load would cost a bus round trip of its own
        const size_t n16 = bytes / 16;
        const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
        for (size_t i0 = tid; i0 < n16; i0 += 4 * nt) {
            uint4 r[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + u * nt < n16) r[u] = s4[i0 + u * nt];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (i0 + u * nt < n16) d4[i0 + u * nt] = r[u];
        }
        done = n16 * 16;
    }
    for (size_t i = done + tid; i < bytes; i += nt) dst[i] = src[i];
}

// New tokens' K and V rows written into their page slots: token i (request q_req[i], or i
// when q_req is null, position q_pos[i]) goes to page block_table[b][pos / 64], row pos % 64,
// all 4 groups.  With a block table that maps a request's pages cyclically onto a few physical
// pages this is the window layers' ring buffer: a token overwrites the one `ring` tokens
// before it ([P2] Step-5-Preview 如何实现1M长上下文 §第一招: the write goes to a fixed set of
// slots by a modulo of the position).  One CTA per token; threads 0..95 copy K, 128..223 V.
__global__ void __launch_bounds__(256) kv_append_kernel(__nv_bfloat16 *__restrict__ k_cache,
                                                        __nv_bfloat16 *__restrict__ v_cache, int64_t n_pages,
                                                        const int32_t *__restrict__ block_table, int max_pages,
                                                        const int32_t *__restrict__ q_req, int n_req,
                                                        const int32_t *__restrict__ q_pos, int n,
                                                        const __nv_bfloat16 *__restrict__ new_k,
                                                        const __nv_bfloat16 *__restrict__ new_v)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    const int i = blockIdx.x;
    if (i >= n) return;
    const int b = q_req ? q_req[i] : i;
    const int pos = q_pos[i];
    if (b < 0 || b >= n_req || pos < 0 || pos / kPage >= max_pages) {
        if (threadIdx.x == 0) set_error(kErrAttnIndex);
        return;
    }
    const int64_t page = block_table[(int64_t)b * max_pages + pos / kPage];
    if (page < 0 || page >= n_pages) {
        if (threadIdx.x == 0) set_error(kErrAttnIndex);
        return;
    }
    constexpr int kChunks = kD / 8;                          // 16-byte chunks of a 192-wide row
    const int t = threadIdx.x & 127, which = threadIdx.x >> 7;
    if (t < kG * kChunks) {
        const int g = t / kChunks, c = t % kChunks;
        const __nv_bfloat16 *src = (which ? new_v : new_k) + ((int64_t)i * kG + g) * kD + c * 8;
        __nv_bfloat16 *dst = (which ? v_cache : k_cache) + ((page * kG + g) * kPage + pos % kPage) * kD + c * 8;
        *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
    }
}

}  // namespace dsa
