// A1 region compression: every complete 8-token region of index_k becomes one 256-d e4m3
// summary per KV group with one fp32 scale ([P1] kwkr.cn/news/601179 §DSA ②;
// [P2] Step-5-Preview 如何实现1M长上下文 §区域压缩CSA: only full regions are summarised).
//
// One warp per (region, group): lane l owns dimensions 8l..8l+7 and reads them for the
// 8 tokens with 16-byte loads (a region-group is 4 KiB of contiguous bf16 rows).  The
// arithmetic is fixed bit for bit:
//   m_j   = fp32( (sum_{t=0..7} k_tj) * 0.125 ), the sum in fp64 in token order,
//   scale = fp32( max_j |m_j| / 448 )  (IEEE division),
//   code  = cvt.rn.satfinite.e4m3( fp32(m_j / scale) ),  all 0 if scale == 0.
// HBM-bound and negligible next to the scan (4 KiB read, 260 B written per region-group).
#pragma once

#include "common.cuh"

namespace dsa {

__global__ void __launch_bounds__(128) compress_regions_kernel(
    const __nv_bfloat16 *__restrict__ index_k, int64_t row_stride, int64_t n_rows,
    const int64_t *__restrict__ src_row, const int64_t *__restrict__ dst_slot, int n_regions,
    uint8_t *__restrict__ summaries, float *__restrict__ scales, int64_t n_slots)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = blockIdx.x; i < n_regions; i += gridDim.x) {
        const int64_t r0 = src_row[i], slot = dst_slot[i];
        if (r0 < 0 || r0 + kRegion > n_rows || slot < 0 || slot >= n_slots) {
            if (threadIdx.x == 0) set_error(kErrCompressIndex);
            continue;
        }
        double s[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = 0.0;
        const __nv_bfloat16 *base = index_k + r0 * row_stride + g * kDI + lane * 8;
        uint4 v[kRegion];
#pragma unroll
        for (int t = 0; t < kRegion; ++t)
            v[t] = __ldg(reinterpret_cast<const uint4 *>(base + (int64_t)t * row_stride));
#pragma unroll
        for (int t = 0; t < kRegion; ++t) {
            const uint32_t w[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s[2 * j] = __dadd_rn(s[2 * j], (double)bf16_lo(w[j]));
                s[2 * j + 1] = __dadd_rn(s[2 * j + 1], (double)bf16_hi(w[j]));
            }
        }
        float m[8];
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            m[j] = __double2float_rn(__dmul_rn(s[j], 0.125));
            amax = fmaxf(amax, fabsf(m[j]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float scale = __fdiv_rn(amax, 448.0f);
        uint32_t c01 = 0, c23 = 0, c45 = 0, c67 = 0;
        if (scale != 0.0f) {
            c01 = cvt_e4m3x2(__fdiv_rn(m[0], scale), __fdiv_rn(m[1], scale));
            c23 = cvt_e4m3x2(__fdiv_rn(m[2], scale), __fdiv_rn(m[3], scale));
            c45 = cvt_e4m3x2(__fdiv_rn(m[4], scale), __fdiv_rn(m[5], scale));
            c67 = cvt_e4m3x2(__fdiv_rn(m[6], scale), __fdiv_rn(m[7], scale));
        }
        uint2 out;
        out.x = c01 | (c23 << 16);
        out.y = c45 | (c67 << 16);
        const int64_t row = (int64_t)g * n_slots + slot;
        *reinterpret_cast<uint2 *>(summaries + row * kDI + lane * 8) = out;
        if (lane == 0) scales[row] = scale;
    }
}

}  // namespace dsa
