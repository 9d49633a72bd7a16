// A3 top-k region selection ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: a radix-
// style top-k keeps the best regions and always includes the query's own region).
//
// Per row (query, group) with own = q_pos/8 and need = min(k-1, own):
//   hist   : 4096-bin histogram of the top 12 bits of the order-preserving score key
//            (grid over row chunks, smem histograms flushed with global atomics);
//   gather : every CTA finds the threshold bin T (the bin holding the need-th largest
//            key) from the global histogram; keys in bins above T are certainly selected,
//            keys in bin T are candidates (warp-aggregated appends to workspace lists);
//   final  : one CTA per row radix-refines the candidates on the remaining key bits and
//            then on the inverted region index (so equal scores prefer the lower index),
//            marks the chosen regions plus the own region in a smem bitmap and emits them
//            in ascending order with a block prefix sum.  No full sort anywhere.
#pragma once

#include "common.cuh"

namespace dsa {
namespace topk {

constexpr int kBins = 4096;           // first-level bins: key bits 31..20
constexpr int kChunk = 4096;          // scores per CTA in hist/gather
constexpr int kThreads = 256;
constexpr int kFinalThreads = 1024;
constexpr int kMaxRegions = 1 << 20;  // ld limit: bitmap in smem, 20-bit region indices

struct Ws {
    uint32_t *hist;     // [rows][kBins]
    uint32_t *ctr;      // [rows][4]: sure count, candidate count
    int32_t *sure;      // [rows][k]
    uint2 *cand;        // [rows][ld]: (key, region)
};

__device__ __forceinline__ int64_t row_own(const int32_t *q_pos, int row)
{
    const int p = q_pos[row >> 2];
    return p < 0 ? -1 : p / kRegion;
}

// Inclusive scan over the threads of a block (NT threads, values in thread order).
template <int NT>
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t *warp_sums)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = (lane < NT / 32) ? warp_sums[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += x;
        }
        if (lane < NT / 32) warp_sums[lane] = w;
    }
    __syncthreads();
    const uint32_t add = warp > 0 ? warp_sums[warp - 1] : 0u;
    __syncthreads();
    return v + add;
}

// Over the bins of `hist` in DESCENDING order, find the bin where the running count first
// reaches m (1 <= m <= total).  Every thread returns the bin and the count strictly above.
template <int NT>
__device__ __forceinline__ void find_desc(const uint32_t *hist, int nb, uint32_t m, uint32_t *scratch,
                                          int &bin_out, uint32_t &above_out)
{
    const int bpt = (nb + NT - 1) / NT;
    const int p0 = threadIdx.x * bpt;
    uint32_t s = 0;
    for (int i = 0; i < bpt; ++i)
        if (p0 + i < nb) s += hist[nb - 1 - (p0 + i)];
    const uint32_t incl = block_inclusive_scan<NT>(s, scratch);
    if (incl >= m && incl - s < m) {
        uint32_t run = incl - s;
        for (int i = 0; i < bpt; ++i) {
            const int b = nb - 1 - (p0 + i);
            const uint32_t h = hist[b];
            if (run + h >= m) {
                scratch[32] = (uint32_t)b;
                scratch[33] = run;
                break;
            }
            run += h;
        }
    }
    __syncthreads();
    bin_out = (int)scratch[32];
    above_out = scratch[33];
    __syncthreads();
}

__global__ void __launch_bounds__(kThreads) hist_kernel(const float *__restrict__ scores, int64_t ld,
                                                        const int32_t *__restrict__ q_pos, int k, Ws ws)
{
    __shared__ uint32_t h[kBins];
    const int row = blockIdx.y;
    const int64_t own = row_own(q_pos, row);
    if (own < 0 || own > ld) return;
    const int64_t need = min((int64_t)(k - 1), own);
    if (need == own || need == 0) return;             // all eligible selected, or only the own region
    const int64_t c0 = (int64_t)blockIdx.x * kChunk;
    if (c0 >= own) return;
    for (int i = threadIdx.x; i < kBins; i += kThreads) h[i] = 0;
    __syncthreads();
    const float *src = scores + (int64_t)row * ld;
    const int64_t c1 = min(own, c0 + kChunk);
    for (int64_t r = c0 + threadIdx.x; r < c1; r += kThreads) atomicAdd(&h[score_key(src[r]) >> 20], 1u);
    __syncthreads();
    uint32_t *gh = ws.hist + (int64_t)row * kBins;
    for (int i = threadIdx.x; i < kBins; i += kThreads)
        if (h[i]) atomicAdd(&gh[i], h[i]);
}

__global__ void __launch_bounds__(kThreads) gather_kernel(const float *__restrict__ scores, int64_t ld,
                                                          const int32_t *__restrict__ q_pos, int k, Ws ws)
{
    __shared__ uint32_t h[kBins];
    __shared__ uint32_t scratch[40];
    const int row = blockIdx.y;
    const int64_t own = row_own(q_pos, row);
    if (own < 0 || own > ld) return;
    const int64_t need = min((int64_t)(k - 1), own);
    if (need == own || need == 0) return;
    const int64_t c0 = (int64_t)blockIdx.x * kChunk;
    if (c0 >= own) return;
    const uint32_t *gh = ws.hist + (int64_t)row * kBins;
    for (int i = threadIdx.x; i < kBins; i += kThreads) h[i] = gh[i];
    __syncthreads();
    int T;
    uint32_t above;
    find_desc<kThreads>(h, kBins, (uint32_t)need, scratch, T, above);

    const float *src = scores + (int64_t)row * ld;
    const int64_t c1 = min(own, c0 + kChunk);
    uint32_t *ctr = ws.ctr + (int64_t)row * 4;
    int32_t *sure = ws.sure + (int64_t)row * k;
    uint2 *cand = ws.cand + (int64_t)row * ld;
    const int lane = threadIdx.x & 31;
    for (int64_t base = c0; base < c1; base += kThreads) {
        const int64_t r = base + threadIdx.x;
        uint32_t key = 0;
        int bin = -1;
        if (r < c1) {
            key = score_key(src[r]);
            bin = (int)(key >> 20);
        }
        const bool is_sure = bin > T, is_cand = bin == T;
        const unsigned ms = __ballot_sync(0xffffffffu, is_sure);
        const unsigned mc = __ballot_sync(0xffffffffu, is_cand);
        uint32_t bs = 0, bc = 0;
        if (lane == 0) {
            if (ms) bs = atomicAdd(&ctr[0], (uint32_t)__popc(ms));
            if (mc) bc = atomicAdd(&ctr[1], (uint32_t)__popc(mc));
        }
        bs = __shfl_sync(0xffffffffu, bs, 0);
        bc = __shfl_sync(0xffffffffu, bc, 0);
        const unsigned below = (1u << lane) - 1u;
        if (is_sure) {
            const uint32_t pos = bs + __popc(ms & below);
            if (pos < (uint32_t)need) sure[pos] = (int32_t)r;
        }
        if (is_cand) {
            const uint32_t pos = bc + __popc(mc & below);
            if (pos < (uint64_t)ld) cand[pos] = make_uint2(key, (uint32_t)r);
        }
    }
}

// Composite rank key of a candidate: score key, then the inverted region index so that
// among equal scores the lower region index ranks higher.
__device__ __forceinline__ uint64_t composite(uint2 c)
{
    return ((uint64_t)c.x << 32) | (uint64_t)(0xFFFFFFFFu - c.y);
}

__global__ void __launch_bounds__(kFinalThreads) final_kernel(const int32_t *__restrict__ q_pos, int64_t ld, int k,
                                                              Ws ws, int32_t *__restrict__ sel_idx,
                                                              int32_t *__restrict__ sel_count)
{
    extern __shared__ uint32_t bitmap[];                 // (ld + 1 + 31) / 32 words
    __shared__ uint32_t h[kBins];
    __shared__ uint32_t scratch[40];
    const int row = blockIdx.x;
    const int tid = threadIdx.x;
    int32_t *out = sel_idx + (int64_t)row * k;
    const int64_t own = row_own(q_pos, row);
    if (own < 0 || own > ld) {
        if (tid == 0) {
            set_error(kErrTopkRow);
            sel_count[row] = 0;
        }
        for (int i = tid; i < k; i += kFinalThreads) out[i] = -1;
        return;
    }
    const int64_t need = min((int64_t)(k - 1), own);
    const int words = (int)((own + 1 + 31) / 32);
    for (int i = tid; i < words; i += kFinalThreads) bitmap[i] = 0;
    __syncthreads();

    if (need == own) {
        for (int i = tid; i < words; i += kFinalThreads) {
            const int64_t lo = (int64_t)i * 32;
            const int64_t nbits = min((int64_t)32, own + 1 - lo);
            bitmap[i] = nbits >= 32 ? 0xFFFFFFFFu : ((1u << nbits) - 1u);
        }
    } else if (need > 0) {
        const uint32_t *ctr = ws.ctr + (int64_t)row * 4;
        const uint32_t n_sure = ctr[0], n_cand = ctr[1];
        const bool counts_ok = n_sure <= (uint32_t)need && n_cand <= (uint64_t)own;
        const int32_t *sure = ws.sure + (int64_t)row * k;
        const uint2 *cand = ws.cand + (int64_t)row * ld;
        const int64_t m = need - (int64_t)n_sure;
        if (!counts_ok || m < 1 || m > (int64_t)n_cand) {
            if (tid == 0) set_error(kErrTopkInternal);
        } else {
            for (uint32_t i = tid; i < n_sure; i += kFinalThreads) {
                const int32_t r = sure[i];
                if (r >= 0 && r < own) atomicOr(&bitmap[r >> 5], 1u << (r & 31));
            }
            // radix refinement of the candidates (all share key bits 31..20)
            uint64_t prefix = 0, pmask = 0;
            uint32_t m_rem = (uint32_t)m;
            bool all_equal_taken = (m_rem == n_cand);
            const int shifts[4] = {40, 32, 10, 0};
            const int widths[4] = {12, 8, 10, 10};
            for (int pass = 0; pass < 4 && !all_equal_taken; ++pass) {
                const int sh = shifts[pass], nb = 1 << widths[pass];
                for (int i = tid; i < nb; i += kFinalThreads) h[i] = 0;
                __syncthreads();
                for (uint32_t i = tid; i < n_cand; i += kFinalThreads) {
                    const uint64_t c = composite(cand[i]);
                    if ((c & pmask) == prefix) atomicAdd(&h[(c >> sh) & (uint64_t)(nb - 1)], 1u);
                }
                __syncthreads();
                int B;
                uint32_t above;
                find_desc<kFinalThreads>(h, nb, m_rem, scratch, B, above);
                m_rem -= above;
                prefix |= (uint64_t)B << sh;
                pmask |= (uint64_t)(nb - 1) << sh;
                all_equal_taken = (h[B] == m_rem);
                __syncthreads();
            }
            if (!all_equal_taken) {
                if (tid == 0) set_error(kErrTopkInternal);
            } else {
                for (uint32_t i = tid; i < n_cand; i += kFinalThreads) {
                    const uint2 cd = cand[i];
                    const uint64_t c = composite(cd) & pmask;
                    if (c >= prefix && cd.y < (uint64_t)own) atomicOr(&bitmap[cd.y >> 5], 1u << (cd.y & 31));
                }
            }
        }
    }
    __syncthreads();
    if (tid == 0) atomicOr(&bitmap[own >> 5], 1u << (own & 31));
    __syncthreads();

    // ordered emit: thread i owns words [i*wpt, (i+1)*wpt)
    const int wpt = (words + kFinalThreads - 1) / kFinalThreads;
    const int w0 = tid * wpt;
    uint32_t cnt = 0;
    for (int i = 0; i < wpt; ++i)
        if (w0 + i < words) cnt += __popc(bitmap[w0 + i]);
    const uint32_t incl = block_inclusive_scan<kFinalThreads>(cnt, scratch);
    uint32_t pos = incl - cnt;
    for (int i = 0; i < wpt; ++i) {
        if (w0 + i >= words) break;
        uint32_t b = bitmap[w0 + i];
        while (b) {
            const int bit = __ffs(b) - 1;
            b &= b - 1;
            if (pos < (uint32_t)k) out[pos] = (w0 + i) * 32 + bit;
            ++pos;
        }
    }
    if (tid == kFinalThreads - 1) {
        const uint32_t total = incl;
        if (total != (uint32_t)(need + 1)) set_error(kErrTopkInternal);
        sel_count[row] = (int32_t)min(total, (uint32_t)k);
        scratch[34] = total;
    }
    __syncthreads();
    for (int i = (int)scratch[34] + tid; i < k; i += kFinalThreads) out[i] = -1;
}

}  // namespace topk
}  // namespace dsa
