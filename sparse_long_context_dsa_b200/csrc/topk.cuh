// A3 top-k region selection ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: a radix-
// style top-k keeps the best regions and always includes the query's own region).
//
// Per row (query, group) with own = q_pos/8 and need = min(k-1, own):
//   hist   : 4096-bin histogram of the top 12 bits of the order-preserving score key
//            (grid over row chunks, smem histograms flushed with global atomics);
//   select : every CTA finds the threshold bin T (the bin holding the need-th largest
//            key) from the global histogram; keys in bins above T are certainly selected,
//            keys in bin T are candidates (per-CTA block-scan compaction, one atomic
//            reservation per list).  The last CTA of the row to finish (atomic counter, no
//            waiting) radix-refines the candidates on the remaining key bits and then on
//            the inverted region index (so equal scores prefer the lower index), marks the
//            chosen regions plus the own region in a smem bitmap and emits them in
//            ascending order with a block prefix sum.  No full sort anywhere.
#pragma once

#include "common.cuh"

namespace dsa {
namespace topk {

constexpr int kBins = 4096;           // first-level bins: key bits 31..20
constexpr int kChunk = 4096;          // scores per CTA in hist/gather
constexpr int kThreads = 256;
constexpr int kSelectThreads = 512;
constexpr int kMaxRegions = 1 << 20;  // ld limit: bitmap in smem, 20-bit region indices
constexpr int kCandStage = 4096;      // candidates staged in smem by the final phase

struct Ws {
    uint32_t *hist;     // [rows][kBins]
    uint32_t *ctr;      // [rows][4]: sure count, candidate count, finished CTAs
    int32_t *sure;      // [rows][k]
    uint2 *cand;        // [rows][ld]: (key, region)
    int gshift;         // rows per query = 2^gshift (the KV groups of the call)
};

__device__ __forceinline__ int64_t row_own(const int32_t *q_pos, int row, int gshift)
{
    const int p = q_pos[row >> gshift];
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
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    __shared__ uint32_t h[kBins];
    const int row = blockIdx.y;
    const int64_t own = row_own(q_pos, row, ws.gshift);
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

// Composite rank key of a candidate: score key, then the inverted region index so that
// among equal scores the lower region index ranks higher.
__device__ __forceinline__ uint64_t composite(uint2 c)
{
    return ((uint64_t)c.x << 32) | (uint64_t)(0xFFFFFFFFu - c.y);
}

// Final selection of one row by one CTA: marks the sure regions, radix-refines the
// candidates (all share key bits 31..20) on the remaining key bits and then on the
// inverted region index, adds the own region and emits the set in ascending order.
template <int NT>
__device__ void finish_row(int row, int64_t own, int64_t need, int64_t ld, int k, const Ws &ws, uint32_t *bitmap,
                           uint32_t *h, uint32_t *scratch, uint2 *cstage, int32_t *__restrict__ sel_idx,
                           int32_t *__restrict__ sel_count)
{
    const int tid = threadIdx.x;
    int32_t *out = sel_idx + (int64_t)row * k;
    const int words = (int)((own + 1 + 31) / 32);
    for (int i = tid; i < words; i += NT) bitmap[i] = 0;
    __syncthreads();

    if (need == own) {
        for (int i = tid; i < words; i += NT) {
            const int64_t lo = (int64_t)i * 32;
            const int64_t nbits = min((int64_t)32, own + 1 - lo);
            bitmap[i] = nbits >= 32 ? 0xFFFFFFFFu : ((1u << nbits) - 1u);
        }
    } else if (need > 0) {
        const uint32_t *ctr = ws.ctr + (int64_t)row * 4;
        const uint32_t n_sure = __ldcg(&ctr[0]), n_cand = __ldcg(&ctr[1]);
        const bool counts_ok = n_sure <= (uint32_t)need && n_cand <= (uint64_t)own;
        const int32_t *sure = ws.sure + (int64_t)row * k;
        const uint2 *cand = ws.cand + (int64_t)row * ld;
        // the candidates (usually a few hundred) are read once into smem when they fit
        if (n_cand <= (uint32_t)kCandStage && counts_ok) {
            for (uint32_t i = tid; i < n_cand; i += NT) cstage[i] = __ldcg(&cand[i]);
            cand = cstage;
        }
        const int64_t m = need - (int64_t)n_sure;
        if (!counts_ok || m < 1 || m > (int64_t)n_cand) {
            if (tid == 0) set_error(kErrTopkInternal);
        } else {
            for (uint32_t i = tid; i < n_sure; i += NT) {
                const int32_t r = __ldcg(&sure[i]);
                if (r >= 0 && r < own) atomicOr(&bitmap[r >> 5], 1u << (r & 31));
            }
            uint64_t prefix = 0, pmask = 0;
            uint32_t m_rem = (uint32_t)m;
            bool all_equal_taken = (m_rem == n_cand);
            const int shifts[4] = {40, 32, 10, 0};
            const int widths[4] = {12, 8, 10, 10};
            for (int pass = 0; pass < 4 && !all_equal_taken; ++pass) {
                const int sh = shifts[pass], nb = 1 << widths[pass];
                for (int i = tid; i < nb; i += NT) h[i] = 0;
                __syncthreads();
                for (uint32_t i = tid; i < n_cand; i += NT) {
                    const uint64_t c = composite(cand[i]);
                    if ((c & pmask) == prefix) atomicAdd(&h[(c >> sh) & (uint64_t)(nb - 1)], 1u);
                }
                __syncthreads();
                int B;
                uint32_t above;
                find_desc<NT>(h, nb, m_rem, scratch, B, above);
                m_rem -= above;
                prefix |= (uint64_t)B << sh;
                pmask |= (uint64_t)(nb - 1) << sh;
                all_equal_taken = (h[B] == m_rem);
                __syncthreads();
            }
            if (!all_equal_taken) {
                if (tid == 0) set_error(kErrTopkInternal);
            } else {
                for (uint32_t i = tid; i < n_cand; i += NT) {
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
    const int wpt = (words + NT - 1) / NT;
    const int w0 = tid * wpt;
    uint32_t cnt = 0;
    for (int i = 0; i < wpt; ++i)
        if (w0 + i < words) cnt += __popc(bitmap[w0 + i]);
    const uint32_t incl = block_inclusive_scan<NT>(cnt, scratch);
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
    if (tid == NT - 1) {
        const uint32_t total = incl;
        if (total != (uint32_t)(need + 1)) set_error(kErrTopkInternal);
        sel_count[row] = (int32_t)min(total, (uint32_t)k);
        scratch[34] = total;
    }
    __syncthreads();
    for (int i = (int)scratch[34] + tid; i < k; i += NT) out[i] = -1;
}

// Threshold-bin gather of one row chunk, then (in the last CTA of the row to finish,
// found with an atomic counter: no CTA ever waits on another) the final selection.
// Dynamic smem: the row bitmap, (ld + 1 + 31) / 32 words.
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const float *__restrict__ scores, int64_t ld,
                                                                const int32_t *__restrict__ q_pos, int k, Ws ws,
                                                                int32_t *__restrict__ sel_idx,
                                                                int32_t *__restrict__ sel_count)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint32_t dyn[];                 // [kCandStage] uint2, then the bitmap
    uint2 *cstage = reinterpret_cast<uint2 *>(dyn);
    uint32_t *bitmap = dyn + 2 * kCandStage;
    __shared__ uint32_t h[kBins];
    __shared__ uint32_t scratch[40];
    constexpr int NT = kSelectThreads;
    const int row = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t own = row_own(q_pos, row, ws.gshift);
    if (own < 0 || own > ld) {
        if (blockIdx.x == 0) {
            if (tid == 0) {
                set_error(kErrTopkRow);
                sel_count[row] = 0;
            }
            for (int i = tid; i < k; i += NT) sel_idx[(int64_t)row * k + i] = -1;
        }
        return;
    }
    const int64_t need = min((int64_t)(k - 1), own);
    if (need == own || need == 0) {                   // no selection needed: one CTA emits
        if (blockIdx.x == 0) finish_row<NT>(row, own, need, ld, k, ws, bitmap, h, scratch, cstage, sel_idx, sel_count);
        return;
    }
    const int64_t c0 = (int64_t)blockIdx.x * kChunk;
    if (c0 >= own) return;
    const int n_chunks = (int)((own + kChunk - 1) / kChunk);

    // this thread's entries r = c0 + e*NT + tid: issue their loads before the histogram's
    constexpr int E = kChunk / NT;
    const float *src = scores + (int64_t)row * ld;
    uint32_t key[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int64_t r = c0 + e * NT + tid;
        key[e] = (r < own) ? score_key(__ldcg(&src[r])) : 0u;
    }
    const uint32_t *gh = ws.hist + (int64_t)row * kBins;
    uint32_t hv[kBins / NT];
#pragma unroll
    for (int i = 0; i < kBins / NT; ++i) hv[i] = __ldcg(&gh[i * NT + tid]);
#pragma unroll
    for (int i = 0; i < kBins / NT; ++i) h[i * NT + tid] = hv[i];
    __syncthreads();
    int T;
    uint32_t above;
    find_desc<NT>(h, kBins, (uint32_t)need, scratch, T, above);

    // classify, count, block-scan, one atomic reservation per list and CTA, then write
    int cls[E];                                        // 2 = sure, 1 = candidate, 0 = neither
    uint32_t ns = 0, nc = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int64_t r = c0 + e * NT + tid;
        cls[e] = 0;
        if (r < own) {
            const int bin = (int)(key[e] >> 20);
            cls[e] = bin > T ? 2 : (bin == T ? 1 : 0);
        }
        ns += cls[e] == 2;
        nc += cls[e] == 1;
    }
    const uint32_t incl = block_inclusive_scan<NT>((ns << 16) | nc, scratch);
    uint32_t *ctr = ws.ctr + (int64_t)row * 4;
    if (tid == NT - 1) {
        const uint32_t tot_s = incl >> 16, tot_c = incl & 0xFFFFu;
        scratch[36] = tot_s ? atomicAdd(&ctr[0], tot_s) : 0u;
        scratch[37] = tot_c ? atomicAdd(&ctr[1], tot_c) : 0u;
    }
    __syncthreads();
    uint32_t ps = scratch[36] + ((incl - ((ns << 16) | nc)) >> 16);
    uint32_t pc = scratch[37] + ((incl - ((ns << 16) | nc)) & 0xFFFFu);
    int32_t *sure = ws.sure + (int64_t)row * k;
    uint2 *cand = ws.cand + (int64_t)row * ld;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int64_t r = c0 + e * NT + tid;
        if (cls[e] == 2) {
            if (ps < (uint32_t)need) sure[ps] = (int32_t)r;
            ++ps;
        } else if (cls[e] == 1) {
            if (pc < (uint64_t)ld) cand[pc] = make_uint2(key[e], (uint32_t)r);
            ++pc;
        }
    }
    // publish, then find out whether this CTA is the row's last
    __threadfence();
    __syncthreads();
    if (tid == 0) scratch[38] = (atomicAdd(&ctr[2], 1u) == (uint32_t)(n_chunks - 1)) ? 1u : 0u;
    __syncthreads();
    if (scratch[38] == 0) return;
    __threadfence();
    finish_row<NT>(row, own, need, ld, k, ws, bitmap, h, scratch, cstage, sel_idx, sel_count);
}

}  // namespace topk
}  // namespace dsa
