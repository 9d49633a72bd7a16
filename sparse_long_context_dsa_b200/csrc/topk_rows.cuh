// A3 top-k region selection for many rows of moderate length (a prefill chunk: 8,192 rows of
// up to 65,536 scores), one CTA per (query, group) row, no global scratch ([P2] Step-5-Preview
// 如何实现1M长上下文 §索引器打分: a radix-style top-k keeps the best regions and always includes
// the query's own region).
//  1. one pass over the row: thread t of 256 reads entries t, t+256, ... (coalesced) and keeps
//     the maximum of each of its 8 strided groups (entry t + 256j joins group j % 8): 2,048
//     group maxima per row.  Five CTAs share an SM, so one row's threshold and emit overlap
//     the other rows' streaming;
//  2. 256-bin histogram levels over the group maxima narrow the need-th largest maximum to a
//     range [elo, ehi) holding at most 64 maxima (or one value).  At least need groups have a
//     maximum >= elo, so at least need scores are >= elo; the scores >= elo all lie in those
//     at most need + 64 groups;
//  3. a second pass (the row is still in L2) compacts the scores >= elo into smem as
//     (score, region) composites, warp-aggregated;
//  4. the exact threshold over the composites (topkc::block_threshold: histogram levels and a
//     pairwise rank; ties go to the lower region), the selection marked in a bitmap of the
//     regions with the own region, emitted in ascending order.
// Rows whose candidates would not fit (long runs of equal scores) take the same threshold
// over the whole row, read from memory in every level (slow, exact).
#pragma once

#include "topk_cluster.cuh"

namespace dsa {
namespace topkr {

using topkc::block_scan_incl;
using topkc::block_threshold;
using topkc::desc_bin_search;
using topkc::key_levels;
using topkc::threshold_selects;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kGroupsPerThread = 8;
constexpr int kMaxLd = 65536;                       // scores per row
constexpr int kMaxCand = 4096;                      // candidates kept in smem (more: the whole-row path)
constexpr int kBitmapWords = kMaxLd / 32 + 1;
constexpr int kBatch = 16;                          // loads in flight per thread
// smem (bytes)
constexpr size_t kOffCand = 0;                                               // [kMaxCand] composites
constexpr size_t kOffBitmap = kOffCand + (size_t)kMaxCand * 8;                // [kBitmapWords]
constexpr size_t kOffList = kOffBitmap + ((size_t)kBitmapWords * 4 + 15) / 16 * 16;   // [32] composites
constexpr size_t kOffHs = kOffList + 32 * 8;                                  // [256]
constexpr size_t kSmemBytes = kOffHs + 256 * 4 + 16;
static_assert(5 * kSmemBytes <= 227 * 1024, "five CTAs per SM");

__global__ void __launch_bounds__(kThreads, 5)
    topk_rows_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ q_pos, int k,
                     int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_count, int gshift)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t *cand = reinterpret_cast<uint64_t *>(smem_raw + kOffCand);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem_raw + kOffBitmap);
    uint64_t *list = reinterpret_cast<uint64_t *>(smem_raw + kOffList);
    uint32_t *hs = reinterpret_cast<uint32_t *>(smem_raw + kOffHs);
    __shared__ uint32_t scan_ws[40];
    __shared__ uint32_t sh_min, sh_max, sh_nin, sh_ncand;
    __shared__ uint64_t bc[2 * kWarps];

    const int tid = threadIdx.x, lane = tid & 31;
    const int row = blockIdx.x;
    const int p = q_pos[row >> gshift];   // rows per query = 2^gshift (the call's KV groups)
    const bool valid = p >= 0 && (int64_t)(p / kRegion) <= ld;
    const int64_t own = valid ? p / kRegion : 0;
    const int64_t need = valid ? min((int64_t)(k - 1), own) : 0;
    int32_t *out = sel_idx + (int64_t)row * k;
    if (!valid || own > kMaxLd) {
        if (tid == 0) {
            set_error(valid ? kErrTopkInternal : kErrTopkRow);
            sel_count[row] = 0;
        }
        for (int i = tid; i < k; i += kThreads) out[i] = -1;
        return;
    }
    if (need == own || need == 0) {                     // every eligible region (or none), then own
        for (int i = tid; i < k; i += kThreads) out[i] = i < need ? i : (i == need ? (int32_t)own : -1);
        if (tid == 0) sel_count[row] = (int32_t)(need + 1);
        return;
    }
    if (tid == 0) {
        sh_min = 0xFFFFFFFFu;
        sh_max = 0u;
        sh_nin = 0u;
        sh_ncand = 0u;
    }
    const int n = (int)own;                             // eligible entries 0 .. own-1
    const float *src = scores + (int64_t)row * ld;
    // ---- 1. group maxima (0: a group with no eligible entry).  The maximum is taken over the
    // floats (entries past the row as -inf) and turned into a key once per group: fmaxf skips
    // a NaN and may return -0 for +0, so a group's key can only fall short of its largest
    // entry's, which lowers the bound below and keeps the candidates a superset of the
    // selection.  Group j of thread t first holds entry j * kThreads + t (kBatch is a multiple
    // of kGroupsPerThread).
    static_assert(kBatch % kGroupsPerThread == 0, "group j's first entry is j * kThreads + t");
    float gf[kGroupsPerThread];
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) gf[j] = -INFINITY;
    for (int base = 0; base < n; base += kThreads * kBatch) {
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = base + u * kThreads + tid;
            v[u] = i < n ? __ldcg(src + i) : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) gf[u & (kGroupsPerThread - 1)] = fmaxf(gf[u & (kGroupsPerThread - 1)], v[u]);
    }
    uint32_t gm[kGroupsPerThread];
#pragma unroll
    for (int j = 0; j < kGroupsPerThread; ++j) gm[j] = j * kThreads + tid < n ? score_key(gf[j]) : 0u;
    __syncthreads();                                    // shared counters initialised
    // ---- 2. the bound: a range [elo, ehi) of group maxima holding the need-th largest
    auto gvalid = [&](int u) { return gm[u] != 0u; };
    auto gkey = [&](int u) { return gm[u]; };
    uint64_t elo, ehi;
    uint32_t above, n_in;
    key_levels<kGroupsPerThread>(gvalid, gkey, (uint32_t)need, 64u, hs, &sh_min, &sh_max, scan_ws + 32, elo, ehi,
                                 above, n_in);
    const uint32_t lo_key = (uint32_t)elo;
    // ---- 3. candidates: scores >= elo, compacted (warp-aggregated slots).  The test runs on
    // floats against lo_f, the float whose key is lo_key: !(v < lo_f) holds for every entry of
    // key >= lo_key, and also for NaN and for the other zero, so the candidates are again a
    // superset; their exact keys are formed only for the candidates
    const float lo_f = __uint_as_float((lo_key & 0x80000000u) ? (lo_key & 0x7FFFFFFFu) : ~lo_key);
    const unsigned below = (1u << lane) - 1u;
    for (int base = 0; base < n; base += kThreads * kBatch) {
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = base + u * kThreads + tid;
            v[u] = i < n ? __ldcg(src + i) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = base + u * kThreads + tid;
            const bool c = i < n && !(v[u] < lo_f);
            const unsigned m = __ballot_sync(0xffffffffu, c);
            if (m == 0u) continue;
            const uint32_t key = score_key(v[u]);
            uint32_t slot0 = 0;
            if (lane == 0) slot0 = atomicAdd(&sh_ncand, (uint32_t)__popc(m));
            slot0 = __shfl_sync(0xffffffffu, slot0, 0);
            const uint32_t slot = slot0 + __popc(m & below);
            if (c && slot < (uint32_t)kMaxCand) cand[slot] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)i);
        }
    }
    if (tid == 0) sh_max = 0u;
    __syncthreads();
    const uint32_t n_cand = sh_ncand;
    uint64_t elo2, ehi2, cp, cm;
    const int words = (int)((own + 1 + 31) / 32);
    if (n_cand <= (uint32_t)kMaxCand) {
        // ---- 4. the exact threshold over the candidates (read from smem on demand)
        constexpr int R = kMaxCand / kThreads;          // 16
        auto cvalid = [&](int u) { return (uint32_t)(u * kThreads + tid) < n_cand; };
        auto ccomp = [&](int u) { return cand[u * kThreads + tid]; };
        const int r_used = (int)((n_cand + kThreads - 1) / kThreads);
        block_threshold<R>(cvalid, ccomp, (uint32_t)need, lo_key, hs, list, nullptr, &sh_max, &sh_nin, scan_ws + 32,
                           bc, &elo2, &ehi2, &cp, &cm, r_used);
        for (int i = tid; i < words; i += kThreads) bitmap[i] = 0u;
        __syncthreads();
#pragma unroll 4
        for (int u = 0; u < r_used; ++u)
            if (cvalid(u) && threshold_selects(ccomp(u), elo2, ehi2, cp, cm)) {
                const uint32_t r = 0xFFFFFFFFu - (uint32_t)ccomp(u);
                atomicOr(&bitmap[r >> 5], 1u << (r & 31));
            }
    } else {
        // equal scores in bulk: the same threshold over the whole row, read in every level
        constexpr int R = kMaxLd / kThreads;            // 256
        auto rvalid = [&](int u) { return u * kThreads + tid < n; };
        auto rcomp = [&](int u) {
            const int i = u * kThreads + tid;
            return ((uint64_t)score_key(__ldcg(src + i)) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)i);
        };
        block_threshold<R>(rvalid, rcomp, (uint32_t)need, 0u, hs, list, nullptr, &sh_max, &sh_nin, scan_ws + 32, bc,
                           &elo2, &ehi2, &cp, &cm, (n + kThreads - 1) / kThreads);
        for (int i = tid; i < words; i += kThreads) bitmap[i] = 0u;
        __syncthreads();
#pragma unroll 4
        for (int u = 0; u < R; ++u)
            if (rvalid(u) && threshold_selects(rcomp(u), elo2, ehi2, cp, cm)) {
                const uint32_t r = (uint32_t)(u * kThreads + tid);
                atomicOr(&bitmap[r >> 5], 1u << (r & 31));
            }
    }
    if (tid == 0) atomicOr(&bitmap[own >> 5], 1u << (own & 31));
    __syncthreads();
    // ---- 5. ascending emit: thread t owns the bitmap words [t*wpt, (t+1)*wpt)
    const int wpt = (words + kThreads - 1) / kThreads;
    const int w0 = tid * wpt;
    uint32_t bcnt = 0;
    for (int i = 0; i < wpt; ++i)
        if (w0 + i < words) bcnt += __popc(bitmap[w0 + i]);
    const uint32_t incl = block_scan_incl<kThreads>(bcnt, scan_ws);
    uint32_t opos = incl - bcnt;
    for (int i = 0; i < wpt; ++i) {
        if (w0 + i >= words) break;
        uint32_t bits = bitmap[w0 + i];
        while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1;
            if (opos < (uint32_t)k) out[opos] = (w0 + i) * 32 + bit;
            ++opos;
        }
    }
    if (tid == kThreads - 1) {
        if (incl != (uint32_t)(need + 1)) set_error(kErrTopkInternal);
        sel_count[row] = (int32_t)(need + 1);
    }
    for (int i = (int)need + 1 + tid; i < k; i += kThreads) out[i] = -1;
}

}  // namespace topkr
}  // namespace dsa
