// A3 top-k region selection, one thread-block cluster per (query, group) row
// ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: a radix-style top-k keeps the best
// regions and always includes the query's own region).
//
// For few long rows (decode: 4 rows of up to 131,071 scores per query) a row is split over
// a cluster of CL CTAs; CTA `rank` owns the contiguous region range [rank*part, ...).
// Fast path, two cluster barriers in all:
//  1. every thread's share of the CTA's range is loaded coalesced (all loads, the query
//     position's included, in flight at once: the partition follows the row length, and
//     entries at or beyond the own region are masked afterwards), staged in shared memory
//     and taken back as a run of 32 consecutive order-preserving keys: a group.  The group
//     maxima go to every CTA of the cluster;
//  2. every CTA selects the same bound L from the group maxima: the lower edge of the (at
//     most two) 8-bit digit bins that hold the need-th largest maximum.  At least `need`
//     groups have a maximum >= L, so at least `need` keys are >= L, and few more (groups
//     holding two of the best keys);
//  3. the keys >= L are pushed in region order, with each CTA's count, into rank 0's shared
//     memory; rank 0 gathers them densely (still in region order), selects exactly the need
//     largest (key desc, then region asc) and writes them with one ordered compaction, the
//     own region last.  The exact step takes one 2048-bin histogram of the candidate keys
//     over [L, row maximum] and one block scan from the top bin; the bin that holds the
//     need-th largest key is either taken whole or ranked by one warp.
// When the candidates do not fit (many equal scores, or k beyond the group count) every CTA
// sees it in the pushed counts and the cluster runs an exact distributed radix select
// instead: per digit every CTA histograms its keys that match the prefix found so far, the
// cluster sums the histograms through distributed shared memory (each CTA reduces a slice of
// the bins) and every CTA locates the digit; equal keys at the threshold are taken lowest
// region first (a prefix of per-rank tie counts, then an ordered block scan), and the output
// is an ordered compaction over the ranks.  No global scratch, no waiting on other CTAs
// except the cluster's hardware barriers.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace dsa {
namespace topkc {

namespace cg = cooperative_groups;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kPartMax = 16384;                 // scores per CTA
constexpr int kPer = kPartMax / kThreads;       // 32 per thread: one group
constexpr int kPadded = kPartMax + kPartMax / 8;    // fallback: key i at i + 4*(i/32)
constexpr int kMaxCluster = 8;                  // portable cluster size
constexpr int kGroups = kThreads * kMaxCluster; // group maxima per row (at most)
constexpr int kBins = 4096;                     // fallback digit bins
constexpr int kSlots = 8192;                    // candidate slots at rank 0 (kSlots / CL per rank)
constexpr int kDense = 2048;                    // gathered candidates at rank 0
constexpr int kDPer = kDense / kThreads;
// fast-path smem layout (bytes)
constexpr size_t kOffSlots = 0;
constexpr size_t kOffGmax = kOffSlots + (size_t)kSlots * 8;
constexpr size_t kOffHw = kOffGmax + (size_t)kGroups * 4;
constexpr size_t kOffHs = kOffHw + (size_t)kWarps * 256 * 4;
constexpr size_t kOffDense = kOffHs + 256 * 4;
constexpr size_t kFastBytes = kOffDense + (size_t)kDense * 8;
// the staged keys [kPadded] after them; the fallback's hist [2][kBins], gsl [2][kBins] and
// sl_copy [kBins] overlay the fast-path regions (used only after the second barrier)
constexpr size_t kOffKeys = kFastBytes;
constexpr size_t kFallbackBytes = 5 * (size_t)kBins * 4;
constexpr size_t kSmemBytes = kOffKeys + (size_t)kPadded * 4 + 1024;
static_assert(kOffDense % 16 == 0, "aligned smem regions");
static_assert(kFallbackBytes <= kOffKeys, "fallback buffers stay clear of the staged keys");
static_assert(kOffKeys % 16 == 0, "aligned key staging");

// 4 words of padding after every 32 keys: a thread's run of 32 keys is 16-byte aligned and the
// 8 threads of a 16-byte load phase hit distinct banks.
__device__ __forceinline__ int padded(int i) { return i + 4 * (i >> 5); }

template <int NT>
__device__ __forceinline__ uint32_t block_scan_incl(uint32_t v, uint32_t *ws)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
    }
    if (lane == 31) ws[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = (lane < NT / 32) ? ws[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += x;
        }
        if (lane < NT / 32) ws[lane] = w;
    }
    __syncthreads();
    const uint32_t add = warp > 0 ? ws[warp - 1] : 0u;
    __syncthreads();
    return v + add;
}


// The same inclusive block scan with one barrier: every thread adds up the totals of the
// warps before its own (NT / 32 broadcast reads) instead of waiting for one warp to scan
// them.  *total receives the block's sum.  The caller separates consecutive uses of `ws`
// with a barrier (the next writes to ws must not overtake this scan's reads).
template <int NT>
__device__ __forceinline__ uint32_t block_scan_incl1(uint32_t v, uint32_t *ws, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
    }
    if (lane == 31) ws[warp] = v;
    __syncthreads();
    uint32_t add = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const uint32_t x = ws[w];
        add += w < warp ? x : 0u;
        tot += x;
    }
    *total = tot;
    return v + add;
}

// Block-wide min and max (every thread gets both); `ws` needs 2 * kWarps entries.
template <typename T>
__device__ __forceinline__ void block_minmax(T &mn, T &mx, T *ws)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const T a = __shfl_xor_sync(0xffffffffu, mn, o), b = __shfl_xor_sync(0xffffffffu, mx, o);
        mn = a < mn ? a : mn;
        mx = b > mx ? b : mx;
    }
    if (lane == 0) {
        ws[warp] = mn;
        ws[kWarps + warp] = mx;
    }
    __syncthreads();
#pragma unroll 4
    for (int w = 0; w < kWarps; ++w) {
        const T a = ws[w], b = ws[kWarps + w];
        mn = a < mn ? a : mn;
        mx = b > mx ? b : mx;
    }
    __syncthreads();
}

template <typename T>
__device__ __forceinline__ int top_differing_bit(T a, T b)
{
    if (a == b) return -1;
    if constexpr (sizeof(T) == 8) return 63 - __clzll((long long)(a ^ b));
    else return 31 - __clz((int)(a ^ b));
}

// The m-th largest (1 <= m <= count) of the block's register-held values (v[u] of a thread
// counts when bit u of `valid` is set), by digits of at most 8 bits from bit `top` down;
// every value agrees with `first` on the bits above `top` (top = -1: all values equal).
// Each warp histograms into its own 256 bins (values crowd into few bins near the top of a
// score distribution: the conflicts stay inside a warp), 256 threads add the warps' bins
// and one warp scans them.  Returns (prefix, mask): the values v with (v & mask) >= prefix
// are the m largest when the values are distinct; otherwise every value equal to the m-th
// one satisfies it too.  With max_digits the search stops early: then at least m values
// satisfy it (those in the bins at and above the m-th one's).  `hw` needs kWarps * 256
// words, `hs` 256, `res` 3.
template <typename T, int R>
__device__ void cta_select_reg(const T (&v)[R], uint32_t valid, uint32_t m, int top, T first, uint32_t *hw,
                               uint32_t *hs, uint32_t *res, T &prefix_out, T &mask_out, int max_digits = 64)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kBitsT = 8 * sizeof(T);
    T pmask = top >= kBitsT - 1 ? (T)0 : (~(T)0 << (top + 1));
    T prefix = first & pmask;
    uint32_t m_rem = m;
    uint32_t *myh = hw + warp * 256;
    for (int hi = top, d = 0; hi >= 0 && d < max_digits; hi -= 8, ++d) {
        const int sh = max(hi - 7, 0);
        const uint32_t nb = 1u << (hi - sh + 1);
#pragma unroll
        for (int b = lane; b < 256; b += 32) myh[b] = 0;
        __syncwarp();
#pragma unroll
        for (int u = 0; u < R; ++u)
            if (((valid >> u) & 1u) && (v[u] & pmask) == prefix)
                atomicAdd(&myh[(uint32_t)(v[u] >> sh) & (nb - 1)], 1u);
        __syncthreads();
        if (tid < 256) {
            uint32_t s = 0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) s += hw[w * 256 + tid];
            hs[tid] = s;
        }
        __syncthreads();
        if (warp == 0) {
            // descending: lane owns bins nb-1-8*lane .. nb-8-8*lane
            uint32_t c[8], s = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int bin = (int)nb - 1 - (lane * 8 + u);
                c[u] = bin >= 0 ? hs[bin] : 0u;
                s += c[u];
            }
            uint32_t incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += x;
            }
            const uint32_t excl = incl - s;
            if (excl < m_rem && incl >= m_rem) {
                uint32_t run = excl;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (run + c[u] >= m_rem) {
                        res[0] = (uint32_t)((int)nb - 1 - (lane * 8 + u));
                        res[1] = run;
                        res[2] = c[u];
                        break;
                    }
                    run += c[u];
                }
            }
        }
        __syncthreads();
        const uint32_t B = res[0], above = res[1], binc = res[2];
        m_rem -= above;
        prefix |= (T)B << sh;
        pmask |= (T)(nb - 1) << sh;
        if (binc == m_rem) break;
    }
    prefix_out = prefix;
    mask_out = pmask;
}

// One warp: the bin (scanning 256 bins from the top) that holds the m-th largest value, the
// count above it and its own count, into res[0..2] (m <= total count).
__device__ __forceinline__ void desc_bin_search(const uint32_t *h, uint32_t m, uint32_t *res)
{
    const int lane = threadIdx.x & 31;
    uint32_t c[8], s = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        c[u] = h[255 - (lane * 8 + u)];
        s += c[u];
    }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    const uint32_t excl = incl - s;
    if (excl < m && incl >= m) {
        uint32_t run = excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (run + c[u] >= m) {
                res[0] = (uint32_t)(255 - (lane * 8 + u));
                res[1] = run;
                res[2] = c[u];
                break;
            }
            run += c[u];
        }
    }
}

// Exact threshold of the m largest among the block's (key, region) items, each thread holding
// R of them (item u of a thread counts when valid(u); comp(u) = key << 32 | ~region, all
// distinct, so ties of equal keys go to the lower region).  Levels of 256-bin histograms over
// the 64-bit composites (power-of-two bin widths: the first over [min, max], each next one
// inside the previous level's bin of the m-th largest) narrow the m-th largest down to a bin of
// at most 32 items, which one warp ranks pairwise.  The result is the m-th largest composite T:
// afterwards an item is selected iff comp >= T (returned as *cp with *cm = all ones, *elo = 0,
// *ehi = 2^32, the form threshold_selects takes); exactly m items are.  Needs 1 <= m <= the
// valid count.  hs: 256 words; list: 32 8-byte words; sh_kmax, sh_nin: zeroed before the call
// (klo and hw are unused: kept for the callers' layout).
template <int R, typename Valid, typename Comp>
__device__ bool block_threshold(Valid valid, Comp comp, uint32_t m, uint32_t klo, uint32_t *hs, uint64_t *list,
                                uint32_t *hw, uint32_t *sh_kmax, uint32_t *sh_nin, uint32_t *res, uint64_t *bc,
                                uint64_t *elo, uint64_t *ehi, uint64_t *cp, uint64_t *cm, int r_used = R)
{
    (void)klo;
    (void)hw;
    (void)sh_kmax;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ unsigned long long s_min, s_max;
    uint64_t cmn = ~0ull, cmx = 0ull;
#pragma unroll 8
    for (int u = 0; u < R && u < r_used; ++u)
        if (valid(u)) {
            const uint64_t c = comp(u);
            cmn = c < cmn ? c : cmn;
            cmx = c > cmx ? c : cmx;
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t a = __shfl_xor_sync(0xffffffffu, cmn, o), b2 = __shfl_xor_sync(0xffffffffu, cmx, o);
        cmn = a < cmn ? a : cmn;
        cmx = b2 > cmx ? b2 : cmx;
    }
    if (tid == 0) {
        s_min = ~0ull;
        s_max = 0ull;
    }
    if (tid < 256) hs[tid] = 0u;
    __syncthreads();
    if (lane == 0) {
        atomicMin(&s_min, (unsigned long long)cmn);
        atomicMax(&s_max, (unsigned long long)cmx);
    }
    __syncthreads();
    cmn = s_min;
    cmx = s_max;
    uint64_t rlo = cmn;
    int bsh = cmx == cmn ? 0 : max(0, 56 - __clzll((long long)(cmx - cmn)));   // (cmx - cmn) >> bsh < 256
    uint32_t m_rem = m, bin = 0, n_in = 0;
    uint64_t width = ~0ull;                                  // extent of the current range [rlo, rlo + width)
    for (int level = 0; level < 8; ++level) {
#pragma unroll 8
        for (int u = 0; u < R && u < r_used; ++u) {
            if (!valid(u)) continue;
            const uint64_t c = comp(u);
            if (c >= rlo && c - rlo < width) atomicAdd(&hs[(uint32_t)((c - rlo) >> bsh)], 1u);
        }
        __syncthreads();
        if (warp == 0) desc_bin_search(hs, m_rem, res);
        __syncthreads();
        bin = res[0];
        m_rem -= res[1];
        n_in = res[2];
        if (tid < 256) hs[tid] = 0u;
        if (n_in <= 32 || bsh == 0) break;
        rlo += (uint64_t)bin << bsh;
        width = 1ull << bsh;                                 // the next level stays inside this bin
        bsh = max(0, bsh - 8);
        __syncthreads();
    }
    // the bin's members (at most 32: a bin of width 1 holds one composite)
    const uint64_t blo = rlo + ((uint64_t)bin << bsh);
#pragma unroll 8
    for (int u = 0; u < R && u < r_used; ++u) {
        if (!valid(u)) continue;
        const uint64_t c = comp(u);
        if (c >= blo && ((c - blo) >> bsh) == 0ull) list[atomicAdd(sh_nin, 1u)] = c;
    }
    __syncthreads();
    if (warp == 0) {
        const uint64_t e = lane < (int)n_in ? list[lane] : 0ull;
        uint32_t gt = 0;
        for (int j = 0; j < (int)n_in; ++j) gt += __shfl_sync(0xffffffffu, e, j) > e ? 1u : 0u;
        if (lane < (int)n_in && gt == m_rem - 1) bc[0] = e;
    }
    __syncthreads();
    *elo = 0ull;
    *ehi = 1ull << 32;
    *cp = bc[0];
    *cm = ~0ull;
    return true;
}

__device__ __forceinline__ bool threshold_selects(uint64_t c, uint64_t elo, uint64_t ehi, uint64_t cp, uint64_t cm)
{
    const uint64_t kk = c >> 32;
    return kk >= ehi || (kk >= elo && (c & cm) >= cp);
}

// Histogram levels over the block's keys (thread item u valid when valid(u)): the range
// [elo, ehi) holding the m-th largest key, `above` keys >= ehi, n_in keys in the range;
// stops once n_in <= cap or the range is one value.  Needs m <= the valid count.
template <int R, typename Valid, typename Key>
__device__ void key_levels(Valid valid, Key key, uint32_t m, uint32_t cap, uint32_t *hs, uint32_t *sh_min,
                           uint32_t *sh_max, uint32_t *res, uint64_t &elo, uint64_t &ehi, uint32_t &above,
                           uint32_t &n_in)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t kmn = 0xFFFFFFFFu, kmx = 0u;
#pragma unroll
    for (int u = 0; u < R; ++u)
        if (valid(u)) {
            kmn = min(kmn, key(u));
            kmx = max(kmx, key(u));
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
        kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
    }
    if (lane == 0) {
        atomicMin(sh_min, kmn);
        atomicMax(sh_max, kmx);
    }
    if (tid < 256) hs[tid] = 0u;
    __syncthreads();
    kmn = *sh_min;
    kmx = *sh_max;
    uint64_t rlo = kmn, width = ~0ull;
    int bsh = max(0, 24 - __clz((int)(kmx - kmn)));
    uint32_t m_rem = m, bin = 0;
    above = 0;
    for (int level = 0; level < 4; ++level) {
#pragma unroll
        for (int u = 0; u < R; ++u) {
            if (!valid(u)) continue;
            const uint64_t kk = key(u);
            if (kk >= rlo && kk - rlo < width) atomicAdd(&hs[(uint32_t)((kk - rlo) >> bsh)], 1u);
        }
        __syncthreads();
        if (warp == 0) desc_bin_search(hs, m_rem, res);
        __syncthreads();
        bin = res[0];
        above += res[1];
        m_rem -= res[1];
        n_in = res[2];
        if (tid < 256) hs[tid] = 0u;
        if (n_in <= cap || bsh == 0) break;
        rlo += (uint64_t)bin << bsh;
        width = 1ull << bsh;
        bsh = max(0, bsh - 8);
        __syncthreads();
    }
    elo = rlo + ((uint64_t)bin << bsh);
    ehi = elo + (1ull << bsh);
    __syncthreads();
}

// The m-th largest composite among a block's dense candidates, threshold form: afterwards a
// candidate c is selected iff c >= *t_out, and exactly m are.  Thread t holds entries
// d0 .. d0 + R - 1 of `total` (cv[u] = key << 32 | ~region, all distinct; every key in
// [klo, khi]; 1 <= m <= total).  One 2048-bin histogram of the keys over [klo, khi] (`h`,
// 2048 words, zeroed by the caller), one block scan from the top bin to the bin b holding
// the m-th largest; b is taken whole when it holds exactly the count still missing, else one
// warp ranks its members (key desc, then region asc) when they are at most 32.  Returns
// false, with nothing decided, when b holds more than 32 candidates (equal keys in bulk):
// the caller then runs the general levels.  `list`: 33 8-byte words; `res`: 3 words;
// `sh_n`: one word.  Needs blockDim.x == kThreads == 512 (4 bins per thread).
template <int R>
__device__ bool dense_exact_threshold(const uint64_t (&cv)[R], uint32_t d0, uint32_t total, uint32_t m, uint32_t klo,
                                      uint32_t khi, uint32_t *h, uint64_t *list, uint32_t *res, uint32_t *scan_ws,
                                      uint32_t *sh_n, uint64_t *t_out)
{
    static_assert(kThreads * 4 == 2048, "4 bins per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t range = khi - klo;
    const int sh = range < 2048u ? 0 : (32 - __clz((int)range)) - 11;       // range >> sh < 2048
    // a key above khi (a NaN score, which the chunk maxima skip) counts in the top bin: the
    // same bin in both passes, so the counts stay exact and no index leaves the histogram
    auto bin_of = [&](uint64_t c) { return min(2047u, ((uint32_t)(c >> 32) - klo) >> sh); };
#pragma unroll
    for (int u = 0; u < R; ++u)
        if (d0 + u < total) atomicAdd(&h[bin_of(cv[u])], 1u);
    __syncthreads();
    // thread t: bins 2047 - 4t down to 2044 - 4t (thread 0 holds the top bins)
    const uint4 q4 = reinterpret_cast<const uint4 *>(h)[kThreads - 1 - tid];
    const uint32_t c[4] = {q4.w, q4.z, q4.y, q4.x};
    const uint32_t s = c[0] + c[1] + c[2] + c[3];
    uint32_t all;
    const uint32_t incl = block_scan_incl1<kThreads>(s, scan_ws, &all);   // the barrier below separates ws uses
    (void)all;
    const uint32_t excl = incl - s;
    if (excl < m && incl >= m) {
        uint32_t run = excl;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (run + c[u] >= m) {
                res[0] = 2047u - 4u * (uint32_t)tid - (uint32_t)u;
                res[1] = run;
                res[2] = c[u];
                break;
            }
            run += c[u];
        }
    }
    if (tid == 0) *sh_n = 0u;
    __syncthreads();
    const uint32_t b = res[0], above = res[1], nb = res[2];
    const uint32_t m_rem = m - above;                                        // 1 <= m_rem <= nb
    if (nb == m_rem) {
        *t_out = (uint64_t)(klo + (b << sh)) << 32;                          // every key of b and above
        return true;
    }
    if (nb > 32u) return false;
#pragma unroll
    for (int u = 0; u < R; ++u)
        if (d0 + u < total && bin_of(cv[u]) == b) list[atomicAdd(sh_n, 1u)] = cv[u];
    __syncthreads();
    if (warp == 0) {
        const uint64_t e = lane < (int)nb ? list[lane] : 0ull;
        uint32_t gt = 0;
        for (int j = 0; j < (int)nb; ++j) gt += __shfl_sync(0xffffffffu, e, j) > e ? 1u : 0u;
        if (lane < (int)nb && gt == m_rem - 1) list[32] = e;
    }
    __syncthreads();
    *t_out = list[32];
    return true;
}

// kSingle: one CTA per row (launched without a cluster; CL = 1), else a cluster of CL CTAs.
// kMaxima: the indexer scan that wrote the scores also wrote chunk_max[row][c], the largest
// score of regions 32c .. 32c+31 (row stride cm_stride, a multiple of 4): the cluster then
// bounds the threshold from those maxima and reads only the chunks that can hold a selected
// region (the other paths when the maxima tie in bulk).
template <bool kSingle, bool kMaxima = false>
__global__ void __launch_bounds__(kThreads, 1)
    topk_cluster_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ q_pos, int k,
                        int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_count,
                        const float *__restrict__ chunk_max, int64_t cm_stride, int gshift)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ uint32_t scan_ws[40];                                         // block scans + select results
    __shared__ uint32_t tot[2];                                              // slice totals (double-buffered)
    __shared__ uint32_t sh_count[2];                                         // tie count, selected count
    __shared__ int sh_bin, sh_q;
    __shared__ uint32_t sh_above, sh_binc, sh_run;
    __shared__ uint32_t slice_tot[kMaxCluster];
    __shared__ uint32_t cand_cnt[kMaxCluster];                               // pushed by every rank
    __shared__ uint64_t mm_ws[2 * kWarps];
    __shared__ uint32_t sh_kmin, sh_kmax, sh_nin;

    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    // kMaxima: this thread's 8 chunk maxima go out with the query position (entries past the
    // row's eligible chunks are masked once the position is known)
    float4 cm_a = make_float4(0.f, 0.f, 0.f, 0.f), cm_b = cm_a;
    if constexpr (kMaxima) {
        if ((int64_t)tid * 8 + 8 <= cm_stride) {
            const float4 *cm4 = reinterpret_cast<const float4 *>(chunk_max + (int64_t)row * cm_stride + tid * 8);
            cm_a = __ldcg(cm4);
            cm_b = __ldcg(cm4 + 1);
        }
    }

    // ---- loads: this thread's group is the CTA's entries tid, tid+512, ... (coalesced)
    const int p = q_pos[row >> gshift];   // rows per query = 2^gshift (the call's KV groups)
    const int64_t part = ((ld + CL - 1) / CL + 31) / 32 * 32;              // whole 32-region chunks
    const int64_t lo = min(ld, (int64_t)rank * part), hi_ld = min(ld, lo + part);
    const float *src = scores + (int64_t)row * ld + lo;
    if (part > kPartMax) {             // the host sizes the cluster so that a part fits
        if (rank == 0 && tid == 0) {
            set_error(kErrTopkInternal);
            sel_count[row] = 0;
        }
        return;
    }
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + kOffKeys);      // [kPadded] staged keys
    auto stage_keys = [&]() {
        const int n_ld = (int)(hi_ld - lo);
        float v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = u * kThreads + tid;
            v[u] = i < n_ld ? __ldcg(src + i) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = u * kThreads + tid;
            if (i < n_ld) keys[padded(i)] = score_key(v[u]);
        }
    };
    if constexpr (!kMaxima) stage_keys();
    const bool valid = p >= 0 && (int64_t)(p / kRegion) <= ld;
    const int64_t own = valid ? p / kRegion : 0;
    const int64_t need = valid ? min((int64_t)(k - 1), own) : 0;
    const int cnt = (int)max((int64_t)0, min(own, hi_ld) - lo);            // this CTA's eligible keys
    const bool trivial = (need == 0 || need == own);
    // this thread's group: CTA entries [tid*32, tid*32 + nmine)
    const int nmine = max(0, min(kPer, cnt - tid * kPer));
    if (tid == 0) {
        sh_kmin = 0xFFFFFFFFu;
        sh_kmax = 0u;
        sh_nin = 0u;
    }
    if (tid < 256) reinterpret_cast<uint32_t *>(smem_raw + kOffHs)[tid] = 0u;
    if (rank == 0) reinterpret_cast<uint4 *>(smem_raw + kOffDense)[tid] = make_uint4(0u, 0u, 0u, 0u);   // 2048 bins
    __syncthreads();                                                        // keys staged
    auto key_at = [&](int i) -> uint32_t { return keys[padded(i)]; };

    // groups holding an eligible entry, over the cluster (the same count in every CTA)
    uint32_t n_groups = 0;
    for (int q = 0; q < CL; ++q) {
        const int64_t lq = min(ld, (int64_t)q * part), hq = min(ld, lq + part);
        const int64_t cq = max((int64_t)0, min(own, hq) - lq);
        n_groups += (uint32_t)((cq + kPer - 1) / kPer);
    }
    bool fast_ok = false;
    uint64_t *dense = reinterpret_cast<uint64_t *>(smem_raw + kOffDense);       // [kDense]
    uint32_t *hw = reinterpret_cast<uint32_t *>(smem_raw + kOffHw);
    uint32_t *hs = reinterpret_cast<uint32_t *>(smem_raw + kOffHs);
    int32_t *out = sel_idx + (int64_t)row * k;
    // after the candidate barrier: the fast-path decision (the same in every CTA from the pushed
    // counts) and, at rank 0, the exact selection among the gathered candidates, emitted in order
    uint64_t *slots = reinterpret_cast<uint64_t *>(smem_raw + kOffSlots);
    auto finish_fast = [&](uint32_t Lk, uint32_t Kmax, int lg_slot, uint32_t slot_n) -> bool {
        // the counts and each rank's first dense entry, in registers (the same in every thread)
        uint32_t first[kMaxCluster];
        uint32_t total = 0;
        bool overflow = false;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) {
            const uint32_t cq = q < CL ? cand_cnt[q] : 0u;
            first[q] = total;
            total += cq;
            overflow |= cq > slot_n;
        }
        const bool fast_ok = !overflow && total >= (uint32_t)need && total <= (uint32_t)kDense;
        if (fast_ok && rank == 0) {
            // ---- dense gather in region order: thread t takes entries [t*kDPer, (t+1)*kDPer);
            // entry d is in the last rank whose first entry is <= d (ranks without candidates
            // share their first entry with the next rank)
            uint64_t cv[kDPer];
            const uint32_t d0 = tid * kDPer;
#pragma unroll
            for (int u = 0; u < kDPer; ++u) {
                const uint32_t d = d0 + u;
                uint32_t base = 0;
#pragma unroll
                for (int q = 0; q < kMaxCluster; ++q)
                    if (q < CL && d >= first[q]) base = ((uint32_t)q << lg_slot) - first[q];
                cv[u] = d < total ? slots[base + d] : 0ull;
            }
            // ---- the need-th largest candidate: every key lies in [Lk, Kmax]
            uint64_t T = 0;
            bool ok = dense_exact_threshold<kDPer>(cv, d0, total, (uint32_t)need, Lk, Kmax,
                                                   reinterpret_cast<uint32_t *>(dense), reinterpret_cast<uint64_t *>(hs),
                                                   scan_ws + 32, scan_ws, &sh_nin, &T);
            if (!ok) {
                // more than 32 candidates in the threshold bin (equal keys in bulk): general levels
                auto valid_u = [&](int u) { return d0 + (uint32_t)u < total; };
                auto comp_u = [&](int u) { return cv[u]; };
                uint64_t elo, ehi, cm;
                __syncthreads();                                            // the bins are read
                ok = block_threshold<kDPer>(valid_u, comp_u, (uint32_t)need, Lk, hs, dense, hw, &sh_kmax, &sh_nin,
                                            scan_ws + 32, mm_ws, &elo, &ehi, &T, &cm);
            }
            if (ok) {
                // ---- ordered emit: the candidates >= T, exactly need of them
                uint32_t cs = 0;
#pragma unroll
                for (int u = 0; u < kDPer; ++u) cs += (d0 + u < total && cv[u] >= T) ? 1u : 0u;
                uint32_t n_sel;
                const uint32_t sincl = block_scan_incl1<kThreads>(cs, scan_ws, &n_sel);   // last use of ws here
                (void)n_sel;
                uint32_t opos = sincl - cs;
#pragma unroll
                for (int u = 0; u < kDPer; ++u) {
                    if (d0 + u < total && cv[u] >= T) {
                        if (opos < (uint32_t)need) out[opos] = (int32_t)(0xFFFFFFFFu - (uint32_t)cv[u]);
                        ++opos;
                    }
                }
                if (tid == kThreads - 1) {
                    if (sincl != (uint32_t)need) set_error(kErrTopkInternal);
                    out[need] = (int32_t)own;                               // own > every eligible region
                    sel_count[row] = (int32_t)(need + 1);
                }
                for (int i = (int)need + 1 + tid; i < k; i += kThreads) out[i] = -1;
            } else {
                // more than kDense candidates share one key: cannot happen with total <= kDense
                if (tid == 0) {
                    set_error(kErrTopkInternal);
                    sel_count[row] = 0;
                }
            }
        }
        return fast_ok;
    };
    if constexpr (kMaxima) {
        bool mfast = false;
        uint32_t Lk = 0;
        const int lg_slot = __ffs(kSlots / CL) - 1;                         // CL is a power of 2
        const uint32_t slot_n = 1u << lg_slot;
        constexpr int kM = 8;                                                // chunk maxima per thread
        const int n_ch = (int)((own + 31) / 32);                             // chunks with an eligible region
        if (!trivial && n_ch >= need && n_ch <= kThreads * kM) {
            // ---- 1. the row's chunk maxima (thread t: chunks [8t, 8t + 8)) and the bound: the
            // lower edge L of a range holding the need-th largest maximum and at most 64 maxima
            uint32_t mk[kM];
            {
                static_assert(kM == 8, "two float4 of chunk maxima per thread");
                const float mv[kM] = {cm_a.x, cm_a.y, cm_a.z, cm_a.w, cm_b.x, cm_b.y, cm_b.z, cm_b.w};
#pragma unroll
                for (int u = 0; u < kM; ++u) mk[u] = tid * kM + u < n_ch ? score_key(mv[u]) : 0u;
            }
            auto mvalid = [&](int u) { return tid * kM + u < n_ch; };
            auto mkey = [&](int u) { return mk[u]; };
            uint64_t elo, ehi;
            uint32_t above, n_in;
            key_levels<kM>(mvalid, mkey, (uint32_t)need, 64u, hs, &sh_kmin, &sh_kmax, scan_ws + 32, elo, ehi, above,
                           n_in);
            const uint32_t Kmax = sh_kmax;                                  // the row's largest maximum
            mfast = n_in <= 64u;                                            // else maxima tie in bulk
            Lk = (uint32_t)elo;
            if (mfast) {
                // ---- 2. this CTA's chunks with maximum >= L, in region order
                uint32_t *list = reinterpret_cast<uint32_t *>(smem_raw + kOffGmax);   // chunk ids
                uint32_t take = 0;
#pragma unroll
                for (int u = 0; u < kM; ++u) {
                    const int64_t c = tid * kM + u;
                    if (mvalid(u) && mk[u] >= Lk && c * 32 >= lo && c * 32 < hi_ld) take |= 1u << u;
                }
                const uint32_t nc = __popc(take);
                uint32_t n_cc_u;
                const uint32_t cincl = block_scan_incl1<kThreads>(nc, scan_ws, &n_cc_u);   // barrier below
                const int n_cc = (int)n_cc_u;
                {
                    uint32_t pos = cincl - nc;
#pragma unroll
                    for (int u = 0; u < kM; ++u)
                        if ((take >> u) & 1u) list[pos++] = (uint32_t)(tid * kM + u);
                }
                __syncthreads();
                // ---- 3. their scores (warp per chunk, 16 chunks of a warp in flight), counted per chunk
                constexpr int kCap = kPadded / 32;                          // chunks that fit the key stage
                const int nst = min(n_cc, kCap);
                uint32_t *ccnt = hw;
                const float *srow = scores + (int64_t)row * ld;
                const int64_t lim = min(own, hi_ld);                        // eligible regions of this CTA
                constexpr int kRound = 16;
                for (int base = warp; base < nst; base += kWarps * kRound) {
                    float v[kRound];
#pragma unroll
                    for (int j = 0; j < kRound; ++j) {
                        const int i = base + kWarps * j;
                        const int64_t r = i < nst ? (int64_t)list[i] * 32 + lane : lim;
                        v[j] = r < lim ? __ldcg(srow + r) : 0.0f;
                    }
#pragma unroll
                    for (int j = 0; j < kRound; ++j) {
                        const int i = base + kWarps * j;
                        if (i < nst) {
                            const int64_t r = (int64_t)list[i] * 32 + lane;
                            const uint32_t key = r < lim ? score_key(v[j]) : 0u;
                            keys[i * 32 + lane] = key;
                            const unsigned m = __ballot_sync(0xffffffffu, key >= Lk && key != 0u);
                            if (lane == 0) ccnt[i] = __popc(m);
                        }
                    }
                }
                __syncthreads();
                // region-order offsets: thread t takes staged chunks [2t, 2t + 2)
                uint32_t cc0 = 2 * tid < nst ? ccnt[2 * tid] : 0u, cc1 = 2 * tid + 1 < nst ? ccnt[2 * tid + 1] : 0u;
                uint32_t cta_total;
                const uint32_t oincl = block_scan_incl1<kThreads>(cc0 + cc1, scan_ws, &cta_total);   // barrier below
                if (2 * tid < nst) ccnt[2 * tid] = oincl - cc0 - cc1;
                if (2 * tid + 1 < nst) ccnt[2 * tid + 1] = oincl - cc1;
                __syncthreads();
                // ---- 4. candidates (key, ~region) into rank 0's slots, counts to every CTA
                uint64_t *dst = reinterpret_cast<uint64_t *>(cluster.map_shared_rank(slots, 0)) +
                                ((size_t)rank << lg_slot);
                const unsigned below = (1u << lane) - 1u;
                for (int i = warp; i < nst; i += kWarps) {
                    const uint32_t key = keys[i * 32 + lane];
                    const bool c = key >= Lk && key != 0u;
                    const unsigned m = __ballot_sync(0xffffffffu, c);
                    const uint32_t off = ccnt[i] + __popc(m & below);
                    if (c && off < slot_n)
                        dst[off] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (list[i] * 32 + (uint32_t)lane));
                }
                // more candidate chunks than the stage holds: report an overflow (every CTA falls back)
                const uint32_t reported = n_cc > kCap ? slot_n + 1 : cta_total;
                if (tid < CL) *cluster.map_shared_rank(&cand_cnt[rank], tid) = reported;
                if (tid == 0) {
                    sh_kmax = 0u;
                    sh_nin = 0u;
                }
                cluster.sync();                                             // candidates and counts in place
                fast_ok = finish_fast(Lk, Kmax, lg_slot, slot_n);
            }
        }
        if (!fast_ok) {
            stage_keys();                                                   // the fallback reads every key
            __syncthreads();
        }
    } else if constexpr (kSingle) {
      if (!trivial) {
        // ---- one CTA holds the row: the exact threshold over its keys directly (entry u of
        // a thread is u*512 + tid, as loaded), emitted in region order through a bitmap
        // the keys stay in smem (read again per pass) to keep registers for the passes
        auto valid_u = [&](int u) { return u * kThreads + tid < cnt; };
        auto comp_u = [&](int u) {
            return ((uint64_t)keys[padded(u * kThreads + tid)] << 32) |
                   (uint64_t)(0xFFFFFFFFu - (uint32_t)(lo + u * kThreads + tid));
        };
        uint32_t kmin = 0xFFFFFFFFu;
#pragma unroll
        for (int u = 0; u < kPer; ++u) kmin = valid_u(u) ? min(kmin, keys[padded(u * kThreads + tid)]) : kmin;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        if (lane == 0) atomicMin(&sh_kmin, kmin);
        __syncthreads();
        uint64_t elo, ehi, cp, cm;
        fast_ok = block_threshold<kPer>(valid_u, comp_u, (uint32_t)need, sh_kmin, hs, dense, hw, &sh_kmax, &sh_nin,
                                        scan_ws + 32, mm_ws, &elo, &ehi, &cp, &cm);
        if (fast_ok) {
            uint32_t *bitmap = hw;                                          // own + 1 <= kPartMax bits
            const int words = (int)((own + 1 + 31) / 32);
            __syncthreads();                                                // hw free again
            for (int i = tid; i < words; i += kThreads) bitmap[i] = 0u;
            __syncthreads();
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                if (valid_u(u) && threshold_selects(comp_u(u), elo, ehi, cp, cm)) {
                    const int r = u * kThreads + tid;                       // lo = 0 with one CTA
                    atomicOr(&bitmap[r >> 5], 1u << (r & 31));
                }
            }
            if (tid == 0) atomicOr(&bitmap[own >> 5], 1u << (own & 31));
            __syncthreads();
            const int wpt = (words + kThreads - 1) / kThreads;
            uint32_t bc = 0;
            for (int i = 0; i < wpt; ++i)
                if (tid * wpt + i < words) bc += __popc(bitmap[tid * wpt + i]);
            const uint32_t bincl = block_scan_incl<kThreads>(bc, scan_ws);
            uint32_t opos = bincl - bc;
            for (int i = 0; i < wpt; ++i) {
                const int w = tid * wpt + i;
                if (w >= words) break;
                uint32_t bits = bitmap[w];
                while (bits) {
                    const int bit = __ffs(bits) - 1;
                    bits &= bits - 1;
                    if (opos < (uint32_t)k) out[opos] = w * 32 + bit;
                    ++opos;
                }
            }
            if (tid == kThreads - 1) {
                if (bincl != (uint32_t)(need + 1)) set_error(kErrTopkInternal);
                sel_count[row] = (int32_t)(need + 1);
            }
            for (int i = (int)need + 1 + tid; i < k; i += kThreads) out[i] = -1;
        }
      }
    } else if (!trivial && (int64_t)n_groups >= need) {
        uint32_t *gmax = reinterpret_cast<uint32_t *>(smem_raw + kOffGmax);
        uint32_t key[kPer];
        {
            const uint4 *run = reinterpret_cast<const uint4 *>(keys + padded(tid * kPer));
#pragma unroll
            for (int j = 0; j < kPer / 4; ++j) {
                const uint4 w = run[j];
                key[4 * j] = w.x;
                key[4 * j + 1] = w.y;
                key[4 * j + 2] = w.z;
                key[4 * j + 3] = w.w;
            }
        }
        // ---- group maximum to every CTA (0 = no eligible entry: below every score key)
        uint32_t gm = 0;
#pragma unroll
        for (int u = 0; u < kPer; ++u) gm = (u < nmine && key[u] > gm) ? key[u] : gm;
        for (int q = 0; q < CL; ++q) cluster.map_shared_rank(gmax, q)[rank * kThreads + tid] = gm;
        cluster.sync();                                                     // all group maxima in place
        // ---- the bound L (the same in every CTA): a 256-bin histogram of the group maxima over
        // [gmin, gmax] with a power-of-two bin width; L is the lower edge of the bin that holds
        // the need-th largest maximum (groups without an eligible entry, maximum 0, take no part)
        uint32_t g8[kMaxCluster];
        uint32_t gmin = 0xFFFFFFFFu, gmx = 0u;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) {
            g8[q] = q < CL ? gmax[q * kThreads + tid] : 0u;
            if (g8[q] != 0u) {
                gmin = min(gmin, g8[q]);
                gmx = max(gmx, g8[q]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
            gmx = max(gmx, __shfl_xor_sync(0xffffffffu, gmx, o));
        }
        if (lane == 0) {
            atomicMin(&sh_kmin, gmin);
            atomicMax(&sh_kmax, gmx);
        }
        __syncthreads();
        gmin = sh_kmin;
        gmx = sh_kmax;
        const int gsh = max(0, 24 - __clz((int)(gmx - gmin)));                // (gmx - gmin) >> gsh < 256
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q)
            if (g8[q] != 0u) atomicAdd(&hs[(g8[q] - gmin) >> gsh], 1u);
        __syncthreads();
        if (warp == 0) desc_bin_search(hs, (uint32_t)need, scan_ws + 32);
        __syncthreads();
        const uint32_t Lk = gmin + (scan_ws[32] << gsh);
        // ---- candidates (key >= L) in region order into rank 0's slots [rank*slot_n, ...),
        // the count to every CTA
        const int lg_slot = __ffs(kSlots / CL) - 1;                         // CL is a power of 2
        const uint32_t slot_n = 1u << lg_slot;
        uint32_t c = 0;
#pragma unroll
        for (int u = 0; u < kPer; ++u) c += (u < nmine && key[u] >= Lk) ? 1u : 0u;
        const uint32_t incl = block_scan_incl<kThreads>(c, scan_ws);
        const uint32_t cta_total = scan_ws[kWarps - 1];
        uint64_t *dst = reinterpret_cast<uint64_t *>(cluster.map_shared_rank(slots, 0)) + ((size_t)rank << lg_slot);
        uint32_t pos = incl - c;
        const uint32_t rbase = 0xFFFFFFFFu - (uint32_t)(lo + tid * kPer);  // ~region of key[0]
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            if (u < nmine && key[u] >= Lk) {
                if (pos < slot_n) dst[pos] = ((uint64_t)key[u] << 32) | (uint64_t)(rbase - (uint32_t)u);
                ++pos;
            }
        }
        if (tid < CL) *cluster.map_shared_rank(&cand_cnt[rank], tid) = cta_total;
        if (tid == 0) {
            sh_kmax = 0u;
            sh_nin = 0u;
        }
        cluster.sync();                                                     // candidates and counts in place
        fast_ok = finish_fast(Lk, gmx, lg_slot, slot_n);
    }
    if (fast_ok) return;               // nothing reads another CTA's smem after the barrier

    // ---- fallback: exact distributed radix select over the staged keys
    uint32_t *hist = reinterpret_cast<uint32_t *>(smem_raw);                 // [2][kBins]
    uint32_t *gsl = hist + 2 * kBins;                                        // [2][kBins] reduced slices
    uint32_t *sl_copy = gsl + 2 * kBins;                                     // [kBins] local copy of a slice


    // ---- distributed radix select of the need-th largest key (fallback and trivial rows)
    uint32_t prefix = 0, pmask = 0;
    uint32_t m_rem = (uint32_t)need;
    bool resolved = (need == 0 || need == own || fast_ok);   // uniform over the cluster
    bool ties_all = true;                            // all keys equal to the prefix are taken
    const int shifts[3] = {20, 8, 0};
    const int widths[3] = {12, 12, 8};
    for (int pass = 0; pass < 3 && !resolved; ++pass) {
        const int sh = shifts[pass], nb = 1 << widths[pass], buf = pass & 1;
        uint32_t *h = hist + buf * kBins;
        uint32_t *gs = gsl + buf * kBins;
        for (int i = tid; i < nb; i += kThreads) h[i] = 0;
        __syncthreads();
        for (int i = tid; i < cnt; i += kThreads) {
            const uint32_t key = key_at(i);
            if ((key & pmask) == prefix) atomicAdd(&h[(key >> sh) & (nb - 1)], 1u);
        }
        cluster.sync();                                                    // local histograms ready
        // reduce this CTA's slice of the bins over the cluster (independent remote loads)
        const int sl = nb / CL, b0 = rank * sl;
        uint32_t part_tot = 0;
        for (int b = tid; b < sl; b += kThreads) {
            uint32_t v[kMaxCluster];
#pragma unroll
            for (int q = 0; q < kMaxCluster; ++q) v[q] = q < CL ? cluster.map_shared_rank(h, q)[b0 + b] : 0u;
            uint32_t s = 0;
#pragma unroll
            for (int q = 0; q < kMaxCluster; ++q) s += v[q];
            gs[b0 + b] = s;
            part_tot += s;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part_tot += __shfl_xor_sync(0xffffffffu, part_tot, o);
        if ((tid & 31) == 0) scan_ws[tid >> 5] = part_tot;
        __syncthreads();
        if (tid == 0) {
            uint32_t t = 0;
            for (int w = 0; w < kThreads / 32; ++w) t += scan_ws[w];
            tot[buf] = t;
        }
        cluster.sync();                                                    // slices and totals ready
        // locate the slice (from the top) holding the m_rem-th largest key, then the bin:
        // the CL totals and the chosen slice are copied in parallel, then a block scan
        if (tid < CL) slice_tot[tid] = cluster.map_shared_rank(tot, tid)[buf];
        __syncthreads();
        if (tid == 0) {
            uint32_t run = 0;
            int qs = CL - 1;
            for (; qs > 0; --qs) {
                if (run + slice_tot[qs] >= m_rem) break;
                run += slice_tot[qs];
            }
            sh_q = qs;
            sh_run = run;
        }
        __syncthreads();
        {
            const int qs = sh_q;
            const uint32_t *rs = cluster.map_shared_rank(gs, qs) + qs * sl;
            for (int b = tid; b < sl; b += kThreads) sl_copy[b] = rs[b];
            __syncthreads();
            // descending over the slice: thread t owns bins [sl-1-t*bpt .. ] in order
            const int bpt = (sl + kThreads - 1) / kThreads;
            const int p0 = tid * bpt;
            uint32_t c = 0;
            for (int u = 0; u < bpt; ++u)
                if (p0 + u < sl) c += sl_copy[sl - 1 - (p0 + u)];
            const uint32_t target = m_rem - sh_run;
            const uint32_t incl = block_scan_incl<kThreads>(c, scan_ws);
            if (incl >= target && incl - c < target) {
                uint32_t run = incl - c;
                for (int u = 0; u < bpt; ++u) {
                    const int b = sl - 1 - (p0 + u);
                    const uint32_t hc = sl_copy[b];
                    if (run + hc >= target) {
                        sh_bin = qs * sl + b;
                        sh_binc = hc;
                        sh_above = sh_run + run;
                        break;
                    }
                    run += hc;
                }
            }
        }
        __syncthreads();
        const int B = sh_bin;
        m_rem -= sh_above;
        prefix |= (uint32_t)B << sh;
        pmask |= (uint32_t)(nb - 1) << sh;
        if (sh_binc == m_rem) resolved = true;          // every key with this prefix is taken
        else if (pass == 2) { resolved = true; ties_all = false; }
        __syncthreads();
    }

    if (!fast_ok) {                                          // uniform over the cluster
        // ---- selection and ordered emit.  Warp w owns the contiguous entries
        // [w*span, (w+1)*span); inside a warp, lane l reads entry base + 32j + l (conflict-free
        // smem), and ballots keep index order.  Equal keys at the exact threshold (when the last
        // digit left more of them than needed) are taken lowest region first: rank by rank, warp
        // by warp, then in ballot order.
        const int span = ((cnt + kWarps - 1) / kWarps + 31) & ~31;
        const int wb = warp * span, we = min(cnt, wb + span);
        const bool take_all = (need == own);
        const bool take_none = (need == 0);
        auto klass = [&](int i) -> int {                         // 2 selected, 1 tie, 0 neither
            if (i >= we) return 0;
            if (take_all) return 2;
            if (take_none) return 0;
            const uint32_t key = key_at(i), km = key & pmask;
            if (km > prefix) return 2;
            if (km != prefix) return 0;
            return ties_all ? 2 : 1;
        };
        uint32_t w_sel = 0, w_tie = 0;
        for (int i = wb + lane; i < wb + span; i += 32) {
            const int c = klass(i);
            if (!__any_sync(0xffffffffu, c != 0)) continue;                 // most groups hold nothing
            w_sel += __popc(__ballot_sync(0xffffffffu, c == 2));
            w_tie += __popc(__ballot_sync(0xffffffffu, c == 1));
        }
        __shared__ uint32_t wsel[kWarps], wtie[kWarps];
        if (lane == 0) {
            wsel[warp] = w_sel;
            wtie[warp] = w_tie;
        }
        __syncthreads();
        uint32_t cta_ties = 0, tie_before_warp = 0;
        for (int w = 0; w < kWarps; ++w) {
            if (w < warp) tie_before_warp += wtie[w];
            cta_ties += wtie[w];
        }
        uint32_t take_here = 0;                                  // ties this CTA takes
        if (!ties_all) {
            if (tid == 0) sh_count[0] = cta_ties;
            cluster.sync();
            uint32_t before = 0;
            for (int q = 0; q < rank; ++q) before += cluster.map_shared_rank(sh_count, q)[0];
            take_here = before >= m_rem ? 0u : min(m_rem - before, cta_ties);
        }
        const uint32_t warp_ties = tie_before_warp >= take_here ? 0u : min(w_tie, take_here - tie_before_warp);
        __syncthreads();
        if (lane == 0) wsel[warp] = w_sel + warp_ties;             // this warp's selected count
        __syncthreads();
        uint32_t warp_off = 0, cta_total = 0;
        for (int w = 0; w < kWarps; ++w) {
            if (w < warp) warp_off += wsel[w];
            cta_total += wsel[w];
        }
        if (tid == 0) sh_count[1] = cta_total;
        cluster.sync();
        uint32_t out_off = 0;
        for (int q = 0; q < rank; ++q) out_off += cluster.map_shared_rank(sh_count, q)[1];
        int32_t *out = sel_idx + (int64_t)row * k;
        uint32_t pos = out_off + warp_off, ties_left = warp_ties;
        const unsigned below = (1u << lane) - 1u;
        for (int i = wb + lane; i < wb + span; i += 32) {
            const int c = klass(i);
            if (!__any_sync(0xffffffffu, c != 0)) continue;
            const unsigned mt = __ballot_sync(0xffffffffu, c == 1);
            const uint32_t tie_rank = __popc(mt & below);
            const bool sel = (c == 2) || (c == 1 && tie_rank < ties_left);
            const unsigned ms = __ballot_sync(0xffffffffu, sel);
            if (sel && pos + __popc(ms & below) < (uint32_t)k) out[pos + __popc(ms & below)] = (int32_t)(lo + i);
            pos += __popc(ms);
            const uint32_t took = min((uint32_t)__popc(mt), ties_left);
            ties_left -= took;
        }
        if (rank == CL - 1) {
            uint32_t total = out_off + cta_total;
            if (valid) {
                if (total != (uint32_t)need && tid == 0) set_error(kErrTopkInternal);
                if (tid == 0) {
                    if (need < k) out[need] = (int32_t)own;        // own > every eligible region
                    sel_count[row] = (int32_t)min(need + 1, (int64_t)k);
                }
                for (int i = (int)need + 1 + tid; i < k; i += kThreads) out[i] = -1;
            } else {
                if (tid == 0) {
                    set_error(kErrTopkRow);
                    sel_count[row] = 0;
                }
                for (int i = tid; i < k; i += kThreads) out[i] = -1;
            }
        }
    }
    cluster.sync();                                          // no CTA leaves while others read its smem
}

}  // namespace topkc
}  // namespace dsa
