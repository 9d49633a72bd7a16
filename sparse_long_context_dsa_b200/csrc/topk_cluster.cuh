// A3 top-k region selection, one thread-block cluster per (query, group) row
// ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: a radix-style top-k keeps the best
// regions and always includes the query's own region).
//
// For few long rows (decode: 4 rows of up to 131,071 scores per query) a row is split over
// a cluster of CL CTAs.  CTA `rank` owns the contiguous region range
// [rank*part, rank*part + part) and keeps its order-preserving score keys in smem.  A radix
// select finds the need-th largest key over the whole row: per digit (key bits 31..20,
// 19..8, 7..0) every CTA histograms its keys that match the prefix found so far, the
// cluster sums the histograms through distributed shared memory (each CTA reduces a slice
// of the bins), and every CTA locates the digit from the slice totals.  Equal keys at the
// threshold are taken lowest region first: the ranks own ascending ranges, so a prefix of
// per-rank tie counts says how many ties each CTA takes, and inside a CTA an ordered block
// scan picks the first ones.  The output (ascending region indices) is an ordered
// compaction: each CTA writes its selected regions at the offset given by the counts of the
// ranks before it.  No global scratch, no atomics, no waiting on other CTAs except the
// cluster's hardware barriers.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace dsa {
namespace topkc {

namespace cg = cooperative_groups;

constexpr int kThreads = 512;
constexpr int kPartMax = 16384;        // keys per CTA held in smem (64 KiB)
constexpr int kMaxCluster = 8;         // portable cluster size
constexpr int kBins = 4096;
constexpr int kCandMax = 2048;         // candidates per CTA on the fast path
constexpr int kCandTotal = 4096;       // candidates gathered at rank 0
constexpr int kSample = 4096;          // sampled scores for the lower bound
constexpr size_t kSmemBytes = (size_t)kPartMax * 4 + 5 * kBins * 4 + 1024;
static_assert(kCandMax * 8 <= 2 * kBins * 4 && kCandTotal * 8 <= 2 * kBins * 4 && kSample <= kBins,
              "fast-path buffers fit");

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


// Single-CTA radix select over n smem values (descending): finds the digits of the m-th
// largest value (1 <= m <= n).  Returns (prefix, mask) such that exactly m values v satisfy
// (v & mask) >= prefix.  `h` needs 4096 words, `ws` 40 words.  Values are distinct or the
// caller accepts that all values equal to the m-th are counted (the last digit decides).
template <typename T, int NT, int ND>
__device__ void cta_select_desc(const T *vals, uint32_t n, uint32_t m, const int (&shifts)[ND],
                                const int (&widths)[ND], uint32_t *h, uint32_t *ws, T &prefix_out, T &mask_out)
{
    const int tid = threadIdx.x;
    T prefix = 0, pmask = 0;
    uint32_t m_rem = m;
    for (int d = 0; d < ND; ++d) {
        const int sh = shifts[d], nb = 1 << widths[d];
        for (int i = tid; i < nb; i += NT) h[i] = 0;
        __syncthreads();
        for (uint32_t i = tid; i < n; i += NT) {
            const T v = vals[i];
            if ((v & pmask) == prefix) atomicAdd(&h[(uint32_t)(v >> sh) & (uint32_t)(nb - 1)], 1u);
        }
        __syncthreads();
        // descending scan: thread t owns bins nb-1-t*bpt ... downwards
        const int bpt = (nb + NT - 1) / NT;
        const int p0 = tid * bpt;
        uint32_t c = 0;
        for (int u = 0; u < bpt; ++u)
            if (p0 + u < nb) c += h[nb - 1 - (p0 + u)];
        const uint32_t incl = block_scan_incl<NT>(c, ws);
        if (incl >= m_rem && incl - c < m_rem) {
            uint32_t run = incl - c;
            for (int u = 0; u < bpt; ++u) {
                const int b = nb - 1 - (p0 + u);
                if (run + h[b] >= m_rem) {
                    ws[32] = (uint32_t)b;
                    ws[33] = run;
                    ws[34] = h[b];
                    break;
                }
                run += h[b];
            }
        }
        __syncthreads();
        const uint32_t B = ws[32], above = ws[33], binc = ws[34];
        __syncthreads();
        m_rem -= above;
        prefix |= (T)B << sh;
        pmask |= (T)(nb - 1) << sh;
        if (binc == m_rem) break;
    }
    prefix_out = prefix;
    mask_out = pmask;
}

__global__ void __launch_bounds__(kThreads, 1)
    topk_cluster_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ q_pos, int k,
                        int32_t *__restrict__ sel_idx, int32_t *__restrict__ sel_count)
{
    extern __shared__ uint8_t smem_raw[];
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw);                 // [kPartMax]
    uint32_t *hist = keys + kPartMax;                                        // [2][kBins]
    uint32_t *gsl = hist + 2 * kBins;                                        // [2][kBins] reduced slices
    uint32_t *sl_copy = gsl + 2 * kBins;                                     // [kBins] local copy of a slice
    __shared__ uint32_t scan_ws[40];                                         // block scans + select results
    __shared__ uint32_t tot[2];                                              // slice totals (double-buffered)
    __shared__ uint32_t sh_count[2];                                         // tie count, selected count
    __shared__ int sh_bin, sh_q;
    __shared__ uint32_t sh_above, sh_binc, sh_run;
    __shared__ uint32_t slice_tot[kMaxCluster];
    __shared__ uint32_t sh_ccount, sh_L;
    __shared__ uint32_t off_s[kMaxCluster + 1];

    cg::cluster_group cluster = cg::this_cluster();
    const int CL = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int tid = threadIdx.x;

    const int p = q_pos[row >> 2];
    const bool valid = p >= 0 && (int64_t)(p / kRegion) <= ld;
    const int64_t own = valid ? p / kRegion : 0;
    const int64_t need = valid ? min((int64_t)(k - 1), own) : 0;
    const int64_t part = (own + CL - 1) / CL;
    const int64_t lo = min(own, (int64_t)rank * part), hi = min(own, lo + part);
    const int cnt = (int)(hi - lo);
    const bool in_smem = part <= kPartMax;
    const float *src = scores + (int64_t)row * ld + lo;
    // rank 0 samples every st-th score of the row (for the fast path's lower bound); its
    // loads are issued together with the key loads
    const bool trivial = (need == 0 || need == own);
    const int64_t st = max((int64_t)1, own / kSample);
    const uint32_t ns = (uint32_t)min((int64_t)kSample, (own + st - 1) / st);
    constexpr int kSPer = kSample / kThreads;
    float sv[kSPer];
    if (rank == 0 && !trivial) {
        const float *row_src = scores + (int64_t)row * ld;
#pragma unroll
        for (int u = 0; u < kSPer; ++u) {
            const uint32_t j = u * kThreads + tid;
            sv[u] = j < ns ? __ldcg(row_src + (int64_t)j * st) : 0.0f;
        }
    }
    if (in_smem) {
        // all loads of this thread in flight at once (<= 32 at part <= kPartMax)
        constexpr int kMaxPer = kPartMax / kThreads;
        float v[kMaxPer];
#pragma unroll
        for (int u = 0; u < kMaxPer; ++u) {
            const int i = u * kThreads + tid;
            v[u] = i < cnt ? __ldcg(src + i) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kMaxPer; ++u) {
            const int i = u * kThreads + tid;
            if (i < cnt) keys[i] = score_key(v[u]);
        }
    }
    auto key_at = [&](int i) -> uint32_t { return in_smem ? keys[i] : score_key(__ldcg(src + i)); };

    // ---- fast path: a sampled lower bound L of the threshold, the keys >= L gathered at
    // rank 0, an exact selection among them there.  Used when at least `need` keys are >= L
    // and they fit (uniform decision after a barrier); otherwise the distributed radix
    // select below, which is exact for any input.
    bool fast_ok = false;
    if (!trivial) {
        if (rank == 0) {
            uint32_t *skeys = sl_copy;
#pragma unroll
            for (int u = 0; u < kSPer; ++u) {
                const uint32_t j = u * kThreads + tid;
                if (j < ns) skeys[j] = score_key(sv[u]);
            }
            __syncthreads();
            // the sample rank whose expected row rank is ~1.5 need, plus a margin; the bound
            // is the lower edge of its 12-bit key bin (any bound is fine: the count of keys
            // above it is verified below)
            uint32_t js = (uint32_t)((3 * need + 2 * st - 1) / (2 * st)) + 8;
            js = min(max(js, 1u), ns);
            const int sh1[1] = {20};
            const int wd1[1] = {12};
            uint32_t lp, lm;
            cta_select_desc<uint32_t, kThreads, 1>(skeys, ns, js, sh1, wd1, hist, scan_ws, lp, lm);
            if (tid == 0) sh_L = lp;                      // low 20 bits 0: <= the js-th sample key
        }
        cluster.sync();                                                     // L published
        const uint32_t Lk = *cluster.map_shared_rank(&sh_L, 0);
        uint64_t *clist = reinterpret_cast<uint64_t *>(hist);                // own candidates
        if (tid == 0) sh_ccount = 0;
        __syncthreads();
        for (int i = tid; i < cnt; i += kThreads) {
            const uint32_t key = key_at(i);
            if (key >= Lk) {
                const uint32_t slot = atomicAdd(&sh_ccount, 1u);
                if (slot < (uint32_t)kCandMax)
                    clist[slot] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)(lo + i));
            }
        }
        cluster.sync();                                                     // candidate lists ready
        uint32_t total = 0;
        bool overflow = false;
        for (int q = 0; q < CL; ++q) {
            const uint32_t c = *cluster.map_shared_rank(&sh_ccount, q);
            total += c;
            overflow |= c > (uint32_t)kCandMax;
        }
        fast_ok = !overflow && total >= (uint32_t)need && total <= (uint32_t)kCandTotal;
        if (fast_ok && rank == 0) {
            uint64_t *call = reinterpret_cast<uint64_t *>(gsl);              // all candidates
            if (tid < CL) slice_tot[tid] = *cluster.map_shared_rank(&sh_ccount, tid);
            __syncthreads();
            if (tid == 0) {
                off_s[0] = 0;
                for (int q = 0; q < CL; ++q) off_s[q + 1] = off_s[q] + slice_tot[q];
            }
            __syncthreads();
            const uint32_t n = off_s[CL];
            // one flat parallel copy: entry i of the concatenation comes from rank q
            for (uint32_t i = tid; i < n; i += kThreads) {
                int q = 0;
                while (q + 1 < CL && i >= off_s[q + 1]) ++q;
                const uint64_t *rl = reinterpret_cast<const uint64_t *>(cluster.map_shared_rank(hist, q));
                call[i] = rl[i - off_s[q]];
            }
            __syncthreads();
            const int shc[5] = {52, 40, 32, 10, 0};
            const int wdc[5] = {12, 12, 8, 10, 10};
            uint64_t cp, cm;
            cta_select_desc<uint64_t, kThreads, 5>(call, n, (uint32_t)need, shc, wdc, sl_copy, scan_ws, cp, cm);
            // mark the selection plus the own region in a bitmap (over this CTA's keys, now
            // unused) and emit it in ascending order
            uint32_t *bitmap = keys;
            const int words = (int)((own + 1 + 31) / 32);
            for (int i = tid; i < words; i += kThreads) bitmap[i] = 0;
            __syncthreads();
            for (uint32_t i = tid; i < n; i += kThreads) {
                const uint64_t c = call[i];
                if ((c & cm) >= cp) {
                    const uint32_t r = 0xFFFFFFFFu - (uint32_t)c;
                    if (r < (uint64_t)own) atomicOr(&bitmap[r >> 5], 1u << (r & 31));
                }
            }
            __syncthreads();
            if (tid == 0) atomicOr(&bitmap[own >> 5], 1u << (own & 31));
            __syncthreads();
            const int wpt = (words + kThreads - 1) / kThreads;
            const int w0 = tid * wpt;
            uint32_t c = 0;
            for (int i = 0; i < wpt; ++i)
                if (w0 + i < words) c += __popc(bitmap[w0 + i]);
            const uint32_t incl = block_scan_incl<kThreads>(c, scan_ws);
            int32_t *out = sel_idx + (int64_t)row * k;
            uint32_t pos = incl - c;
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
            if (tid == kThreads - 1) {
                if (incl != (uint32_t)(need + 1)) set_error(kErrTopkInternal);
                sel_count[row] = (int32_t)min((int64_t)incl, (int64_t)k);
            }
            for (int i = (int)need + 1 + tid; i < k; i += kThreads) out[i] = -1;
        }
    }

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
        const int lane = tid & 31, warp = tid >> 5;
        constexpr int kWarps = kThreads / 32;
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
