// A4 sparse GQA attention for prefill chunks with shared selections ([P1] kwkr.cn/news/601179
// §DSA ④; [P5] Stepfun … Step 5 Preview: neighbouring queries reuse one selection).
//
// Queries of one request that sit next to each other select nearly the same regions (the 8
// queries of a region share their own region and score the same summaries).  A CTA takes 8
// consecutive queries of one KV group and streams the UNION of their selections once:
//  * the union is built in smem: every query's ascending selection ORed into a bitmap of the
//    regions, then compacted in region order;
//  * warp 0 resolves each union region through the block table and loads region pairs (K and
//    V, 12 KiB) with TMA (3-D map, 128-byte swizzle) into a ring of kSlots slots, one full and
//    one empty mbarrier per slot, kSlots pairs ahead of its own compute;
//  * compute warp w owns query w of the block (its 16 heads: one 16-row mma.sync tile, the
//    same QK^T / online-softmax / PV code as the per-row kernel).  It walks its own sorted
//    selection beside the union: a region it did not select is masked (-inf), a pair holding
//    none of its regions is skipped, so the result is exactly its own sparse attention;
//  * each warp writes its query's output and LSE; no merge.
// Every K/V byte gathered serves up to 8 queries instead of one.  Queries of different
// requests in one block are served in successive passes (one union per request).  A pass
// whose union is more than twice its longest selection (queries that share little) is not
// streamed: its rows are flagged in row_shared and the per-row kernel, launched next, serves
// them.
#pragma once

#include <climits>

#include "attention.cuh"
#include "topk_cluster.cuh"

namespace dsa {
namespace attns {

using attn::kPairBytes;
using attn::kQBytes;
using attn::kRegionBytes;
using attn::Params;
using attn::swz;

constexpr int kQueries = 8;                          // queries per CTA (one compute warp each)
constexpr int kThreads = 32 * kQueries;              // warp 0 also issues the loads
constexpr int kSlots = 6;                            // region-pair ring
constexpr int kMaxK = 512;                           // selection length per query
constexpr int kMaxUnion = kQueries * kMaxK;          // union length bound
constexpr int kMaxWords = 8192;                      // bitmap words: regions < 262,144
// smem layout (bytes, after 1024-byte alignment)
constexpr size_t kOffRing = 0;
constexpr size_t kOffQ = kOffRing + (size_t)kSlots * kPairBytes;              // [8][16][192] bf16
constexpr size_t kOffBitmap = kOffQ + (size_t)kQueries * kQBytes;              // [kMaxWords]
constexpr size_t kOffUnion = kOffBitmap + (size_t)kMaxWords * 4;               // [kMaxUnion] int32
constexpr size_t kOffSel = kOffUnion + (size_t)kMaxUnion * 4;                  // [8][kMaxK] int32
constexpr size_t kOffBars = kOffSel + (size_t)kQueries * kMaxK * 4;           // full[kSlots], empty[kSlots]
constexpr size_t kOffSlotInfo = kOffBars + 2 * kSlots * 8;                     // [kSlots][2] region ids, -1 = not loaded
constexpr size_t kSmemBytes = 1024 + kOffSlotInfo + kSlots * 2 * 4 + 64;
static_assert(kOffQ % 1024 == 0, "swizzled Q tiles on 1024-byte boundaries");

__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_shared_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                              const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring = smem + kOffRing;
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + kOffBitmap);
    int32_t *uni = reinterpret_cast<int32_t *>(smem + kOffUnion);
    int32_t *sels = reinterpret_cast<int32_t *>(smem + kOffSel);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBars);
    uint64_t *empty = full + kSlots;
    int32_t *slot_reg = reinterpret_cast<int32_t *>(smem + kOffSlotInfo);     // [kSlots][2]
    __shared__ uint32_t scan_ws[40];
    __shared__ int sh_req[kQueries], sh_own[kQueries], sh_cnt[kQueries], sh_pos[kQueries];
    __shared__ int sh_pass_req, sh_max_own, sh_union;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    // group-major block order: the CTAs resident together gather from one group's cache
    const int n_qblocks = (int)gridDim.x / kG;
    const int g = (int)blockIdx.x / n_qblocks;
    const int q0 = ((int)blockIdx.x - g * n_qblocks) * kQueries;
    if (tid == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQueries);
        }
        fence_mbar_init();
    }
    // every query of the block: request, position, own region, selection count (invalid: req -1)
    if (tid < kQueries) {
        const int q = q0 + tid;
        int req = -1, pos = -1, c = 0;
        if (q < p.nq) {
            const int b = p.q_req ? p.q_req[q] : q;
            pos = p.q_pos[q];
            const int craw = p.sel_count[(int64_t)q * kG + g];
            c = min(max(craw, 0), p.k);
            if (c != craw) set_error(kErrAttnIndex);
            if (b < 0 || b >= p.n_req || pos < 0) set_error(kErrAttnIndex);
            else req = b;
        }
        sh_req[tid] = req;
        sh_pos[tid] = pos;
        if (q < p.nq && req < 0 && p.row_shared) p.row_shared[(int64_t)q * kG + g] = 0;   // the per-row kernel flags it
        sh_own[tid] = pos >= 0 ? pos / kRegion : -1;
        sh_cnt[tid] = req >= 0 ? c : 0;
    }
    __syncthreads();
    // this compute warp's query: Q fragments once (the tile goes through smem for ldmatrix)
    const int my_q = q0 + warp;
    const bool compute = warp < kQueries;
    uint32_t qa[12][4];
    if (compute && sh_req[warp] >= 0) {
        uint8_t *qs = smem + kOffQ + (size_t)warp * kQBytes;
        const __nv_bfloat16 *qsrc = p.q + ((int64_t)my_q * kHQ + g * kHeadsPerGroup) * kD;
        for (int i = lane; i < 16 * kD / 8; i += 32) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(qsrc + (i / (kD / 8)) * kD + (i % (kD / 8)) * 8));
            *reinterpret_cast<uint4 *>(qs + swz(i / (kD / 8), (i % (kD / 8)) * 8)) = v;
        }
        __syncwarp();
        const uint32_t qbase = smem_u32(qs);
        const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int ks = 0; ks < 12; ++ks) {
            const int c = ks * 16 + 8 * (lane >> 4);
            ldmatrix_x4(qbase + swz(r, c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
        }
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
    }

    int pair_ctr = 0;                                   // pairs streamed in earlier passes (ring phases)
    uint32_t done = 0;                                  // bit w: query w has had its pass
    for (int pass = 0; pass < kQueries; ++pass) {
        __syncthreads();                                // the previous pass is over: bitmap, union free
        if (tid == 0) {
            int R = INT_MAX, mo = -1;
            for (int w = 0; w < kQueries; ++w)
                if (!((done >> w) & 1u) && sh_req[w] >= 0) R = min(R, sh_req[w]);
            for (int w = 0; w < kQueries; ++w)
                if (sh_req[w] == R) mo = max(mo, sh_own[w]);
            sh_pass_req = R == INT_MAX ? -1 : R;
            sh_max_own = mo;
        }
        __syncthreads();
        const int R = sh_pass_req;
        if (R < 0) break;
        for (int w = 0; w < kQueries; ++w)
            if (sh_req[w] == R) done |= 1u << w;
        const int words = min(kMaxWords, (sh_max_own + 1 + 31) / 32);
        for (int i = tid; i < words; i += kThreads) bitmap[i] = 0u;
        __syncthreads();
        // ---- the union of this pass's selections, in region order
        const bool active = compute && sh_req[warp] == R;
        if (active) {
            const int c = sh_cnt[warp];
            const int32_t *src = p.sel_idx + ((int64_t)my_q * kG + g) * p.k;
            for (int i = lane; i < c; i += 32) {
                int r = src[i];
                if (r < 0 || r > sh_own[warp] || r / 8 >= p.max_pages || (r >> 5) >= words) {
                    set_error(kErrAttnIndex);
                    r = -1;
                }
                sels[warp * kMaxK + i] = r;
                if (r >= 0) atomicOr(&bitmap[r >> 5], 1u << (r & 31));
            }
        }
        __syncthreads();
        {
            const int wpt = (words + kThreads - 1) / kThreads;
            const int w0 = tid * wpt;
            uint32_t n = 0;
            for (int i = 0; i < wpt; ++i)
                if (w0 + i < words) n += __popc(bitmap[w0 + i]);
            const uint32_t incl = topkc::block_scan_incl<kThreads>(n, scan_ws);
            // stream the union only when it is at most twice the longest selection (the queries
            // share most regions); otherwise these rows go to the per-row kernel that runs next,
            // decided before the union is compacted
            int maxc = 0;
            for (int w = 0; w < kQueries; ++w)
                if (sh_req[w] == R) maxc = max(maxc, sh_cnt[w]);
            const uint32_t total = scan_ws[kThreads / 32 - 1];
            if (p.row_shared == nullptr || total <= 2u * (uint32_t)maxc) {
                uint32_t pos = incl - n;
                for (int i = 0; i < wpt; ++i) {
                    if (w0 + i >= words) break;
                    uint32_t b = bitmap[w0 + i];
                    while (b) {
                        const int bit = __ffs(b) - 1;
                        b &= b - 1;
                        if (pos < (uint32_t)kMaxUnion) uni[pos] = (w0 + i) * 32 + bit;
                        ++pos;
                    }
                }
            }
            if (tid == kThreads - 1) sh_union = (int)min(incl, (uint32_t)kMaxUnion);
        }
        __syncthreads();
        int maxc = 0;
        for (int w = 0; w < kQueries; ++w)
            if (sh_req[w] == R) maxc = max(maxc, sh_cnt[w]);
        const bool share = p.row_shared == nullptr || sh_union <= 2 * maxc;
        if (active && lane == 0 && p.row_shared) p.row_shared[(int64_t)my_q * kG + g] = share ? 1 : 0;
        const int U = share ? sh_union : 0;
        const int n_pairs = (U + 1) / 2;

        // warp 0: issue pair pi of this pass into its slot (waits until the 8 warps released it)
        auto issue = [&](int pi) {
            const int it = pair_ctr + pi, s = it % kSlots;
            const unsigned ph = (unsigned)(it / kSlots) & 1u;
            int y = 0, ok = 0, rg = -1;
            if (lane < 2 && 2 * pi + lane < U) {
                rg = uni[2 * pi + lane];
                const int64_t page = p.block_table[(int64_t)R * p.max_pages + rg / 8];
                if (page < 0 || page >= p.n_pages) {
                    set_error(kErrAttnIndex);
                } else {
                    y = (int)((page * kG + g) * kPage + (rg % 8) * kRegion);
                    ok = 1;
                }
            }
            mbar_wait(&empty[s], ph ^ 1u);
            if (lane < 2) slot_reg[2 * s + lane] = ok ? rg : -1;
            const int ok0 = __shfl_sync(0xffffffffu, ok, 0), ok1 = __shfl_sync(0xffffffffu, ok, 1);
            __syncwarp();
            if (lane == 0) {
                const unsigned bytes = (unsigned)(ok0 + ok1) * 2u * kRegionBytes;
                if (bytes == 0) mbar_arrive(&full[s]);
                else mbar_arrive_expect_tx(&full[s], bytes);
            }
            __syncwarp();
            if (lane < 2 && ok) {
                uint8_t *dst = ring + (size_t)s * kPairBytes;
                tma_load_3d(dst + lane * kRegionBytes, &tmap_k, 0, 0, y, &full[s]);
                tma_load_3d(dst + (2 + lane) * kRegionBytes, &tmap_v, 0, 0, y, &full[s]);
            }
        };
        if (warp == 0)
            for (int pi = 0; pi < min(kSlots, n_pairs); ++pi) issue(pi);
        {
            // ---------------- compute warp: its query over the union, unselected regions masked
            const int c = active ? sh_cnt[warp] : 0;
            const int pos = sh_pos[warp];
            const int32_t *msel = sels + warp * kMaxK;
            int ptr = 0;                                // walks this query's selection beside the union
            const int gq = lane >> 2, t = lane & 3;
            float o[24][4];
#pragma unroll
            for (int i = 0; i < 24; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
            float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.0f, 0.0f};
            bool ok = true;
            for (int pi = 0; pi < n_pairs; ++pi) {
                const int it = pair_ctr + pi, s = it % kSlots;
                const unsigned ph = (unsigned)(it / kSlots) & 1u;
                ok = mbar_wait(&full[s], ph);
                if (!ok) break;
                if (active) {
                    const int u0 = uni[2 * pi], u1 = 2 * pi + 1 < U ? uni[2 * pi + 1] : -1;
                    while (ptr < c && msel[ptr] < u0) ++ptr;
                    const bool m0 = ptr < c && msel[ptr] == u0;
                    bool m1 = false;
                    if (u1 >= 0) {
                        while (ptr < c && msel[ptr] < u1) ++ptr;
                        m1 = ptr < c && msel[ptr] == u1;
                    }
                    const int rr[2] = {u0, u1};
                    const bool rv[2] = {m0 && slot_reg[2 * s] >= 0, m1 && slot_reg[2 * s + 1] >= 0};
                    if (rv[0] || rv[1]) {
                        const uint32_t kt = smem_u32(ring + (size_t)s * kPairBytes);
                        const uint32_t vt = kt + 2 * kRegionBytes;
                        float sc[2][4];
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt) {
                            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
                            const uint32_t tile = kt + nt * kRegionBytes;
                            const int r = lane & 7;
#pragma unroll
                            for (int kp = 0; kp < 6; ++kp) {   // two k-steps (32 dims) per ldmatrix.x4
                                const int cc = kp * 32 + 8 * (lane >> 3);
                                uint32_t b0, b1, b2, b3;
                                ldmatrix_x4(tile + swz(r, cc), b0, b1, b2, b3);
                                mma_bf16_16816(sc[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0,
                                               b1);
                                mma_bf16_16816(sc[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2],
                                               qa[2 * kp + 1][3], b2, b3);
                            }
                        }
                        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int tok = 8 * rr[nt] + 2 * t + (e & 1);
                                const bool keep = rv[nt] && tok <= pos;
                                const float v = keep ? sc[nt][e] * p.scale_log2 : -INFINITY;
                                sc[nt][e] = v;
                                mx[e >> 1] = fmaxf(mx[e >> 1], v);
                            }
                        // lazy rescaling: the reference max mrow moves only when a block's max exceeds it by
                        // more than kSlack (log2 units; P stays below 2^kSlack): the same softmax, rarely rescaled
                        float alpha[2], mref[2];
                        bool grow_any = false;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                            const bool grow = mx[h] > mrow[h] + attn::kSlack;
                            alpha[h] = grow ? exp2f(mrow[h] - mx[h]) : 1.0f;
                            if (grow) mrow[h] = mx[h];
                            grow_any |= grow;
                            mref[h] = (mrow[h] == -INFINITY) ? 0.0f : mrow[h];
                        }
                        float ps[2] = {0.0f, 0.0f};
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float pv = exp2f(sc[nt][e] - mref[e >> 1]);
                                sc[nt][e] = pv;
                                ps[e >> 1] += pv;
                            }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], 1);
                            ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], 2);
                            lrow[h] = lrow[h] * alpha[h] + ps[h];
                        }
                        if (__any_sync(0xffffffffu, grow_any)) {
#pragma unroll
                            for (int nd = 0; nd < 24; ++nd) {
                                o[nd][0] *= alpha[0];
                                o[nd][1] *= alpha[0];
                                o[nd][2] *= alpha[1];
                                o[nd][3] *= alpha[1];
                            }
                        }
                        const uint32_t pa0 = pack_bf16x2(sc[0][0], sc[0][1]);
                        const uint32_t pa1 = pack_bf16x2(sc[0][2], sc[0][3]);
                        const uint32_t pa2 = pack_bf16x2(sc[1][0], sc[1][1]);
                        const uint32_t pa3 = pack_bf16x2(sc[1][2], sc[1][3]);
                        const int r = lane & 7;
                        const int reg = (lane >> 3) & 1;
                        const int dsub = 8 * (lane >> 4);
#pragma unroll
                        for (int nd = 0; nd < 24; nd += 2) {
                            uint32_t b0, b1, b2, b3;
                            ldmatrix_x4_trans(vt + reg * kRegionBytes + swz(r, nd * 8 + dsub), b0, b1, b2, b3);
                            // a masked region's slot may hold another region or stale smem: its P is
                            // 0, but 0 * NaN is not
                            if (!rv[0]) b0 = b2 = 0u;
                            if (!rv[1]) b1 = b3 = 0u;
                            mma_bf16_16816(o[nd], pa0, pa1, pa2, pa3, b0, b1);
                            mma_bf16_16816(o[nd + 1], pa0, pa1, pa2, pa3, b2, b3);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (warp == 0 && pi + kSlots < n_pairs) issue(pi + kSlots);
            }
            if (active) {
                // ---- this query's output: O / L per head, LSE
                const int64_t obase = ((int64_t)my_q * kHQ + g * kHeadsPerGroup) * kD;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int hr = gq + 8 * h;
                    const float L = lrow[h];
                    const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
#pragma unroll
                    for (int nd = 0; nd < 24; ++nd)
                        *reinterpret_cast<__nv_bfloat162 *>(p.out + obase + (int64_t)hr * kD + nd * 8 + 2 * t) =
                            __floats2bfloat162_rn(o[nd][2 * h] * inv, o[nd][2 * h + 1] * inv);
                    if (p.lse && t == 0)
                        p.lse[(int64_t)my_q * kHQ + g * kHeadsPerGroup + hr] =
                            (L > 0.0f) ? (mrow[h] + log2f(L)) * 0.69314718055994531f : -INFINITY;
                }
            }
            (void)ok;
        }
        pair_ctr += n_pairs;
    }
}

}  // namespace attns
}  // namespace dsa
