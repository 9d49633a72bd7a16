// A4 sparse GQA attention for a few long selections (decode of one or two requests), with
// the split merge inside the kernel ([P1] kwkr.cn/news/601179 §DSA ④; [P3] 100 万 token
// 上下文实测 §一: the hit regions are gathered from the paged cache through the block_table).
//
// A (query, group) row is attended by a cluster of kSplits CTAs; CTA `rank` takes the
// selected regions [32*rank, 32*rank + 32).  Every CTA issues all of its K/V loads at once
// (32 regions x 6 KiB, TMA with the 128-byte swizzle into 16 pair buffers, one mbarrier per
// pair), so a CTA waits for one memory round trip, not one per pair.  Its 8 warps take two
// pairs each: S = Q K^T and O += P V on mma.sync m16n8k16 bf16 with fp32 accumulation and an
// exp2 online softmax, tokens t <= p only.  The warps merge (max, sum, O) in smem and the
// CTA pushes head h of its result into CTA h's inbox through distributed shared memory; after
// one cluster barrier CTA r merges head r of the row from its own inbox (O = sum_c 2^(m_c - M)
// O_c / sum_c 2^(m_c - M) l_c) and writes the bf16 output and the LSE.  No partials in global
// memory, no second kernel.
#pragma once

#include <cooperative_groups.h>

#include "attention.cuh"

namespace dsa {
namespace attnc {

namespace cg = cooperative_groups;
using attn::kPairBytes;
using attn::kQBytes;
using attn::kRegionBytes;
using attn::Params;
using attn::swz;

constexpr int kSplits = 16;                    // CTAs per row (non-portable cluster size)
constexpr int kRegionsPerCta = 32;
constexpr int kPairs = kRegionsPerCta / 2;
constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRow = kD + 8;                   // padded merge row (floats)
constexpr size_t kPairArea = (size_t)kPairs * kPairBytes;                 // 192 KiB
constexpr size_t kMergeO = (size_t)kWarps * 16 * kRow * 4;               // per-warp O for the merge
constexpr size_t kMergeMl = (size_t)kWarps * 16 * 2 * 4;
static_assert(kMergeO + kMergeMl + 16 * kWarps * 4 <= kPairArea, "merge buffers fit in the pair area");
constexpr int kInRow = kD + 4;                 // inbox row per source CTA: O [kD], m, l, pad
constexpr size_t kInbox = (size_t)kSplits * kInRow * 4;                  // outside the pair area
constexpr size_t kSmemBytes = 1024 + kPairArea + kQBytes + 256 + kInbox;
constexpr int kMaxK = kSplits * kRegionsPerCta;                            // 512

__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_cluster_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                               const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *qs = smem + kPairArea;
    uint64_t *bars = reinterpret_cast<uint64_t *>(qs + kQBytes);            // [kPairs]
    float *inbox = reinterpret_cast<float *>(qs + kQBytes + 256);           // [kSplits][kInRow]
    __shared__ int sh_y[kRegionsPerCta], sh_r[kRegionsPerCta], sh_v[kRegionsPerCta];   // per region of the CTA

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int row = blockIdx.y;                                             // query * groups + local group
    const int qi = row >> p.gshift, g = row & ((1 << p.gshift) - 1);
    // the loads that depend on nothing else go out first: the Q tile (into registers, stored
    // to smem once the K/V loads are issued) and this warp's selection entries, beside the
    // selection count
    const __nv_bfloat16 *qsrc = p.q + attn::q_head(p, qi, g) * kD;
    constexpr int kQChunks = 16 * kD / 8;                                   // 384 16-byte chunks
    uint4 qv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int i = tid + u * kThreads;
        if (i < kQChunks) qv[u] = __ldg(reinterpret_cast<const uint4 *>(qsrc + (i / (kD / 8)) * kD + (i % (kD / 8)) * 8));
    }
    auto reg_of = [&](int l) { return (l >> 1) * 16 + 2 * warp + (l & 1); };   // lane l < 4 -> region
    const int j0 = rank * kRegionsPerCta;
    int rr_spec = -1;
    if (lane < 4 && j0 + reg_of(lane) < p.k) rr_spec = p.sel_idx[(int64_t)row * p.k + j0 + reg_of(lane)];
    const int b = p.q_req ? p.q_req[qi] : qi;
    const int pos = p.q_pos[qi];
    const int cnt_raw = p.sel_count[row];
    const int cnt = min(max(cnt_raw, 0), p.k);
    if (cnt != cnt_raw && rank == 0 && tid == 0) set_error(kErrAttnIndex);
    const int nr = max(0, min(kRegionsPerCta, cnt - j0));                   // regions of this CTA
    const bool bad_req = (b < 0 || b >= p.n_req || pos < 0);
    // Warp w owns pairs w and w + 8 (regions 2w, 2w+1, 2w+16, 2w+17 of the CTA): it sets up
    // their barriers, resolves their coordinates (sel_idx -> block_table, lanes 0..3) and
    // issues their TMA loads itself, so the 8 warps issue in parallel.
    if (lane < 2) mbar_init(&bars[warp + 8 * lane], 1);
    fence_mbar_init();
    __syncwarp();
    if (lane < 4) {
        const int j = reg_of(lane);
        int y = 0, r = -1, v = 0;
        if (!bad_req && j < nr) {
            const int rr = rr_spec;
            if (rr < 0 || rr / 8 >= p.max_pages) {
                set_error(kErrAttnIndex);
            } else {
                const int64_t page = p.block_table[(int64_t)b * p.max_pages + rr / 8];
                if (page < 0 || page >= p.n_pages) {
                    set_error(kErrAttnIndex);
                } else {
                    y = (int)(((page << p.gshift) + g) * kPage + (rr % 8) * kRegion);
                    r = rr;
                    v = 1;
                }
            }
        }
        sh_y[j] = y;
        sh_r[j] = r;
        sh_v[j] = v;
        if (warp == 0 && lane == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
    }
    __syncwarp();
    if (lane < 2) {
        const int pr = warp + 8 * lane;
        if (2 * pr < nr) {
            const int va = sh_v[2 * pr], vb = sh_v[2 * pr + 1];
            const unsigned bytes = (va ? 2u * kRegionBytes : 0u) + (vb ? 2u * kRegionBytes : 0u);
            if (bytes == 0) mbar_arrive(&bars[pr]);
            else mbar_arrive_expect_tx(&bars[pr], bytes);
        }
    }
    __syncwarp();
    if (lane < 4) {
        const int j = reg_of(lane), pr = j >> 1, half = j & 1;
        if (sh_v[j]) {
            uint8_t *dst = smem + (size_t)pr * kPairBytes;
            tma_load_3d(dst + half * kRegionBytes, &tmap_k, 0, 0, sh_y[j], &bars[pr]);
            tma_load_3d(dst + (2 + half) * kRegionBytes, &tmap_v, 0, 0, sh_y[j], &bars[pr]);
        }
    }
    // Q tile [16 heads][192] into smem with the K/V tiles' swizzled layout
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int i = tid + u * kThreads;
        if (i < kQChunks) *reinterpret_cast<uint4 *>(qs + swz(i / (kD / 8), (i % (kD / 8)) * 8)) = qv[u];
    }
    __syncthreads();

    // A fragments of Q (16 x 192): 12 k-steps
    uint32_t qa[12][4];
    {
        const uint32_t qbase = smem_u32(qs);
        const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int ks = 0; ks < 12; ++ks) {
            const int c = ks * 16 + 8 * (lane >> 4);
            ldmatrix_x4(qbase + swz(r, c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
        }
    }
    const int gq = lane >> 2, t = lane & 3;
    float o[24][4];
#pragma unroll
    for (int i = 0; i < 24; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.0f, 0.0f};
    const int n_pairs = (nr + 1) / 2;
    bool ok = true;
    for (int pr = warp; pr < n_pairs && ok; pr += kWarps) {
        const int rr[2] = {sh_r[2 * pr], sh_r[2 * pr + 1]};
        const bool rv[2] = {sh_v[2 * pr] != 0, sh_v[2 * pr + 1] != 0};
        ok = mbar_wait(&bars[pr], 0u);
        if (!ok) break;
        const uint32_t kt = smem_u32(smem + (size_t)pr * kPairBytes);
        const uint32_t vt = kt + 2 * kRegionBytes;
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
            const uint32_t tile = kt + nt * kRegionBytes;
            const int r = lane & 7;
#pragma unroll
            for (int kp = 0; kp < 6; ++kp) {       // two k-steps (32 dims) per ldmatrix.x4
                const int c = kp * 32 + 8 * (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(tile + swz(r, c), b0, b1, b2, b3);
                mma_bf16_16816(s[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
                mma_bf16_16816(s[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3],
                               b2, b3);
            }
        }
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 8 * rr[nt] + 2 * t + (e & 1);
                const bool keep = rv[nt] && tok <= pos;
                const float v = keep ? s[nt][e] * p.scale_log2 : -INFINITY;
                s[nt][e] = v;
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
                const float pv = exp2f(s[nt][e] - mref[e >> 1]);
                s[nt][e] = pv;
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
        const uint32_t pa0 = pack_bf16x2(s[0][0], s[0][1]);
        const uint32_t pa1 = pack_bf16x2(s[0][2], s[0][3]);
        const uint32_t pa2 = pack_bf16x2(s[1][0], s[1][1]);
        const uint32_t pa3 = pack_bf16x2(s[1][2], s[1][3]);
        {
            const int r = lane & 7;
            const int reg = (lane >> 3) & 1;
            const int dsub = 8 * (lane >> 4);
#pragma unroll
            for (int nd = 0; nd < 24; nd += 2) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(vt + reg * kRegionBytes + swz(r, nd * 8 + dsub), b0, b1, b2, b3);
                // a region that was not loaded holds stale smem: its P is 0, but 0 * NaN is not
                if (!rv[0]) b0 = b2 = 0u;
                if (!rv[1]) b1 = b3 = 0u;
                mma_bf16_16816(o[nd], pa0, pa1, pa2, pa3, b0, b1);
                mma_bf16_16816(o[nd + 1], pa0, pa1, pa2, pa3, b2, b3);
            }
        }
    }

    // ---- merge the 8 warps into this CTA's (m, l, O) (the pair area is free once every warp
    // is done with its pairs; a warp that gave up on a wait still joins the barriers)
    __syncthreads();
    float *red_o = reinterpret_cast<float *>(smem);                          // [8][16][kRow]
    float *red_ml = red_o + kWarps * 16 * kRow;                              // [8][16][2]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int hr = gq + 8 * h;
        float *rowp = red_o + (warp * 16 + hr) * kRow + 2 * t;
#pragma unroll
        for (int nd = 0; nd < 24; ++nd)
            *reinterpret_cast<float2 *>(rowp + nd * 8) = make_float2(o[nd][2 * h], o[nd][2 * h + 1]);
        if (t == 0) {
            red_ml[(warp * 16 + hr) * 2 + 0] = mrow[h];
            red_ml[(warp * 16 + hr) * 2 + 1] = lrow[h];
        }
    }
    __syncthreads();
    float *wts = red_ml + kWarps * 16 * 2;                                   // [16][8]
    // this CTA's (m, l) of head hr and its O row go to CTA hr's inbox row `rank`
    if (tid < 16) {
        const int hr = tid;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_ml[(w * 16 + hr) * 2]);
        const float Mref = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float wt = exp2f(red_ml[(w * 16 + hr) * 2] - Mref);
            wts[hr * kWarps + w] = wt;
            L += wt * red_ml[(w * 16 + hr) * 2 + 1];
        }
        float *dst = cluster.map_shared_rank(inbox, hr) + rank * kInRow + kD;
        dst[0] = M;
        dst[1] = L;
    }
    __syncthreads();
    for (int e = tid; e < 16 * kD / 4; e += kThreads) {
        const int hr = e / (kD / 4), d = 4 * (e % (kD / 4));
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float4 v = *reinterpret_cast<const float4 *>(red_o + (w * 16 + hr) * kRow + d);
            const float wt = wts[hr * kWarps + w];
            acc.x += wt * v.x;
            acc.y += wt * v.y;
            acc.z += wt * v.z;
            acc.w += wt * v.w;
        }
        *reinterpret_cast<float4 *>(cluster.map_shared_rank(inbox, hr) + rank * kInRow + d) = acc;
    }
    // every CTA's rows are in the inboxes; afterwards no CTA touches another's smem
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");

    // ---- CTA `rank` merges head `rank` of the row from its inbox
    const int hr = rank;
    if (tid < kD) {
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < kSplits; ++c) M = fmaxf(M, inbox[c * kInRow + kD]);
        const float Mref = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f, acc = 0.0f;
#pragma unroll
        for (int c = 0; c < kSplits; ++c) {
            const float wt = exp2f(inbox[c * kInRow + kD] - Mref);
            L += wt * inbox[c * kInRow + kD + 1];
            acc += wt * inbox[c * kInRow + tid];
        }
        const int d = tid;
        const int64_t head = attn::out_head(p, qi, g, hr);
        p.out[head * kD + d] = __float2bfloat16_rn(L > 0.0f ? acc / L : 0.0f);
        if (p.lse && d == 0) p.lse[head] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
}

}  // namespace attnc
}  // namespace dsa
