// A4 sparse GQA attention over the selected regions ([P1] kwkr.cn/news/601179 §DSA ④: only
// the selected regions' real K/V are attended; [P3] 100 万 token 上下文实测 §一: the hit
// regions are gathered from the paged cache through the block_table).
//
// One CTA per (query, group, split of the selection).  The 16 query heads of a group share
// the group's K/V, so each CTA is a 16-row attention tile:
//  * a region is 8 contiguous token rows of one page (3 KiB of K and 3 KiB of V); each warp
//    streams its regions, two at a time, with TMA (3-D tensor map: 64-element column blocks
//    x 3 x rows, 128-byte swizzle, no multicast) into a per-warp double-buffered ring;
//  * S = Q K^T and O += P V run on mma.sync m16n8k16 bf16 (fp32 accumulate), K/V fragments
//    via conflict-free ldmatrix (.trans for V), online softmax in fp32 with exp2;
//  * the causal mask keeps tokens t <= p (it only bites inside the own region);
//  * the 4 warps of a CTA merge their (max, sum, O) in smem; with one split per row the
//    CTA writes the bf16 output, otherwise a partial that combine_kernel merges (LSE).
#pragma once

#include "common.cuh"

namespace dsa {
namespace attn {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kRegionBytes = kRegion * kD * 2;          // 3 KiB
constexpr int kPairBytes = 4 * kRegionBytes;            // K,V of 2 regions: 12 KiB
constexpr int kSlots = 2;                               // pair slots per warp
constexpr int kWarpRing = kSlots * kPairBytes;          // 24 KiB
constexpr int kQBytes = 16 * kD * 2;                    // 6 KiB
constexpr size_t kSmemBytes = 1024 + (size_t)kWarps * kWarpRing + kQBytes + 64;
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
    const __nv_bfloat16 *q;
    const int32_t *block_table;
    const int32_t *q_req;      // nullptr: identity (decode)
    const int32_t *q_pos;
    const int32_t *sel_idx;
    const int32_t *sel_count;
    __nv_bfloat16 *out;
    float *lse;                // may be null
    float *part_o;             // [rows][n_splits][16][192]   (split mode)
    float *part_ml;            // [rows][n_splits][16][2]
    int64_t n_pages;
    int max_pages;
    int n_req;
    int nq;
    int k;
    int rps;                   // regions per split
    int n_splits;
    float scale_log2;          // log2(e) / sqrt(192)
};

// byte offset of element (row, col) in a [rows][3][64] bf16 tile written by TMA with the
// 128-byte swizzle: 16-byte chunk index XOR (128-byte line index & 7)
__device__ __forceinline__ uint32_t swz(int row, int col)
{
    const int blk = col >> 6, c16 = (col & 63) >> 3, line = row * 3 + blk;
    return (uint32_t)(line * 128 + ((c16 ^ (line & 7)) << 4) + (col & 7) * 2);
}

__global__ void __launch_bounds__(kThreads, 2)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                       const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *qs = smem + kWarps * kWarpRing;
    uint64_t *bars = reinterpret_cast<uint64_t *>(qs + kQBytes);   // [kWarps][kSlots]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int row = blockIdx.y;            // query * 4 + group
    const int qi = row >> 2, g = row & 3;
    const int b = p.q_req ? p.q_req[qi] : qi;
    const int pos = p.q_pos[qi];
    const int cnt_raw = p.sel_count[row];
    const int cnt = min(max(cnt_raw, 0), p.k);   // never index past the row of sel_idx
    if (cnt != cnt_raw && split == 0 && threadIdx.x == 0) set_error(kErrAttnIndex);
    const int j0 = split * p.rps;
    const int nr = min(p.rps, cnt - j0);   // regions of this CTA
    if (nr <= 0 && p.n_splits > 1) return; // combine_kernel ignores empty splits
    const bool bad_req = (b < 0 || b >= p.n_req || pos < 0);

    if (threadIdx.x < kWarps * kSlots) mbar_init(&bars[threadIdx.x], 1);
    // Q tile [16 heads][192] into smem with the same swizzled layout as the K/V tiles
    const __nv_bfloat16 *qsrc = p.q + ((int64_t)qi * kHQ + g * kHeadsPerGroup) * kD;
    for (int i = threadIdx.x; i < 16 * kD / 8; i += kThreads) {
        const int r = i / (kD / 8), c = (i % (kD / 8)) * 8;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(qsrc + r * kD + c));
        *reinterpret_cast<uint4 *>(qs + swz(r, c)) = v;
    }
    fence_mbar_init();
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

    const int n_pairs = (max(nr, 0) + 1) >> 1;
    uint8_t *ring = smem + warp * kWarpRing;
    uint64_t *wbar = bars + warp * kSlots;
    const int32_t *sel = p.sel_idx + (int64_t)row * p.k + j0;

    // region validity / tensor row of pair slot regions, decided by lane 0, broadcast
    auto region_row = [&](int j, int &yrow) -> bool {
        if (bad_req || j >= nr) return false;
        const int r = sel[j];
        if (r < 0 || r / 8 >= p.max_pages) {
            set_error(kErrAttnIndex);
            return false;
        }
        const int64_t page = p.block_table[(int64_t)b * p.max_pages + r / 8];
        if (page < 0 || page >= p.n_pages) {
            set_error(kErrAttnIndex);
            return false;
        }
        yrow = (int)((page * kG + g) * kPage + (r % 8) * kRegion);
        return true;
    };
    auto issue = [&](int pi, int slot) {
        // lane 0 only: load K and V of regions 2pi and 2pi+1 of this warp's pair pi
        uint8_t *dst = ring + slot * kPairBytes;
        int y0 = 0, y1 = 0;
        const int ja = 2 * pi, jb = 2 * pi + 1;
        const bool va = region_row(ja, y0), vb = region_row(jb, y1);
        const unsigned bytes = (va ? 2u * kRegionBytes : 0u) + (vb ? 2u * kRegionBytes : 0u);
        if (bytes == 0) {
            mbar_arrive(&wbar[slot]);
            return;
        }
        mbar_arrive_expect_tx(&wbar[slot], bytes);
        if (va) {
            tma_load_3d(dst, &tmap_k, 0, 0, y0, &wbar[slot]);
            tma_load_3d(dst + 2 * kRegionBytes, &tmap_v, 0, 0, y0, &wbar[slot]);
        }
        if (vb) {
            tma_load_3d(dst + kRegionBytes, &tmap_k, 0, 0, y1, &wbar[slot]);
            tma_load_3d(dst + 3 * kRegionBytes, &tmap_v, 0, 0, y1, &wbar[slot]);
        }
    };

    // this warp handles pairs warp, warp + 4, ...
    int my_pairs = 0;
    for (int pi = warp; pi < n_pairs; pi += kWarps) ++my_pairs;
    if (lane == 0) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
        for (int s = 0; s < kSlots && s < my_pairs; ++s) issue(warp + s * kWarps, s);
    }

    for (int i = 0; i < my_pairs; ++i) {
        const int pi = warp + i * kWarps;
        const int slot = i % kSlots;
        const unsigned ph = (unsigned)(i / kSlots) & 1u;
        if (!mbar_wait(&wbar[slot], ph)) break;
        const uint32_t kt = smem_u32(ring + slot * kPairBytes);
        const uint32_t vt = kt + 2 * kRegionBytes;

        // validity of the 16 tokens: region ja = 2pi (n-tile 0), jb = 2pi+1 (n-tile 1)
        int rr[2];
        bool rv[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * pi + h;
            rv[h] = false;
            rr[h] = -1;
            if (!bad_req && j < nr) {
                const int r = sel[j];
                // same checks as the loader (without flagging twice)
                if (r >= 0 && r / 8 < p.max_pages) {
                    const int64_t page = p.block_table[(int64_t)b * p.max_pages + r / 8];
                    if (page >= 0 && page < p.n_pages) {
                        rv[h] = true;
                        rr[h] = r;
                    }
                }
            }
        }

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
        // scale, mask, online softmax (rows gq and gq+8 of this lane)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 8 * rr[nt] + 2 * t + (e & 1);
                const bool ok = rv[nt] && tok <= pos;
                const float v = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
                s[nt][e] = v;
                mx[e >> 1] = fmaxf(mx[e >> 1], v);
            }
        float alpha[2], mref[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            const float mnew = fmaxf(mrow[h], mx[h]);
            mref[h] = (mnew == -INFINITY) ? 0.0f : mnew;
            alpha[h] = exp2f(mrow[h] - mref[h]);
            mrow[h] = mnew;
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
#pragma unroll
        for (int nd = 0; nd < 24; ++nd) {
            o[nd][0] *= alpha[0];
            o[nd][1] *= alpha[0];
            o[nd][2] *= alpha[1];
            o[nd][3] *= alpha[1];
        }
        // P (16 x 16 tokens) as the A operand, straight from the S accumulators
        const uint32_t pa0 = pack_bf16x2(s[0][0], s[0][1]);
        const uint32_t pa1 = pack_bf16x2(s[0][2], s[0][3]);
        const uint32_t pa2 = pack_bf16x2(s[1][0], s[1][1]);
        const uint32_t pa3 = pack_bf16x2(s[1][2], s[1][3]);
        {
            // ldmatrix.x4.trans: matrices (region 0, dims 8nd..), (region 1, dims 8nd..),
            // (region 0, dims 8nd+8..), (region 1, dims 8nd+8..); lane l -> token row l&7
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
        __syncwarp();
        const int next = i + kSlots;
        if (next < my_pairs && lane == 0) {
            fence_proxy_async();
            issue(warp + next * kWarps, slot);
        }
    }

    // ---- merge the 4 warps: write (m, l, O) of each warp to smem (reusing the rings)
    __syncthreads();
    float *red_o = reinterpret_cast<float *>(smem);                      // [4][16][192]
    float *red_ml = red_o + kWarps * 16 * kD;                            // [4][16][2]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int hr = gq + 8 * h;
#pragma unroll
        for (int nd = 0; nd < 24; ++nd) {
            float *dst = red_o + ((warp * 16 + hr) * kD) + nd * 8 + 2 * t;
            dst[0] = o[nd][2 * h];
            dst[1] = o[nd][2 * h + 1];
        }
        if (t == 0) {
            red_ml[(warp * 16 + hr) * 2 + 0] = mrow[h];
            red_ml[(warp * 16 + hr) * 2 + 1] = lrow[h];
        }
    }
    __syncthreads();
    // thread -> (head hr, 24 consecutive dims)
    {
        const int hr = threadIdx.x >> 3;              // 16 heads x 8 threads
        const int d0 = (threadIdx.x & 7) * 24;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_ml[(w * 16 + hr) * 2]);
        const float Mref = (M == -INFINITY) ? 0.0f : M;
        float wgt[kWarps], L = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            wgt[w] = exp2f(red_ml[(w * 16 + hr) * 2] - Mref);
            L += wgt[w] * red_ml[(w * 16 + hr) * 2 + 1];
        }
        const int head = g * kHeadsPerGroup + hr;
        if (p.n_splits == 1) {
            const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
            __nv_bfloat16 *dst = p.out + ((int64_t)qi * kHQ + head) * kD + d0;
#pragma unroll
            for (int d = 0; d < 24; d += 2) {
                float a = 0.0f, c = 0.0f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) {
                    a += wgt[w] * red_o[(w * 16 + hr) * kD + d0 + d];
                    c += wgt[w] * red_o[(w * 16 + hr) * kD + d0 + d + 1];
                }
                *reinterpret_cast<__nv_bfloat162 *>(dst + d) = __floats2bfloat162_rn(a * inv, c * inv);
            }
            if (p.lse && (threadIdx.x & 7) == 0)
                p.lse[(int64_t)qi * kHQ + head] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
        } else {
            const int64_t pidx = ((int64_t)row * p.n_splits + split) * 16 + hr;
            float *dst = p.part_o + pidx * kD + d0;
#pragma unroll
            for (int d = 0; d < 24; ++d) {
                float a = 0.0f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) a += wgt[w] * red_o[(w * 16 + hr) * kD + d0 + d];
                dst[d] = a;
            }
            if ((threadIdx.x & 7) == 0) {
                p.part_ml[pidx * 2 + 0] = M;
                p.part_ml[pidx * 2 + 1] = L;
            }
        }
    }
}

// Merges the per-split partials of one (query, head): O = sum_s 2^(m_s - M) O_s / L.
__global__ void __launch_bounds__(kD) combine_kernel(const Params p)
{
    const int row = blockIdx.x >> 4, hr = blockIdx.x & 15;
    const int qi = row >> 2, g = row & 3;
    const int d = threadIdx.x;
    const int cnt = min(max(p.sel_count[row], 0), p.k);
    const int ns = min(p.n_splits, (cnt + p.rps - 1) / p.rps);
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, p.part_ml[(((int64_t)row * p.n_splits + s) * 16 + hr) * 2]);
    const float Mref = (M == -INFINITY) ? 0.0f : M;
    float L = 0.0f, acc = 0.0f;
    for (int s = 0; s < ns; ++s) {
        const int64_t pidx = ((int64_t)row * p.n_splits + s) * 16 + hr;
        const float w = exp2f(p.part_ml[pidx * 2] - Mref);
        L += w * p.part_ml[pidx * 2 + 1];
        acc += w * p.part_o[pidx * kD + d];
    }
    const int head = g * kHeadsPerGroup + hr;
    p.out[((int64_t)qi * kHQ + head) * kD + d] = __float2bfloat16_rn(L > 0.0f ? acc / L : 0.0f);
    if (p.lse && d == 0) p.lse[(int64_t)qi * kHQ + head] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace attn
}  // namespace dsa
