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
constexpr float kSlack = 8.0f;                          // lazy-rescale slack of the running max (log2 units)

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
    uint8_t *row_shared;       // nullable [nq][4]: 1 = the row was served by the shared-selection kernel
    int window;                // 0: the selection (sel_idx, sel_count); > 0: the last `window` tokens
    int64_t n_pages;
    int max_pages;
    int n_req;
    int nq;
    int k;
    int rps;                   // regions per split
    int n_splits;
    float scale_log2;          // log2(e) / sqrt(192)
    // KV groups held by this call: groups g0 .. g0 + 2^gshift - 1 (all four: g0 = 0, gshift = 2).
    // Rows are (query, local group gl); K/V caches hold only these groups ([pages][ng][64][192]),
    // q is the full [nq][64][192] and out / lse hold the local groups' heads ([nq][16 ng][192]).
    int gshift;
    int g0;
    // window decode with the append folded in (nullable): query q's token at q_pos[q], K and V
    // rows new_k / new_v [nq][4][192], is written to its cache slot and attended from these rows
    const __nv_bfloat16 *new_k;
    const __nv_bfloat16 *new_v;
    __nv_bfloat16 *k_cache;    // the caches the rows go to (with new_k)
    __nv_bfloat16 *v_cache;
};

// Index of head hr of local group gl of query qi in out / lse ([nq][16 << gshift]).
__device__ __forceinline__ int64_t out_head(const Params &p, int qi, int gl, int hr)
{
    return ((int64_t)qi << (p.gshift + 4)) + gl * kHeadsPerGroup + hr;
}

// First Q head of local group gl of query qi in the full q [nq][64][192].
__device__ __forceinline__ int64_t q_head(const Params &p, int qi, int gl)
{
    return (int64_t)qi * kHQ + (p.g0 + gl) * kHeadsPerGroup;
}

// byte offset of element (row, col) in a [rows][3][64] bf16 tile written by TMA with the
// 128-byte swizzle: 16-byte chunk index XOR (128-byte line index & 7)
__device__ __forceinline__ uint32_t swz(int row, int col)
{
    const int blk = col >> 6, c16 = (col & 63) >> 3, line = row * 3 + blk;
    return (uint32_t)(line * 128 + ((c16 ^ (line & 7)) << 4) + (col & 7) * 2);
}

// The rows' regions: the selection, or (window mode) the regions holding tokens
// max(0, pos - window + 1) .. pos, whose first token is the window's lower bound.
__device__ __forceinline__ int window_lo(const Params &p, int pos)
{
    return p.window > 0 ? max(0, pos - p.window + 1) : 0;
}

__device__ __forceinline__ int row_count(const Params &p, int row, int pos, bool &bad)
{
    if (p.window > 0) {
        bad = false;
        return pos < 0 ? 0 : (pos >> 3) - (window_lo(p, pos) >> 3) + 1;   // <= p.k (host-checked)
    }
    const int raw = p.sel_count[row];
    const int c = min(max(raw, 0), p.k);     // never index past the row of sel_idx
    bad = c != raw;
    return c;
}

__global__ void __launch_bounds__(kThreads, 2)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                       const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    // the tensor maps are kernel parameters: their descriptors are fetched while the previous
    // kernel finishes, not in front of the first loads
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
    }
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *qs = smem + kWarps * kWarpRing;
    uint64_t *bars = reinterpret_cast<uint64_t *>(qs + kQBytes);   // [kWarps][kSlots]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // block order: split-major, then group, then query, so that the CTAs resident together
    // gather from one group's (and one split's) share of the cache and reuse it in L2
    const int rows = p.nq << p.gshift;
    const int split = (int)blockIdx.x / rows;
    const int rem = (int)blockIdx.x - split * rows;
    const int g = rem / p.nq, qi = rem - g * p.nq;      // g: local group
    const int row = (qi << p.gshift) + g;  // query * groups + local group
    if (p.row_shared && p.row_shared[row]) return;
    const int b = p.q_req ? p.q_req[qi] : qi;
    const int pos = p.q_pos[qi];
    bool bad_cnt;
    const int cnt = row_count(p, row, pos, bad_cnt);
    if (bad_cnt && split == 0 && threadIdx.x == 0) set_error(kErrAttnIndex);
    const int t_lo = window_lo(p, pos);         // tokens below it are masked (window mode)
    const int j0 = split * p.rps;
    const int nr = min(p.rps, cnt - j0);   // regions of this CTA
    if (nr <= 0 && p.n_splits > 1) return; // combine_kernel ignores empty splits
    const bool bad_req = (b < 0 || b >= p.n_req || pos < 0);
    if (threadIdx.x < kWarps * kSlots) mbar_init(&bars[threadIdx.x], 1);

    const int n_pairs = (max(nr, 0) + 1) >> 1;
    uint8_t *ring = smem + warp * kWarpRing;
    uint64_t *wbar = bars + warp * kSlots;
    const int32_t *sel = p.window > 0 ? nullptr : p.sel_idx + (int64_t)row * p.k + j0;

    // This warp handles pairs warp, warp + 4, ...; its local region q (pair q/2, half q%2)
    // is region j = 2*(warp + 4*(q/2)) + q%2 of the CTA.  Lanes resolve the coordinates of
    // 32 local regions at a time (sel_idx, then block_table) in parallel and keep them in
    // registers; the issuing code reads them with shuffles and records, per ring slot, the
    // region ids and validity the compute side needs.
    int my_pairs = 0;
    for (int pi = warp; pi < n_pairs; pi += kWarps) ++my_pairs;
    int c_base = -64;                   // first local region held by the lane cache
    int c_y = 0, c_r = -1;              // tensor row and region of local region c_base + lane
    int c_v = 0;
    auto refill = [&](int base) {       // warp-collective
        c_base = base;
        const int q = base + lane;
        const int j = 2 * (warp + kWarps * (q >> 1)) + (q & 1);
        c_v = 0;
        c_r = -1;
        if (!bad_req && j < nr) {
            const int r = sel ? sel[j] : (t_lo >> 3) + j0 + j;
            if (r < 0 || r / 8 >= p.max_pages) {
                set_error(kErrAttnIndex);
            } else {
                const int64_t page = p.block_table[(int64_t)b * p.max_pages + r / 8];
                if (page < 0 || page >= p.n_pages) {
                    set_error(kErrAttnIndex);
                } else {
                    c_y = (int)(((page << p.gshift) + g) * kPage + (r % 8) * kRegion);
                    c_r = r;
                    c_v = 1;
                }
            }
        }
    };
    int slot_r[kSlots][2], slot_v[kSlots][2];
    auto issue = [&](int i, int slot) {   // warp-collective; lane 0 issues pair i's loads
        if (2 * i + 1 >= c_base + 32) refill(2 * i);
        const int s0 = 2 * i - c_base, s1 = s0 + 1;
        const int y0 = __shfl_sync(0xffffffffu, c_y, s0), y1 = __shfl_sync(0xffffffffu, c_y, s1);
        const int r0 = __shfl_sync(0xffffffffu, c_r, s0), r1 = __shfl_sync(0xffffffffu, c_r, s1);
        const int va = __shfl_sync(0xffffffffu, c_v, s0), vb = __shfl_sync(0xffffffffu, c_v, s1);
#pragma unroll
        for (int sl = 0; sl < kSlots; ++sl)
            if (sl == slot) {
                slot_r[sl][0] = r0;
                slot_r[sl][1] = r1;
                slot_v[sl][0] = va;
                slot_v[sl][1] = vb;
            }
        if (lane == 0) {
            uint8_t *dst = ring + slot * kPairBytes;
            const unsigned bytes = (va ? 2u * kRegionBytes : 0u) + (vb ? 2u * kRegionBytes : 0u);
            if (bytes == 0) {
                mbar_arrive(&wbar[slot]);
            } else {
                mbar_arrive_expect_tx(&wbar[slot], bytes);
                if (va) {
                    tma_load_3d(dst, &tmap_k, 0, 0, y0, &wbar[slot]);
                    tma_load_3d(dst + 2 * kRegionBytes, &tmap_v, 0, 0, y0, &wbar[slot]);
                }
                if (vb) {
                    tma_load_3d(dst + kRegionBytes, &tmap_k, 0, 0, y1, &wbar[slot]);
                    tma_load_3d(dst + 3 * kRegionBytes, &tmap_v, 0, 0, y1, &wbar[slot]);
                }
            }
        }
    };

    // prologue: resolve this warp's first region coordinates (sel_idx -> block_table) while
    // the Q tile loads, then issue the first pairs' TMA before building the Q fragments
    if (my_pairs > 0) refill(0);
    // Q tile [16 heads][192] into smem with the same swizzled layout as the K/V tiles
    const __nv_bfloat16 *qsrc = p.q + q_head(p, qi, g) * kD;
    static_assert(16 * kD / 8 == 3 * kThreads, "Q tile: three 16-byte chunks per thread");
    uint4 qv[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) {
        const int i = threadIdx.x + u * kThreads;
        qv[u] = __ldg(reinterpret_cast<const uint4 *>(qsrc + (i / (kD / 8)) * kD + (i % (kD / 8)) * 8));
    }
#pragma unroll
    for (int u = 0; u < 3; ++u) {
        const int i = threadIdx.x + u * kThreads;
        *reinterpret_cast<uint4 *>(qs + swz(i / (kD / 8), (i % (kD / 8)) * 8)) = qv[u];
    }
    fence_mbar_init();
    __syncthreads();

#pragma unroll
    for (int s2 = 0; s2 < kSlots; ++s2)
        if (s2 < my_pairs) issue(s2, s2);

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


    for (int i = 0; i < my_pairs; ++i) {
        const int slot = i % kSlots;
        const unsigned ph = (unsigned)(i / kSlots) & 1u;
        int rr[2];
        bool rv[2];
#pragma unroll
        for (int sl = 0; sl < kSlots; ++sl)
            if (sl == slot) {
                rr[0] = slot_r[sl][0];
                rr[1] = slot_r[sl][1];
                rv[0] = slot_v[sl][0] != 0;
                rv[1] = slot_v[sl][1] != 0;
            }
        if (!mbar_wait(&wbar[slot], ph)) break;
        const uint32_t kt = smem_u32(ring + slot * kPairBytes);
        const uint32_t vt = kt + 2 * kRegionBytes;

        // S = Q K^T: even and odd k-steps accumulate separately (four independent mma chains
        // of 6 instead of two of 12), summed at the end
        float s[2][4], s2[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
            s2[nt][0] = s2[nt][1] = s2[nt][2] = s2[nt][3] = 0.0f;
        }
#pragma unroll
        for (int kp = 0; kp < 6; ++kp) {           // two k-steps (32 dims) per ldmatrix.x4
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int c = kp * 32 + 8 * (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kt + nt * kRegionBytes + swz(lane & 7, c), b0, b1, b2, b3);
                mma_bf16_16816(s[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
                mma_bf16_16816(s2[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3],
                               b2, b3);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] += s2[nt][e];
        // scale, mask, online softmax (rows gq and gq+8 of this lane)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 8 * rr[nt] + 2 * t + (e & 1);
                const bool ok = rv[nt] && tok <= pos && tok >= t_lo;
                const float v = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
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
            const bool grow = mx[h] > mrow[h] + kSlack;
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
        if (next < my_pairs) {
            if (lane == 0) fence_proxy_async();
            issue(next, slot);
        }
    }

    // ---- merge the 4 warps: (m, l, O) of each warp to smem (reusing the rings), then
    // element-major combine so that smem reads and global writes are contiguous
    constexpr int kRow = kD + 8;                                         // padded row (floats)
    __syncthreads();
    float *red_o = reinterpret_cast<float *>(smem);                      // [4][16][kRow]
    float *red_ml = red_o + kWarps * 16 * kRow;                          // [4][16][2]
    float *hw = red_ml + kWarps * 16 * 2;                                // [16][4] weights, [16] L, [16] M
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
    if (threadIdx.x < 16) {                                              // per-head weights
        const int hr = threadIdx.x;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_ml[(w * 16 + hr) * 2]);
        const float Mref = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float wt = exp2f(red_ml[(w * 16 + hr) * 2] - Mref);
            hw[hr * 4 + w] = wt;
            L += wt * red_ml[(w * 16 + hr) * 2 + 1];
        }
        hw[64 + hr] = L;
        hw[80 + hr] = M;
    }
    __syncthreads();
    if (p.n_splits == 1) {
        // element e = (head, d) pair of dims: thread covers pairs e = tid + 128*j
        for (int e = threadIdx.x; e < 16 * kD / 2; e += kThreads) {
            const int hr = e / (kD / 2), d = 2 * (e % (kD / 2));
            float a = 0.0f, c = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float2 v = *reinterpret_cast<const float2 *>(red_o + (w * 16 + hr) * kRow + d);
                a += hw[hr * 4 + w] * v.x;
                c += hw[hr * 4 + w] * v.y;
            }
            const float L = hw[64 + hr];
            const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
            *reinterpret_cast<__nv_bfloat162 *>(p.out + out_head(p, qi, g, hr) * kD + d) =
                __floats2bfloat162_rn(a * inv, c * inv);
        }
        if (p.lse && threadIdx.x < 16) {
            const int hr = threadIdx.x;
            const float L = hw[64 + hr], M = hw[80 + hr];
            p.lse[out_head(p, qi, g, hr)] =
                (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
    } else {
        const int64_t pbase = ((int64_t)row * p.n_splits + split) * 16;
        for (int e = threadIdx.x; e < 16 * kD / 4; e += kThreads) {
            const int hr = e / (kD / 4), d = 4 * (e % (kD / 4));
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float4 v = *reinterpret_cast<const float4 *>(red_o + (w * 16 + hr) * kRow + d);
                const float wt = hw[hr * 4 + w];
                acc.x += wt * v.x;
                acc.y += wt * v.y;
                acc.z += wt * v.z;
                acc.w += wt * v.w;
            }
            *reinterpret_cast<float4 *>(p.part_o + (pbase + hr) * kD + d) = acc;
        }
        if (threadIdx.x < 16) {
            const int hr = threadIdx.x;
            p.part_ml[(pbase + hr) * 2 + 0] = hw[80 + hr];
            p.part_ml[(pbase + hr) * 2 + 1] = hw[64 + hr];
        }
    }
}

// Merges the per-split partials of one (query, head): O = sum_s 2^(m_s - M) O_s / L.
// 4 x 192 threads: thread (sg, d) sums splits sg, sg+4, ... of dimension d with all its
// loads in flight, then the 4 partial sums meet in smem.
constexpr int kCombineThreads = 4 * kD;
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    __shared__ float wsm[kD];
    __shared__ float part[kCombineThreads / 32];
    __shared__ float red[2];
    __shared__ float osum[4][kD];
    const int row = blockIdx.x >> 4, hr = blockIdx.x & 15;
    if (p.row_shared && p.row_shared[row]) return;
    const int qi = row >> p.gshift, g = row & ((1 << p.gshift) - 1);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int d = tid % kD, sg = tid / kD;
    bool bad_cnt;
    const int cnt = row_count(p, row, p.q_pos[qi], bad_cnt);
    const int ns = min(p.n_splits, (cnt + p.rps - 1) / p.rps);   // <= kD (host-checked)
    const int64_t pbase = (int64_t)row * p.n_splits * 16 + hr;
    float m = -INFINITY, l = 0.0f;
    if (tid < ns) {
        m = p.part_ml[(pbase + (int64_t)tid * 16) * 2];
        l = p.part_ml[(pbase + (int64_t)tid * 16) * 2 + 1];
    }
    float mx = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) part[w] = mx;
    __syncthreads();
    if (tid == 0) {
        float M = -INFINITY;
        for (int i = 0; i < kCombineThreads / 32; ++i) M = fmaxf(M, part[i]);
        red[0] = M;
    }
    __syncthreads();
    const float M = red[0];
    const float Mref = (M == -INFINITY) ? 0.0f : M;
    const float wt = (tid < ns) ? exp2f(m - Mref) : 0.0f;
    if (tid < kD) wsm[tid] = wt;
    float lw = wt * l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
    __syncthreads();
    if (lane == 0) part[w] = lw;
    __syncthreads();
    if (tid == 0) {
        float L = 0.0f;
        for (int i = 0; i < kCombineThreads / 32; ++i) L += part[i];
        red[1] = L;
    }
    __syncthreads();
    const float L = red[1];
    float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    int s = sg;
    for (; s + 28 < ns; s += 32) {
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] += wsm[s + 4 * u] * p.part_o[(pbase + (int64_t)(s + 4 * u) * 16) * kD + d];
    }
    for (; s < ns; s += 4) acc[0] += wsm[s] * p.part_o[(pbase + (int64_t)s * 16) * kD + d];
    osum[sg][d] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    __syncthreads();
    if (sg == 0) {
        const float o = (osum[0][d] + osum[1][d]) + (osum[2][d] + osum[3][d]);
        const int64_t head = out_head(p, qi, g, hr);
        p.out[head * kD + d] = __float2bfloat16_rn(L > 0.0f ? o / L : 0.0f);
        if (p.lse && d == 0)
            p.lse[head] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
}

}  // namespace attn
}  // namespace dsa
