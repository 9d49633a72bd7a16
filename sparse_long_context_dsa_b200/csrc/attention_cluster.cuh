// A4 sparse GQA attention for a few long selections (decode of one or two requests), and the
// window layers' decode over each query's last `window` tokens (optionally appending the
// query's own token to the cache in the same kernel), with the split merge inside the kernel ([P1] kwkr.cn/news/601179 §DSA ④ and §滑窗注意力; [P3] 100 万 token 上下文实测
// §一: the hit regions are gathered from the paged cache through the block_table).
//
// A (query, group) row is attended by a cluster of S CTAs; CTA `rank` takes the row's
// regions [R*rank, R*rank + R) (the selection, or the window's regions in order).  Shapes:
// S = 16, R = 32 for selections of up to 512 regions; S = 8, R = 10 for windows of up to 80
// regions (a 512-token window touches at most 65), two CTAs per SM.  Every CTA issues all of
// its K/V loads at once (R regions x 6 KiB, TMA with the 128-byte swizzle into R/2 pair
// buffers, one mbarrier per pair), so a CTA waits for one memory round trip, not one per
// pair.  Warp w takes pairs w and w + 8 (those that exist) for S = Q K^T (mma.sync
// m16n8k16 bf16, fp32 accumulate; tokens t <= p only, and t > p - window for a window, in
// log2 units); the CTA's row maximum M of each head goes through smem, every warp writes
// P = 2^(S - M) in bf16 to one [16 heads][8R tokens] tile, and warp w then computes the
// output dims [24w, 24w + 24) of O = P V over all the CTA's tokens.  So no warp merges
// another's O.  The CTA's (M, l, O) of head h goes to CTA h mod S (slot h / S of its inbox
// row for this CTA) as one bulk copy that completes on that CTA's inbox barrier; once its 16
// rows are in, CTA r merges heads r, r + S, ... of the row (O = sum_c 2^(m_c - M) O_c /
// sum_c 2^(m_c - M) l_c) and writes the bf16 output and the LSE.  No partials in global
// memory, no second kernel, no cluster barrier after the start.
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

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kInRow = kD + 4;                 // inbox row per (source CTA, head slot): O [kD], m, l, pad
constexpr int kDimsPerWarp = kD / kWarps;      // 24: three n8 tiles of O per warp
static_assert(kDimsPerWarp == 24, "three n8 tiles of output dims per warp");

// The shape of a row's cluster: S CTAs of R regions each (R even, R <= 32, 16 % S == 0).
template <int S, int R>
struct Shape {
    static constexpr int kSplits = S;
    static constexpr int kRegionsPerCta = R;
    static constexpr int kPairs = R / 2;
    static constexpr int kOwn = (kPairs + kWarps - 1) / kWarps;             // pairs a warp owns, at most
    static constexpr int kHeadsPerCta = kHeadsPerGroup / S;                 // heads a CTA merges
    static constexpr size_t kPairArea = (size_t)kPairs * kPairBytes;
    static constexpr size_t kInbox = (size_t)kHeadsPerGroup * kInRow * 4;   // 16 rows, outside the pair area
    static constexpr int kTokens = 8 * R;
    static constexpr int kPRow = 2 * kTokens + 16;                          // P tile row (bytes), padded
    static constexpr size_t kMl = (size_t)2 * kWarps * 16 * 4;              // per-warp row maxima and sums
    static constexpr size_t kPTile = (size_t)16 * kPRow;
    static constexpr size_t kSmemBytes = 1024 + kPairArea + kQBytes + 256 + kInbox + kMl + kPTile;
    static constexpr int kMaxK = S * R;
    static_assert(R % 2 == 0 && R <= 32 && kHeadsPerGroup % S == 0, "shape");
    static_assert(kInbox % 16 == 0 && kMl % 16 == 0, "the P tile stays 16-byte aligned");
    static_assert((kInRow * 4) % 16 == 0 && (size_t)kHeadsPerGroup * kInRow * 4 <= kPairArea,
                  "inbox rows are whole 16-byte bulk copies; the staged rows fit the pair area");
    static_assert((kPairs + 1) * 8 <= 256, "pair barriers and the inbox barrier fit their 256 bytes");
    // ldmatrix of 8 P rows: row r starts (r * kPRow / 4) mod 32 banks in; 16-byte chunks of the
    // 8 rows fall in distinct 4-bank groups when that step is 4 or 12 modulo 32 (or 20, 28)
    static_assert((kPRow / 4) % 8 == 4, "P rows land in distinct 16-byte bank groups");
};
using Decode = Shape<16, 32>;                  // selections of up to 512 regions
using Window = Shape<8, 10>;                   // windows of up to 80 regions
constexpr int kMaxK = Decode::kMaxK;           // 512

// kWin: window mode (the row's regions are the window's, from the position) instead of a
// selection (sel_idx, sel_count).
template <int S, int R, int kMinBlocks, bool kWin>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    sparse_attn_cluster_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                               const Params p)
{
    using Sh = Shape<S, R>;
    constexpr int kSplits = S, kRegionsPerCta = R, kPairs = Sh::kPairs, kOwn = Sh::kOwn;
    constexpr int kHpc = Sh::kHeadsPerCta, kPRow = Sh::kPRow;
    constexpr size_t kPairArea = Sh::kPairArea;
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    // the tensor maps are kernel parameters (no earlier kernel writes them): their descriptors
    // are fetched while the previous kernel finishes, not in front of the first loads
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmap_k);
        prefetch_tensormap(&tmap_v);
    }
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *qs = smem + kPairArea;
    uint64_t *bars = reinterpret_cast<uint64_t *>(qs + kQBytes);            // [kPairs]
    float *inbox = reinterpret_cast<float *>(qs + kQBytes + 256);           // [kSplits][kHpc][kInRow]
    float *mw = inbox + kHeadsPerGroup * kInRow;                            // [kWarps][16] row maxima
    float *lw = mw + kWarps * 16;                                           // [kWarps][16] row sums
    uint8_t *ptile = reinterpret_cast<uint8_t *>(lw + kWarps * 16);         // P [16 heads][kPRow bytes]
    __shared__ int sh_y[kRegionsPerCta], sh_r[kRegionsPerCta], sh_v[kRegionsPerCta];   // per region of the CTA
    __shared__ int sh_ok[kPairs];                                           // the pair's data landed

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
    // lane l < 2 kOwn of warp w -> region 2 (w + 8 (l / 2)) + l % 2 of the CTA (its owned pairs)
    auto reg_of = [&](int l) { return (l >> 1) * 16 + 2 * warp + (l & 1); };
    const bool reg_lane = lane < 2 * kOwn && reg_of(lane) < kRegionsPerCta;
    const int j0 = rank * kRegionsPerCta;
    constexpr bool win = kWin;
    int rr_spec = -1;
    if (!win && reg_lane && j0 + reg_of(lane) < p.k) rr_spec = p.sel_idx[(int64_t)row * p.k + j0 + reg_of(lane)];
    const int b = p.q_req ? p.q_req[qi] : qi;
    const int pos = p.q_pos[qi];
    // window mode: the regions holding tokens t_lo .. pos, tokens below t_lo masked
    const int t_lo = win ? max(0, pos - p.window + 1) : 0;
    int cnt;
    const int newest = (pos >> 3) - (t_lo >> 3);                            // window mode: the token's region
    if constexpr (win) {
        cnt = pos < 0 ? 0 : min(newest + 1, p.k);
        rr_spec = (t_lo >> 3) + j0 + reg_of(lane);
    } else {
        const int cnt_raw = p.sel_count[row];
        cnt = min(max(cnt_raw, 0), p.k);
        if (cnt != cnt_raw && rank == 0 && tid == 0) set_error(kErrAttnIndex);
    }
    const int nr = max(0, min(kRegionsPerCta, cnt - j0));                   // regions of this CTA
    const bool bad_req = (b < 0 || b >= p.n_req || pos < 0);
    // Warp w owns pairs w and w + 8 (regions 2w, 2w+1, 2w+16, 2w+17 of the CTA): it sets up
    // their barriers, resolves their coordinates (sel_idx -> block_table, lanes 0..3) and
    // issues their TMA loads itself, so the 8 warps issue in parallel.
    if (lane < kOwn && warp + 8 * lane < kPairs) mbar_init(&bars[warp + 8 * lane], 1);
    uint64_t *inbox_bar = &bars[kPairs];                                    // the 16 inbox rows landed
    if (tid == 0) {
        mbar_init(inbox_bar, 1);
        mbar_arrive_expect_tx(inbox_bar, (unsigned)(kHeadsPerGroup * kInRow * 4));
    }
    fence_mbar_init();
    __syncwarp();
    // every CTA's inbox barrier is set up before any CTA copies into it: arrive now, wait
    // before the copies (long after every CTA arrived)
    cluster_arrive_relaxed();
    if (reg_lane) {
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
    }
    __syncwarp();
    if (lane < kOwn) {
        const int pr = warp + 8 * lane;
        if (pr < kPairs && 2 * pr < nr) {
            const int va = sh_v[2 * pr], vb = sh_v[2 * pr + 1];
            const unsigned bytes = (va ? 2u * kRegionBytes : 0u) + (vb ? 2u * kRegionBytes : 0u);
            if (bytes == 0) mbar_arrive(&bars[pr]);
            else mbar_arrive_expect_tx(&bars[pr], bytes);
        }
    }
    __syncwarp();
    if (reg_lane) {
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
    const int n_pairs = (nr + 1) / 2;
    // ---- S = Q K^T of this warp's pairs (warp, warp + 8), in log2 units, masked to t <= p
    float s[kOwn][2][4];
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < kOwn; ++i) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) s[i][nt][0] = s[i][nt][1] = s[i][nt][2] = s[i][nt][3] = -INFINITY;
        const int pr = warp + kWarps * i;
        if (pr >= n_pairs) continue;
        const bool landed = mbar_wait(&bars[pr], 0u);                     // false: error set, pair skipped
        if (lane == 0) sh_ok[pr] = landed ? 1 : 0;
        if (!landed) continue;
        if constexpr (kWin) {
            // the appended token (window decode with the append folded in): its K and V rows
            // from new_k / new_v into this pair's tiles, whatever the load read for its slot,
            // and into its cache slot for the steps to come (this group's rows; the CTA of the
            // row's newest region writes them)
            const int jn = newest - j0;
            if (p.new_k && jn >= 0 && jn < kRegionsPerCta && (jn >> 1) == pr && sh_v[jn]) {
                const int rt = pos & 7;                                     // the token's row in its region
                const int64_t crow = (int64_t)sh_y[jn] + rt;                // and in the cache
                const int64_t src = ((int64_t)qi * kG + p.g0 + g) * kD;
                for (int c = lane; c < 2 * (kD / 8); c += 32) {             // 16-byte chunks: K, then V
                    const int which = c / (kD / 8), cc = c % (kD / 8);
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>((which ? p.new_v : p.new_k) + src + cc * 8));
                    uint8_t *tile = smem + (size_t)pr * kPairBytes + (2 * which + (jn & 1)) * kRegionBytes;
                    *reinterpret_cast<uint4 *>(tile + swz(rt, cc * 8)) = v;
                    *reinterpret_cast<uint4 *>((which ? p.v_cache : p.k_cache) + crow * kD + cc * 8) = v;
                }
                __syncwarp();
            }
        }
        const int rr[2] = {sh_r[2 * pr], sh_r[2 * pr + 1]};
        const bool rv[2] = {sh_v[2 * pr] != 0, sh_v[2 * pr + 1] != 0};
        const uint32_t kt = smem_u32(smem + (size_t)pr * kPairBytes);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const uint32_t tile = kt + nt * kRegionBytes;
            const int r = lane & 7;
#pragma unroll
            for (int kp = 0; kp < 6; ++kp) {       // two k-steps (32 dims) per ldmatrix.x4
                const int c = kp * 32 + 8 * (lane >> 3);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(tile + swz(r, c), b0, b1, b2, b3);
                mma_bf16_16816(acc, qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
                mma_bf16_16816(acc, qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3], b2,
                               b3);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 8 * rr[nt] + 2 * t + (e & 1);
                const float v = (rv[nt] && tok <= pos && tok >= t_lo) ? acc[e] * p.scale_log2 : -INFINITY;
                s[i][nt][e] = v;
                mx[e >> 1] = fmaxf(mx[e >> 1], v);
            }
        }
    }
    // ---- the CTA's row maximum of each head (rows gq and gq + 8 of this lane)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
    }
    if (t == 0) {
        mw[warp * 16 + gq] = mx[0];
        mw[warp * 16 + gq + 8] = mx[1];
    }
    __syncthreads();
    float M[2], mref[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        M[h] = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M[h] = fmaxf(M[h], mw[w * 16 + gq + 8 * h]);
        mref[h] = (M[h] == -INFINITY) ? 0.0f : M[h];
    }
    // ---- P = 2^(S - M): bf16 into the P tile (token column 16 pr + 8 nt + 2t), fp32 row sums
    float ps[2] = {0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < kOwn; ++i) {
        const int pr = warp + kWarps * i;
        if (pr >= n_pairs) continue;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float p0 = exp2f(s[i][nt][0] - mref[0]), p1 = exp2f(s[i][nt][1] - mref[0]);
            const float p2 = exp2f(s[i][nt][2] - mref[1]), p3 = exp2f(s[i][nt][3] - mref[1]);
            ps[0] += p0 + p1;
            ps[1] += p2 + p3;
            const int col = 2 * (16 * pr + 8 * nt + 2 * t);
            *reinterpret_cast<uint32_t *>(ptile + gq * kPRow + col) = pack_bf16x2(p0, p1);
            *reinterpret_cast<uint32_t *>(ptile + (gq + 8) * kPRow + col) = pack_bf16x2(p2, p3);
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], 1);
        ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], 2);
    }
    if (t == 0) {
        lw[warp * 16 + gq] = ps[0];
        lw[warp * 16 + gq + 8] = ps[1];
    }
    __syncthreads();

    // ---- O[:, 24 warp .. 24 warp + 24) = P V, one k-step per pair (16 tokens); the loop is
    // unrolled over the 16 pairs with two accumulator sets (even and odd pairs), so the loads
    // of later pairs overlap the MMAs of earlier ones
    float o[2][3][4];
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
        for (int j = 0; j < 3; ++j) o[a2][j][0] = o[a2][j][1] = o[a2][j][2] = o[a2][j][3] = 0.0f;
    {
        // region j of the CTA takes part when its data landed and it is valid (bit j)
        const unsigned use = __ballot_sync(0xffffffffu, lane < kRegionsPerCta && (lane >> 1) < n_pairs &&
                                                            sh_v[lane] != 0 && sh_ok[lane >> 1] != 0);
        const uint32_t pbase = smem_u32(ptile);
        const int ar = (lane & 7) + 8 * ((lane >> 3) & 1);
        const int r = lane & 7, reg = (lane >> 3) & 1, dsub = 8 * (lane >> 4);
        const int nd0 = 3 * warp;
        const uint32_t vbase = smem_u32(smem) + 2 * kRegionBytes + reg * kRegionBytes;
        const uint32_t voff_b = swz(r, nd0 * 8 + dsub), voff_c = swz(r, (nd0 + 2) * 8);
#pragma unroll
        for (int pr = 0; pr < kPairs; ++pr) {
            const unsigned u2 = (use >> (2 * pr)) & 3u;
            if (u2 == 0u) continue;                                       // uniform: no token of the pair
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(pbase + ar * kPRow + 2 * (16 * pr + 8 * (lane >> 4)), a0, a1, a2, a3);
            const uint32_t vt = vbase + (uint32_t)pr * kPairBytes;
            uint32_t b0, b1, b2, b3, c0, c1;
            ldmatrix_x4_trans(vt + voff_b, b0, b1, b2, b3);
            ldmatrix_x2_trans(vt + voff_c, c0, c1);
            // a region that was not loaded holds stale smem: its P is 0, but 0 * NaN is not
            if (!(u2 & 1u)) b0 = b2 = c0 = 0u;
            if (!(u2 & 2u)) b1 = b3 = c1 = 0u;
            float(&oa)[3][4] = o[pr & 1];
            mma_bf16_16816(oa[0], a0, a1, a2, a3, b0, b1);
            mma_bf16_16816(oa[1], a0, a1, a2, a3, b2, b3);
            mma_bf16_16816(oa[2], a0, a1, a2, a3, c0, c1);
        }
#pragma unroll
        for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[0][j][e] += o[1][j][e];
    }
    // ---- this CTA's (M, l, O) of head h goes to CTA h % S, inbox row (rank, h / S): the rows
    // are staged in the (now free) pair area and sent as 16 bulk copies of kInRow floats, each
    // completing on the destination's inbox barrier, so a CTA waits for its own 16 rows and
    // nothing else
    __syncthreads();                                                        // every warp is done with P and V
    float *stage = reinterpret_cast<float *>(smem);                         // [16][kInRow]
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int col = (3 * warp + j) * 8 + 2 * t;
        *reinterpret_cast<float2 *>(stage + gq * kInRow + col) = make_float2(o[0][j][0], o[0][j][1]);
        *reinterpret_cast<float2 *>(stage + (gq + 8) * kInRow + col) = make_float2(o[0][j][2], o[0][j][3]);
    }
    if (warp == 0 && t == 0) {
        float L[2] = {0.0f, 0.0f};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int w = 0; w < kWarps; ++w) L[h] += lw[w * 16 + gq + 8 * h];
        stage[gq * kInRow + kD] = M[0];
        stage[gq * kInRow + kD + 1] = L[0];
        stage[(gq + 8) * kInRow + kD] = M[1];
        stage[(gq + 8) * kInRow + kD + 1] = L[1];
    }
    fence_proxy_async();                                                    // the rows, to the copy engine
    __syncwarp();
    cluster_wait();
    __syncthreads();
    if (warp == 0 && lane < kHeadsPerGroup) {
        bulk_copy_to_cta(inbox + (rank * kHpc + lane / kSplits) * kInRow, stage + lane * kInRow,
                         (unsigned)(kInRow * 4), inbox_bar, (unsigned)(lane % kSplits));
        bulk_commit();
    }
    const bool inbox_ok = mbar_wait(inbox_bar, 0u);                         // false: error set

    // ---- CTA `rank` merges heads rank + S j (j < 16 / S) of the row from its inbox
    for (int e = tid; inbox_ok && e < kHpc * kD; e += kThreads) {
        const int j = e / kD, d = e % kD, hr = rank + kSplits * j;
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < kSplits; ++c) M = fmaxf(M, inbox[(c * kHpc + j) * kInRow + kD]);
        const float Mref = (M == -INFINITY) ? 0.0f : M;
        float L = 0.0f, acc = 0.0f;
#pragma unroll
        for (int c = 0; c < kSplits; ++c) {
            const float *in = inbox + (c * kHpc + j) * kInRow;
            const float wt = exp2f(in[kD] - Mref);
            L += wt * in[kD + 1];
            acc += wt * in[d];
        }
        const int64_t head = attn::out_head(p, qi, g, hr);
        p.out[head * kD + d] = __float2bfloat16_rn(L > 0.0f ? acc / L : 0.0f);
        if (p.lse && d == 0) p.lse[head] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
    // this CTA's copies have read their rows before its shared memory goes away
    if (warp == 0 && lane < kHeadsPerGroup) bulk_wait_read_all();
}

}  // namespace attnc
}  // namespace dsa
