// A2 indexer scores for a prefill chunk as a tcgen05 FP8 GEMM ([P1] kwkr.cn/news/601179
// §DSA ③; [P2] Step-5-Preview 如何实现1M长上下文 §索引器打分).
//
// For one request's chunk of queries the score is a dense contraction per KV group g:
//   C_g[(q, h)][r] = sum_d q8[q][h][d] * s8[g][r][d]        (e4m3 x e4m3 -> fp32, K = 256)
//   score[q][g][r] = scale[g][r] / 16 * sum_{h in g} z[q][h] * sq[q][h] * ReLU(C_g[(q, h)][r])
// with the query quantised per (query, head) to e4m3 with scale sq = absmax/448 (the FP8
// reading of the method, DSA_Q_FP8).  Layout of the work:
//  * a work unit is (group g, block of 256 regions, range of 128-row query tiles); the
//    CTA keeps the unit's 256 x 256 B summary tile in smem (two TMA boxes of 128-byte
//    columns, 128-byte swizzle) and streams query tiles of 32 queries x 4 heads through a
//    2-stage TMA ring.  Keeping the summaries resident and streaming the (small) queries
//    reads the queries ~129 times and the summaries once per query range instead of the
//    summaries 64 times;
//  * one thread issues 8 tcgen05.mma kind::f8f6f4 (M = 128, N = 256, K = 32) per tile into
//    one of two 256-column TMEM accumulators (512 columns: all of TMEM, one CTA per SM);
//  * four epilogue warps (one per TMEM lane quarter) read 32 columns at a time, apply
//    ReLU * z * sq per row, sum the 4 heads of a query with a two-step shuffle butterfly
//    that leaves every lane 8 finished columns, scale by scale[g][r]/16, mask r < own and
//    store; the accumulator buffer is released to the MMA thread after the last read;
//  * tiles whose queries all have own <= the block's first region are skipped (causal).
#pragma once

#include "common.cuh"

namespace dsa {
namespace gemm {

constexpr int kQPerTile = 32;
constexpr int kBM = kQPerTile * 4;       // 128 rows: (query, head of the group)
constexpr int kBN = 256;                 // regions per summary tile
constexpr int kAStages = 2;
constexpr int kAHalf = kBM * 128;        // one 128-byte K column of a query tile (16 KiB)
constexpr int kABytes = 2 * kAHalf;
constexpr int kBHalf = kBN * 128;        // 32 KiB
constexpr int kBBytes = 2 * kBHalf;
constexpr int kThreads = 192;            // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kTmemCols = 512;           // two 256-column fp32 accumulators
constexpr size_t kSmemBytes = 1024 + kBBytes + kAStages * kABytes + 4 * kBN * 4 + 256;
constexpr uint32_t kIdesc = umma_idesc_e4m3(kBM, kBN);

struct Params {
    const float *qscale;       // [nq][16]  (prepass)
    const float *gate;         // [nq][16]
    const int32_t *q_own;      // [nq] validated own region, -1 = skip (prepass)
    const int32_t *tile_own;   // [n_mtiles] largest own region of the tile's queries (prepass)
    const float *scales;       // [4][n_slots]
    const int64_t *sum_base;   // [1]
    float *scores;             // [nq][4][ld]
    int64_t ld;
    int64_t n_slots;
    int nq;
    int n_rblocks;
    int n_mtiles;
    int m_per_unit;
    int n_mparts;
    int n_units;
};

// The query's own region when the query is valid for this path (request 0, pos >= 0, own
// region within the score row and the pool), else -1.
__device__ __forceinline__ int valid_own(const int32_t *q_req, const int32_t *q_pos, const int64_t *sum_base,
                                         int64_t ld, int64_t n_slots, int q)
{
    const int pos = q_pos[q];
    if (q_req[q] != 0 || pos < 0) return -1;
    const int64_t own = pos / kRegion, base = sum_base[0];
    if (own > ld || base < 0 || base + own > n_slots) return -1;
    return (int)own;
}

// Per (query, head): sq = absmax/448 (IEEE division), codes = e4m3(x / sq), all 0 when the
// head is zero.  One warp per (q, h).  Also the validated own region of every query
// (-1 and an error for an invalid one) and the largest own region of every 32-query tile.
__global__ void __launch_bounds__(128) quantize_kernel(const __nv_bfloat16 *__restrict__ index_q,
                                                       const int32_t *__restrict__ q_req,
                                                       const int32_t *__restrict__ q_pos,
                                                       const int64_t *__restrict__ sum_base, int64_t ld,
                                                       int64_t n_slots, int nq, uint8_t *__restrict__ codes,
                                                       float *__restrict__ qscale, int32_t *__restrict__ q_own,
                                                       int32_t *__restrict__ tile_own, int n_mtiles)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    const int gw = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (gw < nq * kHI) {
        const int q = gw / kHI;
        if (lane == 0 && gw % kHI == 0) {
            const int own = valid_own(q_req, q_pos, sum_base, ld, n_slots, q);
            if (own < 0) set_error(kErrIndexerQuery);
            q_own[q] = own;
        }
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(index_q + (int64_t)gw * kDI + lane * 8));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float x[8];
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[2 * j] = bf16_lo(w[j]);
            x[2 * j + 1] = bf16_hi(w[j]);
            amax = fmaxf(amax, fmaxf(fabsf(x[2 * j]), fabsf(x[2 * j + 1])));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sq = __fdiv_rn(amax, 448.0f);
        uint32_t c[4] = {0, 0, 0, 0};
        if (sq != 0.0f) {
#pragma unroll
            for (int j = 0; j < 4; ++j) c[j] = cvt_e4m3x2(__fdiv_rn(x[2 * j], sq), __fdiv_rn(x[2 * j + 1], sq));
        }
        *reinterpret_cast<uint2 *>(codes + (int64_t)gw * kDI + lane * 8) =
            make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
        if (lane == 0) qscale[gw] = sq;
    }
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < n_mtiles) {
        int m = -1;
        for (int i = 0; i < kQPerTile; ++i) {
            const int q = t * kQPerTile + i;
            if (q < nq) m = max(m, valid_own(q_req, q_pos, sum_base, ld, n_slots, q));
        }
        tile_own[t] = m;
    }
}


// Work unit u -> (group, region block, query-tile range); a unit is active iff one of its
// tiles holds a query whose own region lies beyond the block's first region.
__device__ __forceinline__ void unit_coords(const Params &p, int u, int &g, int &rb, int &t0, int &t1)
{
    const int mp = u % p.n_mparts;
    const int gr = u / p.n_mparts;
    rb = gr % p.n_rblocks;
    g = gr / p.n_rblocks;
    t0 = mp * p.m_per_unit;
    t1 = min(p.n_mtiles, t0 + p.m_per_unit);
}

__device__ __forceinline__ bool tile_active(const Params &p, int t, int rb)
{
    return p.tile_own[t] > rb * kBN;
}

__device__ __forceinline__ bool unit_active(const Params &p, int t0, int t1, int rb)
{
    for (int t = t0; t < t1; ++t)
        if (tile_active(p, t, rb)) return true;
    return false;
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_scores_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sb = smem;                                   // summary tile: 2 K columns x [256][128]
    uint8_t *sa = smem + kBBytes;                         // query tiles: kAStages x 2 K columns x [128][128]
    float *sscale_all = reinterpret_cast<float *>(sa + kAStages * kABytes);    // [4 warps][256] scales / 16
    uint64_t *bars = reinterpret_cast<uint64_t *>(sscale_all + 4 * kBN);
    uint64_t *b_full = bars + 0, *b_empty = bars + 1;
    uint64_t *a_full = bars + 2, *a_empty = bars + 4;     // [kAStages]
    uint64_t *acc_full = bars + 6, *acc_empty = bars + 8; // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(b_full, 1);
        mbar_init(b_empty, 1);
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t base = p.sum_base[0];
    bool ok = true;

    if (warp == 0) {
        // ---------------- TMA producer (one lane)
        if (lane == 0) {
            prefetch_tensormap(&map_a);
            prefetch_tensormap(&map_b);
            int ub = 0, ait = 0;
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                int g, rb, t0, t1;
                unit_coords(p, u, g, rb, t0, t1);
                if (!unit_active(p, t0, t1, rb)) continue;
                ok = mbar_wait(b_empty, (ub & 1) ^ 1);
                if (!ok) break;
                mbar_arrive_expect_tx(b_full, kBBytes);
                const int y = (int)(g * p.n_slots + base + (int64_t)rb * kBN);
                tma_load_2d(sb, &map_b, 0, y, b_full);
                tma_load_2d(sb + kBHalf, &map_b, 128, y, b_full);
                ++ub;
                for (int t = t0; t < t1; ++t) {
                    if (!tile_active(p, t, rb)) continue;
                    const int s = ait % kAStages;
                    ok = mbar_wait(&a_empty[s], ((ait / kAStages) & 1) ^ 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&a_full[s], kABytes);
                    uint8_t *dst = sa + s * kABytes;
                    tma_load_4d(dst, &map_a, 0, 0, g, t * kQPerTile, &a_full[s]);
                    tma_load_4d(dst + kAHalf, &map_a, 128, 0, g, t * kQPerTile, &a_full[s]);
                    ++ait;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one lane)
        if (lane == 0) {
            int ub = 0, ait = 0, cit = 0;
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                int g, rb, t0, t1;
                unit_coords(p, u, g, rb, t0, t1);
                if (!unit_active(p, t0, t1, rb)) continue;
                ok = mbar_wait(b_full, ub & 1);
                if (!ok) break;
                ++ub;
                for (int t = t0; t < t1; ++t) {
                    if (!tile_active(p, t, rb)) continue;
                    const int s = ait % kAStages, buf = cit & 1;
                    ok = mbar_wait(&a_full[s], (ait / kAStages) & 1) &&
                         mbar_wait(&acc_empty[buf], ((cit >> 1) & 1) ^ 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sa + s * kABytes), b0 = smem_u32(sb);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off_a = (kk >> 2) * kAHalf + (kk & 3) * 32;
                        const uint32_t off_b = (kk >> 2) * kBHalf + (kk & 3) * 32;
                        umma_e4m3(tmem + buf * kBN, umma_desc_sw128(a0 + off_a), umma_desc_sw128(b0 + off_b), kIdesc,
                                  kk > 0);
                    }
                    umma_commit(&a_empty[s]);        // the query tile may be overwritten
                    umma_commit(&acc_full[buf]);     // the accumulator is ready
                    ++ait;
                    ++cit;
                }
                if (!ok) break;
                umma_commit(b_empty);                // the summary tile may be overwritten
            }
        }
    } else {
        // ---------------- epilogue: warps 2..5, TMEM lane quarter sp = warp % 4
        const int sp = warp & 3;
        const int qt = sp * 8 + (lane >> 2), h = lane & 3;      // this lane's row: query in tile, head
        const int cb = 16 * (h & 1) + 8 * ((h >> 1) & 1);        // its 8 finished columns in a chunk
        float *wscale = sscale_all + (warp - 2) * kBN;
        int cit = 0;
        for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
            int g, rb, t0, t1;
            unit_coords(p, u, g, rb, t0, t1);
            if (!unit_active(p, t0, t1, rb)) continue;
            // this unit's 256 region scales / 16, staged by each warp in its own smem slice
            // (no barrier across the epilogue warps); entries past the pool read as 0
            {
                const int64_t s0 = g * p.n_slots + base + (int64_t)rb * kBN;
                const int64_t lim = (int64_t)kG * p.n_slots;
#pragma unroll
                for (int j = 0; j < kBN / 32; ++j) {
                    const int64_t i = s0 + j * 32 + lane;
                    wscale[j * 32 + lane] = i < lim ? __ldg(p.scales + i) * 0.0625f : 0.0f;
                }
                __syncwarp();
            }
            for (int t = t0; t < t1; ++t) {
                if (!tile_active(p, t, rb)) continue;
                const int buf = cit & 1;
                const int q = t * kQPerTile + qt;
                const bool qv = q < p.nq;
                const float w = qv ? p.gate[q * kHI + g * 4 + h] * p.qscale[q * kHI + g * 4 + h] : 0.0f;
                const int own = qv ? p.q_own[q] : -1;
                ok = mbar_wait(&acc_full[buf], (cit >> 1) & 1);
                if (!ok) break;
                tc_fence_after();
                float *orow = p.scores + ((int64_t)q * kG + g) * p.ld;
#pragma unroll 1
                for (int ch = 0; ch < kBN / 32; ++ch) {
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * sp) << 16) + buf * kBN + ch * 32, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.0f) * w;
                    // heads h and h^1: keep 16 columns (h&1 ? 16..31 : 0..15)
                    float k16[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float send = (h & 1) ? v[j] : v[16 + j];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                        k16[j] = ((h & 1) ? v[16 + j] : v[j]) + recv;
                    }
                    // heads {h, h^1} and {h^2, h^3}: keep 8 columns
                    float k8[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float send = (h & 2) ? k16[j] : k16[8 + j];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
                        k8[j] = ((h & 2) ? k16[8 + j] : k16[j]) + recv;
                    }
                    const int c0 = ch * 32 + cb;
                    const int64_t r0 = (int64_t)rb * kBN + c0;
                    if (qv && r0 < own) {
                        const float4 sa4 = *reinterpret_cast<const float4 *>(wscale + c0);
                        const float4 sb4 = *reinterpret_cast<const float4 *>(wscale + c0 + 4);
                        const float sc[8] = {sa4.x, sa4.y, sa4.z, sa4.w, sb4.x, sb4.y, sb4.z, sb4.w};
                        if (r0 + 8 <= own && (p.ld & 3) == 0) {
                            *reinterpret_cast<float4 *>(orow + r0) =
                                make_float4(k8[0] * sc[0], k8[1] * sc[1], k8[2] * sc[2], k8[3] * sc[3]);
                            *reinterpret_cast<float4 *>(orow + r0 + 4) =
                                make_float4(k8[4] * sc[4], k8[5] * sc[5], k8[6] * sc[6], k8[7] * sc[7]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (r0 + j < own) orow[r0 + j] = k8[j] * sc[j];
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
                ++cit;
            }
            __syncwarp();                                   // the slice is rewritten by the next unit
        }
    }
    // every role done (or gave up): release TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_free(tmem, kTmemCols);
}

}  // namespace gemm
}  // namespace dsa
