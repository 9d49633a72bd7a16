// A2 indexer scores for a prefill chunk as a tcgen05 FP8 GEMM ([P1] kwkr.cn/news/601179
// §DSA ③; [P2] Step-5-Preview 如何实现1M长上下文 §索引器打分).
//
// For one request's chunk of queries the score is a dense contraction per KV group g:
//   C[r][(q, h)] = sum_d s8[g][r][d] * q8[q][h][d]        (e4m3 x e4m3 -> fp32, K = 256)
//   score[q][g][r] = scale[g][r] / 16 * sum_{h in g} z[q][h] * sq[q][h] * ReLU(C[r][(q, h)])
// with the query quantised per (query, head) to e4m3 with scale sq = absmax/448 (the FP8
// reading of the method, DSA_Q_FP8).  Region-major layout of the work:
//  * a block is 128 regions (the M side: the 128 TMEM lanes) x 64 queries x the group's 4
//    indexer heads (the N side: 256 columns, column 4q + h); the CTA keeps a 64-query tile
//    of codes (256 rows x 256 B = 64 KiB, 128-byte swizzle) resident in smem while 128-region
//    summary blocks (32 KiB) stream through a 4-stage TMA ring;
//  * one thread issues 8 tcgen05.mma kind::f8f6f4 (M = 128, N = 256, K = 32) per block into
//    one of two 256-column TMEM accumulators (512 columns, one CTA per SM).  Large-N
//    instructions matter: the same block cut as 4 heads x (M = 128, N = 64) ran the tensor
//    pipe at a third of the rate;
//  * eight epilogue warps (two per TMEM lane quarter, one per 32-query half) read their
//    128 columns, release the buffer, and for each query form sum_h w_h * ReLU(C) in
//    registers: each thread owns one region, so the head sum stays in the thread, the
//    region's scale is one register (the block's 128 scales arrive with the summaries by
//    TMA), and a warp's 32 lanes write one 128-byte line of a query's score row, masked
//    r < own only on blocks that cross a query's own region;
//  * the blocks (group, query tile, region block) a tile needs (region blocks that start
//    before the tile's largest own region) form one sequence split evenly over a persistent
//    grid.
#pragma once

#include <climits>
#include <type_traits>

#include "common.cuh"

namespace dsa {
namespace gemm {

constexpr int kBM = 128;                 // regions per block (M)
constexpr int kQPerTile = 64;            // queries per tile
constexpr int kHeads = 4;                // indexer heads of a group
constexpr int kBN = kQPerTile * kHeads;  // 256 accumulator columns (N)
constexpr int kQHalf = kBN * 128;        // one 128-byte K column of the query tile (32 KiB)
constexpr int kQBytes = 2 * kQHalf;      // 64 KiB
constexpr int kSHalf = kBM * 128;        // one 128-byte K column of a summary block (16 KiB)
constexpr int kSBytes = 2 * kSHalf;      // 32 KiB
constexpr int kSStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kEpiQueries = kQPerTile * 4 / kEpiWarps;   // queries per epilogue warp (32)
constexpr int kEpiChunks = kEpiQueries / 8;                // 32-column TMEM loads per warp and block
static_assert(kEpiChunks % 2 == 0, "column loads go in pairs");
constexpr int kTmemCols = 512;                  // two 256-column fp32 accumulators
constexpr int kScaleBox = kBM + 4;              // region scales per block, from a 16-byte aligned start
constexpr int kScaleBytes = kScaleBox * 4;      // 528 bytes loaded per block
constexpr int kScaleSlot = 640;                 // slot stride: a TMA destination is 128-byte aligned
constexpr size_t kSmemBytes = 1024 + kQBytes + (size_t)kSStages * (kSBytes + kScaleSlot) +
                              (size_t)kEpiWarps * kEpiQueries * (16 + 4) + 256;
static_assert(kSmemBytes <= 232448, "one CTA per SM");
static_assert(kScaleSlot % 128 == 0 && kScaleSlot >= kScaleBytes, "scale slots");
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
    int n_mtiles;
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
// (-1 and an error for an invalid one) and the largest own region of every query tile.
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
    // the largest own region of every 64-query tile: warp gw takes tile gw (2 queries a lane)
    if (gw < n_mtiles) {
        int m = -1;
#pragma unroll
        for (int i = lane; i < kQPerTile; i += 32) {
            const int q = gw * kQPerTile + i;
            if (q < nq) m = max(m, valid_own(q_req, q_pos, sum_base, ld, n_slots, q));
        }
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) tile_own[gw] = m;
    }
}


// Region blocks tile t needs: those that start before its largest own region.
__device__ __forceinline__ int tile_blocks(const Params &p, int t)
{
    const int o = p.tile_own[t];
    return o > 0 ? (o + kBM - 1) / kBM : 0;
}

// A position in the sequence of blocks (group g, tile t, region block rb), rb fastest.
struct Walk {
    int g, t, rb, nb;
};

__device__ __forceinline__ int64_t total_blocks(const Params &p)
{
    int64_t n = 0;
    for (int t = 0; t < p.n_mtiles; ++t) n += tile_blocks(p, t);
    return n * kG;
}

__device__ __forceinline__ void walk_seek(const Params &p, int64_t idx, Walk &w)
{
    w.g = kG;                                   // past the end unless found
    for (int g = 0; g < kG; ++g)
        for (int t = 0; t < p.n_mtiles; ++t) {
            const int nb = tile_blocks(p, t);
            if (idx < nb) {
                w.g = g;
                w.t = t;
                w.rb = (int)idx;
                w.nb = nb;
                return;
            }
            idx -= nb;
        }
}

__device__ __forceinline__ void walk_next(const Params &p, Walk &w)
{
    if (++w.rb < w.nb) return;
    w.rb = 0;
    do {
        if (++w.t == p.n_mtiles) {
            w.t = 0;
            if (++w.g == kG) return;
        }
        w.nb = tile_blocks(p, w.t);
    } while (w.nb == 0);
}

// This CTA's share [lo, hi) of the block sequence.
__device__ __forceinline__ void cta_range(const Params &p, int64_t &lo, int64_t &hi)
{
    const int64_t total = total_blocks(p);
    lo = total * blockIdx.x / gridDim.x;
    hi = total * (blockIdx.x + 1) / gridDim.x;
}

// 10 warps: 3 share a scheduler's 16K registers, so at most 168 registers per thread
__global__ void __launch_bounds__(kThreads, 1)
    gemm_scores_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_s,
                       const __grid_constant__ CUtensorMap map_sc, const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;                                   // query tile: 2 K columns x [256 rows (q, h)][128 B]
    uint8_t *ss = smem + kQBytes;                         // summary blocks: kSStages x 2 K columns x [128][128 B]
    uint8_t *ssc = ss + kSStages * kSBytes;                                     // [kSStages] scale slots
    float4 *wsm_all = reinterpret_cast<float4 *>(ssc + kSStages * kScaleSlot);  // [warps][pairs][2] weights
    int *own_all = reinterpret_cast<int *>(wsm_all + kEpiWarps * kEpiQueries);  // [warps][queries]
    uint64_t *bars = reinterpret_cast<uint64_t *>(own_all + kEpiWarps * kEpiQueries);
    uint64_t *q_full = bars + 0, *q_empty = bars + 1;
    uint64_t *s_full = bars + 2, *s_empty = bars + 2 + kSStages;                // [kSStages]
    uint64_t *acc_full = bars + 2 + 2 * kSStages, *acc_empty = acc_full + 2;    // [2]
    uint64_t *sc_empty = acc_empty + 2;                                         // [kSStages]
    uint64_t *mma_drain = sc_empty + kSStages;                                  // the MMA issuer's last commit
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_drain + 1);
    static_assert((2 + 3 * kSStages + 4 + 1) * 8 + 4 <= 256, "barriers fit their slot");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], 1);
            mbar_init(&sc_empty[s], kEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);
        }
        mbar_init(mma_drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t base = p.sum_base[0];
    int64_t lo, hi;
    cta_range(p, lo, hi);
    const int64_t n_items = hi - lo;
    bool ok = true;

    if (warp == 0) {
        // ---------------- TMA producer (one lane): the query tile when it changes, then the block
        if (lane == 0 && n_items > 0) {
            prefetch_tensormap(&map_q);
            prefetch_tensormap(&map_s);
            prefetch_tensormap(&map_sc);
            Walk w;
            walk_seek(p, lo, w);
            int cur_g = -1, cur_t = -1, q_loads = 0;
            int64_t issued = 0;                                   // blocks whose loads went out
            for (int64_t it = 0; it < n_items; ++it, walk_next(p, w)) {
                if (w.g != cur_g || w.t != cur_t) {
                    ok = mbar_wait_sleep(q_empty, (q_loads & 1) ^ 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(q_full, kQBytes);
                    // box: 128 B of d x the group's 4 heads x 64 queries -> rows 4q + h
                    tma_load_3d(sq, &map_q, 0, w.g * kHeads, w.t * kQPerTile, q_full);
                    tma_load_3d(sq + kQHalf, &map_q, 128, w.g * kHeads, w.t * kQPerTile, q_full);
                    ++q_loads;
                    cur_g = w.g;
                    cur_t = w.t;
                }
                const int s = (int)(it % kSStages);
                // the slot is free once the MMA has read the summaries and every epilogue
                // warp its scale
                ok = mbar_wait_sleep(&s_empty[s], ((int)(it / kSStages) & 1) ^ 1) &&
                     mbar_wait_sleep(&sc_empty[s], ((int)(it / kSStages) & 1) ^ 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&s_full[s], kSBytes + kScaleBytes);
                const int y = (int)(w.g * p.n_slots + base + (int64_t)w.rb * kBM);
                uint8_t *dst = ss + s * kSBytes;
                tma_load_2d(dst, &map_s, 0, y, &s_full[s]);
                tma_load_2d(dst + kSHalf, &map_s, 128, y, &s_full[s]);
                // scales y .. y + 127 from the 16-byte aligned element y & ~3 (past the pool: 0)
                tma_load_1d(ssc + s * kScaleSlot, &map_sc, y & ~3, &s_full[s]);
                issued = it + 1;
            }
            // drain: none of these loads is in flight when the CTA exits, after a wait that gave
            // up as well (the last phases issued; complete already otherwise)
            if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1);
            for (int s = 0; s < kSStages && s < issued; ++s) {
                const int64_t last = issued - 1 - (issued - 1 - s) % kSStages;
                mbar_wait(&s_full[s], (int)(last / kSStages) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one lane)
        if (lane == 0 && n_items > 0) {
            Walk w;
            walk_seek(p, lo, w);
            int cur_g = -1, cur_t = -1, q_loads = 0;
            for (int64_t it = 0; it < n_items; ++it, walk_next(p, w)) {
                if (w.g != cur_g || w.t != cur_t) {
                    if (q_loads > 0) umma_commit(q_empty);   // the old query tile is free once its MMAs finish
                    ok = mbar_wait_sleep(q_full, q_loads & 1);
                    if (!ok) break;
                    ++q_loads;
                    cur_g = w.g;
                    cur_t = w.t;
                }
                const int s = (int)(it % kSStages), buf = (int)(it & 1);
                ok = mbar_wait_sleep(&s_full[s], (int)(it / kSStages) & 1) &&
                     mbar_wait_sleep(&acc_empty[buf], ((int)(it >> 1) & 1) ^ 1);
                if (!ok) break;
                tc_fence_after();
                // descriptors differ only in the start-address field (16-byte units), which
                // the constant offsets below never carry out of (smem addresses < 256 KiB)
                const uint64_t da = umma_desc_sw128(smem_u32(ss + s * kSBytes)), db = umma_desc_sw128(smem_u32(sq));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off_a = (kk >> 2) * kSHalf + (kk & 3) * 32;
                    const uint32_t off_b = (kk >> 2) * kQHalf + (kk & 3) * 32;
                    umma_e4m3(tmem + buf * kBN, da + (off_a >> 4), db + (off_b >> 4), kIdesc, kk > 0);
                }
                umma_commit(&s_empty[s]);            // the summary block may be overwritten
                umma_commit(&acc_full[buf]);         // the accumulator is ready
            }
            // drain: no MMA of this CTA is in flight when TMEM is released
            umma_commit(mma_drain);
            mbar_wait(mma_drain, 0);
        }
    } else {
        // ---------------- epilogue: warps 2..9.  TMEM lane quarter sp = warp % 4 (the
        // hardware's lane-access rule): regions 32 sp .. 32 sp + 31 of the block, one per
        // thread; query half qq: queries 32 qq .. 32 qq + 31 of the tile (columns 128 qq ..)
        const int e = warp - 2, sp = warp & 3, qq = e >> 2;
        // z * sq / 2 of the 4 heads per query, interleaved by query pair (a, b):
        // wsm[2 i] = {a h0, b h0, a h1, b h1}, wsm[2 i + 1] = {a h2, b h2, a h3, b h3}
        float *wsm = reinterpret_cast<float *>(wsm_all + e * kEpiQueries);
        int *osm = own_all + e * kEpiQueries;             // own region per query (-1: skip)
        if (n_items > 0) {
            Walk w;
            walk_seek(p, lo, w);
            int cur_g = -1, cur_t = -1, own_min = -1;
            const int64_t qstride = (int64_t)kG * p.ld;
            for (int64_t it = 0; it < n_items; ++it, walk_next(p, w)) {
                if (w.g != cur_g || w.t != cur_t) {           // this warp's 16 queries
                    __syncwarp();
                    int o = INT_MAX;
                    if (lane < kEpiQueries) {
                        const int q = w.t * kQPerTile + qq * kEpiQueries + lane;
                        float4 wv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        o = -1;
                        if (q < p.nq) {
                            const int i = q * kHI + w.g * kHeads;
                            wv = make_float4(p.gate[i] * p.qscale[i], p.gate[i + 1] * p.qscale[i + 1],
                                             p.gate[i + 2] * p.qscale[i + 2], p.gate[i + 3] * p.qscale[i + 3]);
                            o = p.q_own[q];
                        }
                        // query lane = 2 i + c of its pair: slots 8 i + 2 h' + c of float4 2 i + h / 2
                        float *wp = wsm + 8 * (lane >> 1) + (lane & 1);
                        wp[0] = 0.5f * wv.x;
                        wp[2] = 0.5f * wv.y;
                        wp[4] = 0.5f * wv.z;
                        wp[6] = 0.5f * wv.w;
                        osm[lane] = o;
                    }
                    // blocks ending at or below every query's own region need no mask (a
                    // query past nq or an invalid one keeps every block masked)
                    own_min = __reduce_min_sync(0xffffffffu, o);
                    __syncwarp();
                    cur_g = w.g;
                    cur_t = w.t;
                }
                const int buf = (int)(it & 1), s = (int)(it % kSStages);
                ok = mbar_wait_sleep(&acc_full[buf], (int)(it >> 1) & 1) &&
                     mbar_wait_sleep(&s_full[s], (int)(it / kSStages) & 1);   // complete already: makes the scales visible
                if (!ok) break;
                tc_fence_after();
                float v[kEpiChunks][32];                          // columns 4q + h of the warp's queries
                {
                    const uint32_t ta = tmem + ((uint32_t)(32 * sp) << 16) + buf * kBN + qq * (kEpiQueries * 4);
#pragma unroll
                    for (int c = 0; c < kEpiChunks; c += 2) tmem_ld32x2(ta + 32 * c, ta + 32 * (c + 1), v[c], v[c + 1]);
                }
                const int64_t y = w.g * p.n_slots + base + (int64_t)w.rb * kBM;
                const float sc =                                  // scale[g][r] / 16
                    reinterpret_cast<const float *>(ssc + s * kScaleSlot)[(int)(y & 3) + 32 * sp + lane] * 0.0625f;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&acc_empty[buf]);              // the MMA may refill this accumulator
                    mbar_arrive(&sc_empty[s]);                 // and the producer this scale slot
                }
                const int r = w.rb * kBM + 32 * sp + lane;     // this thread's region
                // streaming stores (evict first): the 1 GB of scores must not push the
                // summaries, re-read by every query tile, out of L2
                // per query pair (a, b): sum_h w_h / 2 * (v_h + |v_h|) = sum_h w_h ReLU(v_h)
                // (v + |v| is exact), two queries per packed fma
                auto emit = [&](auto masked) {
                    float *dst = p.scores + ((int64_t)(w.t * kQPerTile + qq * kEpiQueries) * kG + w.g) * p.ld + r;
                    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
                    for (int j4 = 0; j4 < kEpiQueries / 4; ++j4) {
                        const int4 o4 = reinterpret_cast<const int4 *>(osm)[j4];
                        const int oj[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
                        for (int u = 0; u < 4; u += 2) {
                            const int j = 4 * j4 + u;                     // queries j, j + 1
                            const float4 w01 = reinterpret_cast<const float4 *>(wsm)[j];
                            const float4 w23 = reinterpret_cast<const float4 *>(wsm)[j + 1];
                            const float *va = &v[j / 8][4 * (j % 8)];
                            const float *vb = va + 4;
                            float2 acc = fmul2(make_float2(va[0] + fabsf(va[0]), vb[0] + fabsf(vb[0])),
                                               make_float2(w01.x, w01.y));
                            acc = ffma2(make_float2(va[1] + fabsf(va[1]), vb[1] + fabsf(vb[1])),
                                        make_float2(w01.z, w01.w), acc);
                            acc = ffma2(make_float2(va[2] + fabsf(va[2]), vb[2] + fabsf(vb[2])),
                                        make_float2(w23.x, w23.y), acc);
                            acc = ffma2(make_float2(va[3] + fabsf(va[3]), vb[3] + fabsf(vb[3])),
                                        make_float2(w23.z, w23.w), acc);
                            acc = fmul2(acc, sc2);
                            // streaming stores (evict first): the 1 GB of scores must not push
                            // the summaries, re-read by every query tile, out of L2
                            if (!decltype(masked)::value || r < oj[u]) __stcs(dst, acc.x);
                            if (!decltype(masked)::value || r < oj[u + 1]) __stcs(dst + qstride, acc.y);
                            dst += 2 * qstride;
                        }
                    }
                };
                if (w.rb * kBM + kBM <= own_min)
                    emit(std::integral_constant<bool, false>());
                else
                    emit(std::integral_constant<bool, true>());
            }
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
