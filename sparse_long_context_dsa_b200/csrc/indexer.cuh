// A2 indexer scores: score[q][g][r] = sum_{h=4g}^{4g+3} z_h ReLU(q_h . s_{r,g}) / 16
// ([P1] kwkr.cn/news/601179 §DSA ③; [P2] Step-5-Preview 如何实现1M长上下文 §索引器打分:
// the 16-head indexer scores the query against every region summary of its request).
//
// The scan streams the request's e4m3 summaries once (256 B per region and group: the
// dominant HBM traffic of a decode step) and is built to run at HBM speed:
//  * one producer warp issues TMA tile loads (2-D tensor map over the group-major pool,
//    128-byte swizzle, no multicast) of four 32-region x 256 B slabs = 32 KiB per stage
//    into a ring of smem stages guarded by mbarriers.  A query's slabs are its (32-region
//    chunk, KV group) pairs in chunk-major order: with all 4 groups a stage is one chunk of
//    every group; a call that holds fewer groups (a GPU of a KV-group-sharded decode, 1 or 2
//    groups) packs 4 or 2 chunks per stage, so the consumers stay as busy;
//  * four consumer warps, one per slab (warp w always meets local group w % groups), read
//    their 32x256 tile with conflict-free ldmatrix and contract it on the tensor cores with
//    mma.sync m16n8k32 e4m3, fp32 accumulate.  A fp32 FFMA dot product would need 4 FMA per summary byte plus e4m3
//    conversions and run out of ALU before HBM; on the tensor pipe the summaries are fed
//    as raw bytes;
//  * the B operand (8 columns) holds the group's 4 heads, each split exactly into two
//    e4m3 parts: q_h / sq_h = hi + lo with sq_h a power of two, hi = e4m3(q/sq),
//    lo = e4m3(q/sq - hi).  A bf16 value has 8 significant bits, hi carries 4 and lo the
//    rest, so the product is the bf16 query's to within e4m3 subnormal resolution of the
//    smallest components (relative 2^-17 of the head's largest value).  With DSA_Q_FP8
//    the query is instead quantised once per head with sq = absmax/448 (lo = 0), the
//    FP8 x FP8 reading of the method;
//  * epilogue: dot = (hi + lo) * sq * scale_r, ReLU, gate, sum over the 4 heads with two
//    shuffles, / 16, masked to r < own;
//  * work assignment: CTA b takes the stage units b, b + G, b + 2G, ... (G CTAs), so at any
//    moment the grid streams one dense window of each group's summaries; with one contiguous
//    range per CTA the CTAs ended up to 7 us apart in a 1M-token decode step (the last one
//    decides when the selection starts), interleaved 5 us, and the scan took 22.1 instead
//    of 23.1 us.
#pragma once

#include "common.cuh"

namespace dsa {
namespace idx {

// Pipeline shape (compile-time tunables; the defaults are the measured best on B200).
#ifndef DSA_SCAN_STAGES
#define DSA_SCAN_STAGES 2
#endif
#ifndef DSA_SCAN_CTAS_PER_SM
#define DSA_SCAN_CTAS_PER_SM 2
#endif
#ifndef DSA_SCAN_CHUNK
#define DSA_SCAN_CHUNK 32
#endif
#ifndef DSA_SCAN_L2_PROMOTION
#define DSA_SCAN_L2_PROMOTION 3          // CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif
constexpr int kChunk = DSA_SCAN_CHUNK;             // regions per stage (multiple of 32)
constexpr int kStages = DSA_SCAN_STAGES;
constexpr int kCtasPerSm = DSA_SCAN_CTAS_PER_SM;
constexpr int kSlabs = 4;                          // 32-region slabs per stage (= consumer warps)
constexpr int kHalfBytes = kChunk * 128;           // one 128-byte column half of a slab
constexpr int kGroupBytes = 2 * kHalfBytes;        // one slab: 8 KiB at 32 regions
constexpr int kStageBytes = kSlabs * kGroupBytes;  // 32 KiB at 32 regions
constexpr int kTiles = kChunk / 16;                // m16 tiles per group per stage
constexpr int kThreads = 160;                      // 4 consumer warps + 1 producer warp
constexpr int kScaleBytes = kSlabs * kChunk * 4;   // fp32 scales of one stage (512 B)
constexpr size_t kSmemBytes =
    (size_t)kStages * (kStageBytes + kScaleBytes) + 1024 /*align*/ + 64 /*barriers*/;

struct Params {
    const __nv_bfloat16 *index_q;
    const float *gate;
    const int32_t *q_req;
    const int32_t *q_pos;
    const float *scales;
    const int64_t *sum_base;
    float *scores;
    float *chunk_max;          // nullable: [nq][4][cm_stride], largest stored score of regions 32c .. 32c+31
    int64_t cm_stride;
    int64_t n_slots;
    int64_t ld;
    int64_t total_units;
    int units_per_query;       // stages per query: ceil(chunks * groups / 4)
    int nq;
    int n_req;
    uint32_t flags;
    // KV groups of the call: g0 .. g0 + groups - 1 (groups 1, 2 or 4).  summaries / scales
    // hold only these groups ([groups][n_slots][256]); scores and chunk_max are
    // [nq][groups][..]; index_q and gate are the full [nq][16][..] (heads 4g .. 4g + 3).
    int groups;
    int gshift;                // log2(groups)
    int g0;
};

// Slab j of stage unit `uu` of a query: its 32-region chunk and local group.
__device__ __forceinline__ void slab_of(const Params &p, int uu, int j, int &chunk, int &gl)
{
    const int sidx = uu * kSlabs + j;
    chunk = sidx >> p.gshift;
    gl = sidx & (p.groups - 1);
}

// Checks one query; returns own (regions before the own region) or -1 if the query is
// invalid.  base receives the request's first slot.
__device__ __forceinline__ int64_t query_own(const Params &p, int qi, int64_t &base)
{
    const int b = p.q_req[qi];
    const int pos = p.q_pos[qi];
    if (b < 0 || b >= p.n_req || pos < 0) return -1;
    const int64_t own = pos / kRegion;
    base = p.sum_base[b];
    if (own > p.ld || base < 0 || base + own > p.n_slots) return -1;
    return own;
}

// B fragments of the group's 4 heads for mma m16n8k32: lane (n = lane/4, t = lane%4)
// holds column n = 2*head + part, k-rows 32j+4t..+3 (b0) and 32j+16+4t..+3 (b1).
__device__ __forceinline__ void load_query_fragments(const Params &p, int qi, int g, int lane, uint32_t (&b)[8][2],
                                                     float &sq_t, float &z_t)
{
    const int n = lane >> 2, t = lane & 3;
    const int head = g * 4 + (n >> 1), part = n & 1;
    const __nv_bfloat16 *qh = p.index_q + ((int64_t)qi * kHI + head) * kDI;
    float x[8][8];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint2 lo4 = __ldg(reinterpret_cast<const uint2 *>(qh + 32 * j + 4 * t));
        const uint2 hi4 = __ldg(reinterpret_cast<const uint2 *>(qh + 32 * j + 16 + 4 * t));
        x[j][0] = bf16_lo(lo4.x); x[j][1] = bf16_hi(lo4.x); x[j][2] = bf16_lo(lo4.y); x[j][3] = bf16_hi(lo4.y);
        x[j][4] = bf16_lo(hi4.x); x[j][5] = bf16_hi(hi4.x); x[j][6] = bf16_lo(hi4.y); x[j][7] = bf16_hi(hi4.y);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[j][e]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));

    float sq;
    if (p.flags & 1u) {
        // FP8 query: one e4m3 code per value, scale absmax/448 (IEEE division), lo = 0
        sq = __fdiv_rn(amax, 448.0f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t c[4] = {0, 0, 0, 0};
            if (sq != 0.0f && part == 0) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    c[e] = cvt_e4m3x2(__fdiv_rn(x[j][2 * e], sq), __fdiv_rn(x[j][2 * e + 1], sq));
            }
            b[j][0] = c[0] | (c[1] << 16);
            b[j][1] = c[2] | (c[3] << 16);
        }
    } else {
        // exact split: sq = 2^(e-8) with amax < 2^e, so |q/sq| < 256 and q/sq is exact
        int e = 0;
        if (amax > 0.0f) frexpf(amax, &e);
        const float inv = (amax > 0.0f) ? ldexpf(1.0f, 8 - e) : 1.0f;
        sq = (amax > 0.0f) ? ldexpf(1.0f, e - 8) : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t c[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const float v0 = x[j][2 * e2] * inv, v1 = x[j][2 * e2 + 1] * inv;
                const uint32_t h = cvt_e4m3x2(v0, v1);
                if (part == 0) {
                    c[e2] = h;
                } else {
                    const float r0 = v0 - e4m3_to_f32(h & 0xFF);
                    const float r1 = v1 - e4m3_to_f32(h >> 8);
                    c[e2] = cvt_e4m3x2(r0, r1);
                }
            }
            b[j][0] = c[0] | (c[1] << 16);
            b[j][1] = c[2] | (c[3] << 16);
        }
    }
    // epilogue constants of head t of the group: sq from lane 8t (column 2t), gate
    sq_t = __shfl_sync(0xffffffffu, sq, 8 * t);
    z_t = __ldg(p.gate + (int64_t)qi * kHI + g * 4 + t);
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    scan_kernel(const __grid_constant__ CUtensorMap tmap, const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    // the tensor map is a kernel parameter: its descriptor is fetched while the previous
    // kernel finishes, not in front of the first stage's loads
    if (threadIdx.x == 32 * kSlabs) prefetch_tensormap(&tmap);
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *sscale = reinterpret_cast<float *>(smem + kStages * kStageBytes);      // [kStages][4][32]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * (kStageBytes + kScaleBytes));
    uint64_t *empty = full + kStages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1 + 32);   // expect_tx arrive + one arrive per producer lane (scales)
            mbar_init(&empty[s], kSlabs);
        }
        fence_mbar_init();
    }
    __syncthreads();


    if (warp == kSlabs) {
        // ---------------- producer warp: lane 0 issues the TMA loads of the summaries; every
        // lane copies 4 of the stage's 128 fp32 scales into smem asynchronously
        const uint64_t pol = l2_evict_first_policy();     // the summaries are read once per query
        int it = 0;
        constexpr int kScalesPerLane = kSlabs * kChunk / 32;      // 4 at 32 regions per stage
        const int sg = (lane * kScalesPerLane) / kChunk, sr = (lane * kScalesPerLane) % kChunk;
        for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x) {
            const int qi = (int)(u / p.units_per_query);
            const int uu = (int)(u - (int64_t)qi * p.units_per_query);
            int64_t base;
            const int64_t own = query_own(p, qi, base);
            int c_first;
            int gl_first;
            slab_of(p, uu, 0, c_first, gl_first);
            if (own < 0 || (int64_t)c_first * kChunk >= own) continue;
            const int s = it % kStages;
            const unsigned ph = (unsigned)(it / kStages) & 1u;
            if (!mbar_wait(&empty[s], ph ^ 1u)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                uint8_t *st = smem + s * kStageBytes;
#pragma unroll
                for (int j = 0; j < kSlabs; ++j) {
                    // slabs past the own region (the last stage of a query) are loaded and ignored
                    int c;
                    int gl;
                    slab_of(p, uu, j, c, gl);
                    const int y = (int)(gl * p.n_slots + base + (int64_t)c * kChunk);
                    tma_load_2d_hint(st + j * kGroupBytes, &tmap, 0, y, &full[s], pol);
                    tma_load_2d_hint(st + j * kGroupBytes + kHalfBytes, &tmap, 128, y, &full[s], pol);
                }
            }
            // scales: asynchronous 4-byte copies that arrive on the stage's barrier when they
            // land, so the producer never waits for them
            int c;
            int gl;
            slab_of(p, uu, sg, c, gl);
            const float *srow = p.scales + gl * p.n_slots + base;
#pragma unroll
            for (int e = 0; e < kScalesPerLane; ++e) {
                const int64_t r = (int64_t)c * kChunk + sr + e;
                cp_async_4(sscale + (s * kSlabs + sg) * kChunk + sr + e, srow + (r < own ? r : 0), r < own);
            }
            cp_async_mbar_arrive(&full[s]);
            ++it;
        }
        return;
    }

    // ---------------- consumers: warp j contracts slab j (local group j % groups)
    const int g = warp % p.groups;
    const int n = lane >> 2, t = lane & 3;
    uint32_t bfrag[8][2];
    float sq_t = 0.0f, z_t = 0.0f;
    int cached_q = -1;
    int it = 0;
    for (int64_t u = blockIdx.x; u < p.total_units; u += gridDim.x) {
        const int qi = (int)(u / p.units_per_query);
        const int uu = (int)(u - (int64_t)qi * p.units_per_query);
        int64_t base;
        const int64_t own = query_own(p, qi, base);
        if (own < 0) {
            if (uu == 0 && warp == 0 && lane == 0) set_error(kErrIndexerQuery);
            continue;
        }
        int c_first;
        int gl_first;
        slab_of(p, uu, 0, c_first, gl_first);
        if ((int64_t)c_first * kChunk >= own) continue;
        int chunk;
        int gl;
        slab_of(p, uu, warp, chunk, gl);
        const int64_t r0 = (int64_t)chunk * kChunk;
        if (qi != cached_q) {
            load_query_fragments(p, qi, p.g0 + g, lane, bfrag, sq_t, z_t);
            cached_q = qi;
        }
        const int s = it % kStages;
        const unsigned ph = (unsigned)(it / kStages) & 1u;
        if (!mbar_wait(&full[s], ph)) break;
        // scales of this lane's 4 rows (tile m: rows n and n+8), staged by the producer
        float sc[kTiles][2];
#pragma unroll
        for (int m = 0; m < kTiles; ++m)
#pragma unroll
            for (int h = 0; h < 2; ++h) sc[m][h] = sscale[(s * kSlabs + warp) * kChunk + 16 * m + 8 * h + n];
        const uint32_t tile = smem_u32(smem + s * kStageBytes + warp * kGroupBytes);
        float acc[kTiles][4];
#pragma unroll
        for (int m = 0; m < kTiles; ++m) {
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][e] = 0.0f;
            // ldmatrix.x4: lane l addresses row (16m + 8*((l>>3)&1) + (l&7)), 16-byte chunk
            // 2*(j%4) + (l>>4) of column half j/4; 128-byte swizzle XORs the chunk with row&7
            const int row = 16 * m + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int chunk = 2 * (j & 3) + (lane >> 4);
                const uint32_t addr = tile + (j >> 2) * kHalfBytes + row * 128 + ((chunk ^ (row & 7)) << 4);
                uint32_t a[4];
                ldmatrix_x4(addr, a[0], a[1], a[2], a[3]);
                mma_e4m3_16832(acc[m], a, bfrag[j][0], bfrag[j][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        ++it;
        if (r0 >= own) continue;                              // a slab past the own region

        float *out = p.scores + ((int64_t)qi * p.groups + g) * p.ld;
        float cmax = -1.0f;                                   // below every score (scores are >= +0)
#pragma unroll
        for (int m = 0; m < kTiles; ++m) {
            float v0 = z_t * fmaxf((acc[m][0] + acc[m][1]) * sq_t * sc[m][0], 0.0f);
            float v1 = z_t * fmaxf((acc[m][2] + acc[m][3]) * sq_t * sc[m][1], 0.0f);
            v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
            v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
            if (t < 2) {
                const int64_t r = r0 + 16 * m + 8 * t + n;
                const float v = (t == 0 ? v0 : v1) * 0.0625f;
                if (r < own) {
                    out[r] = v;
                    cmax = fmaxf(cmax, v);
                }
            }
        }
        if (p.chunk_max) {                                    // the chunk's largest stored score
            static_assert(kChunk == 32, "chunk maxima cover 32 regions");
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
            if (lane == 0) p.chunk_max[((int64_t)qi * p.groups + g) * p.cm_stride + r0 / kChunk] = cmax;
        }
    }
}

}  // namespace idx
}  // namespace dsa
