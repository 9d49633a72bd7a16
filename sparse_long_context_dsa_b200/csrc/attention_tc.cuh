// A4 sparse GQA attention for prefill blocks whose queries share their selections, on the
// tcgen05 tensor cores ([P1] kwkr.cn/news/601179 §DSA ④; [P5] Stepfun … Step 5 Preview:
// neighbouring queries reuse one selection).
//
// A CTA takes 8 consecutive queries of one request and one KV group: 128 rows (query, head) of
// one attention tile.  The union of their selections is built in smem (a region bitmap,
// compacted in region order; the running count per bitmap word gives each selected region its
// union position) together with each union region's 8-bit membership (which queries selected
// it) and one bit per tile that needs no mask (every query selected all its regions, all at or
// before the earliest position).  The union streams in tiles of 8 regions (64 tokens),
// flash-attention style:
//  * two TMA warps load each region's K (one warp) and V (the other) as ONE 3 KiB box of a
//    3-D view of the cache whose dimensions are the 64 dims of a block, the token rows and the
//    3 blocks (block stride 128 B below the row stride 384 B), so that it lands as [block]
//    [8 rows][128 B] with the 128-byte swizzle (8-token atoms 3 KiB apart), into separate
//    4-stage rings: a K stage frees as soon as S has read it, a V stage once P V has; a region
//    that is invalid or past the union is loaded from rows past the cache, which fill zeros;
//  * one thread issues S = Q K^T (M = 128, N = 64, K = 192: 12 tcgen05.mma.kind::f16, Q
//    read from TMEM where the softmax warps put it at the start) into one of two 64-column
//    TMEM buffers, and O += P V (M = 128, N = 192, K = 64: 4 MMAs with
//    P read from TMEM and V an MN-major smem operand) into a 192-column TMEM accumulator;
//    S runs two tiles ahead of P V, so the tensor pipe has S queued while a softmax runs;
//  * eight softmax warps, two per row (one row per thread, the TMEM lane; one warp takes the
//    tile's first 32 tokens, the other the last 32, and the two agree on the row's running
//    max through smem each tile), mask the tile (the region must be the row's query's, the
//    token at or before its position), keep the online softmax in exp2 with lazy rescaling
//    (the reference max moves only past a slack of 2^8; O is rescaled in TMEM then), write P
//    as packed bf16 into TMEM (two tokens per column, the A operand of P V), and at the end
//    write O / l and the LSE.
// Every wait is bounded; after the loops the producers wait for their last loads and the MMA
// issuer for a final commit, so nothing is in flight when TMEM is released.
// Blocks spanning several requests, with an invalid query, or whose union exceeds twice the
// longest selection are flagged in row_shared and left to the per-row kernel that runs next.
#pragma once

#include <climits>

#include "attention.cuh"
#include "topk_cluster.cuh"

namespace dsa {
namespace attntc {

using attn::Params;

constexpr int kQueries = 8;                          // queries per CTA: 8 x 16 heads = 128 rows
constexpr int kThreads = 384;                        // warp 0 K loads, 1 MMA, 2 V loads, 4..11 softmax
constexpr int kMaxK = 512;                           // selection length per query
constexpr int kMaxUnion = 2 * kMaxK;                 // a longer union is not shared
constexpr int kMaxWords = 8192;                      // bitmap words: regions < 262,144
constexpr int kTileRegions = 8;                      // regions per tile: 64 tokens
constexpr int kRegionBox = 3 * 8 * 128;              // one region of K or V: [3 blocks][8 rows][128 B]
constexpr int kTileBytes = kTileRegions * kRegionBox;        // 24 KiB: K or V of one tile
constexpr int kStages = 4;                                   // per ring (K and V)
// smem layout (bytes, after 1024-byte alignment)
constexpr size_t kOffK = 0;                                          // kStages K tiles
constexpr size_t kOffV = kOffK + (size_t)kStages * kTileBytes;       // kStages V tiles
constexpr size_t kOffUni = kOffV + (size_t)kStages * kTileBytes;     // [kMaxUnion] region ids
constexpr size_t kOffRow = kOffUni + (size_t)kMaxUnion * 4;          // [kMaxUnion] cache rows (TMA y)
constexpr size_t kOffMask = kOffRow + (size_t)kMaxUnion * 4;         // [kMaxUnion / 4] membership bytes
constexpr size_t kOffXch = kOffMask + (size_t)kMaxUnion;             // [2 buffers][2 halves][128 rows] f32
constexpr size_t kOffBars = kOffXch + 2 * 2 * 128 * 4;
constexpr size_t kSmemBytes = 1024 + kOffBars + 512;
// set-up scratch, overlaid on the K/V rings (used before the first load)
constexpr size_t kOffBitmap = kOffK;                                 // [kMaxWords]
constexpr size_t kOffSel = kOffBitmap + (size_t)kMaxWords * 4;       // [8][kMaxK]
constexpr size_t kOffRank = kOffSel + (size_t)kQueries * kMaxK * 4;  // [kMaxWords] union rank of each word's first bit
static_assert(kOffRank + (size_t)kMaxWords * 4 <= kOffUni, "set-up scratch fits the rings");
static_assert(kSmemBytes <= 232448, "one CTA per SM");
// TMEM columns: S at 0 and 64; Q (192 bf16 dims, two per column) at 128; P (64 bf16 tokens
// in 32 columns) at 224 and 256; O at 288
constexpr int kTmemCols = 512;
constexpr int kQCol = 128;
constexpr int kPCol = 224;
constexpr int kOCol = 288;
static_assert(kOCol + kD <= kTmemCols, "TMEM map fits");

// kind::f16 instruction descriptor: BF16 x BF16 -> F32; b_mn: B operand MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor (128-byte swizzle) in two 32-bit halves: lo = start
// address >> 4 | LBO >> 4 << 16 (the start address of a later tile is lo + byte offset / 16,
// no carry below 256 KiB), hi = SBO >> 4 | version (sm_100) | layout.
__device__ __forceinline__ uint32_t desc_lo(uint32_t smem_addr, uint32_t lbo)
{
    return ((smem_addr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t desc_hi(uint32_t sbo) { return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29); }

// tcgen05.mma kind::f16 with A from TMEM and B from smem (descriptor halves), the accumulate
// flag an immediate: the issuing thread spends a handful of instructions per MMA.
template <bool kAccumulate>
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi, uint32_t idesc)
{
    const uint64_t b = ((uint64_t)b_hi << 32) | b_lo;
    if constexpr (kAccumulate)
        asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 1;" ::"r"(d_tmem), "r"(a_tmem), "l"(b),
                     "r"(idesc)
                     : "memory");
    else
        asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 0;" ::"r"(d_tmem), "r"(a_tmem), "l"(b),
                     "r"(idesc)
                     : "memory");
}

// hardware base-2 exponential (ex2.approx, flush-to-zero); ex2(-inf) = +0
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes written from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
          "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]),
          "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]),
          "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes written from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
          "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// tmap_k / tmap_v: 3-D views (64 dims, n_pages * 4 * 64 rows, 3 blocks) of the caches, box
// {64, 8, 3} (one region), 128-byte swizzle.  kv_rows: the views' row count (a load there
// reads zeros).
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                          const Params p, int kv_rows)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ks = smem + kOffK;
    uint8_t *vs = smem + kOffV;
    int32_t *uni = reinterpret_cast<int32_t *>(smem + kOffUni);
    int32_t *urow = reinterpret_cast<int32_t *>(smem + kOffRow);
    uint32_t *umask = reinterpret_cast<uint32_t *>(smem + kOffMask);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + kOffBitmap);
    int32_t *sels = reinterpret_cast<int32_t *>(smem + kOffSel);
    uint32_t *rank = reinterpret_cast<uint32_t *>(smem + kOffRank);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBars);
    uint64_t *k_full = bars, *k_empty = bars + kStages, *v_full = bars + 2 * kStages, *v_empty = bars + 3 * kStages;
    uint64_t *s_full = bars + 4 * kStages, *s_empty = s_full + 2, *p_full = s_full + 4, *p_free = s_full + 6;
    // o_done[j & 1] completes when P V of tile j has (and with it every earlier MMA): two
    // barriers, since P V runs two tiles behind S and a waiter must be at most one phase behind
    uint64_t *o_done = s_full + 8;
    uint64_t *x_full = o_done + 2;                        // [4 quarters][2 buffers]
    uint64_t *q_ready = x_full + 8;
    uint64_t *mma_drain = q_ready + 1;                    // the MMA issuer's last commit
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_drain + 1);
    static_assert((4 * kStages + 20) * 8 + 4 <= 512, "barriers fit their slot");
    float *xch = reinterpret_cast<float *>(smem + kOffXch);
    __shared__ uint32_t scan_ws[40];
    __shared__ int sh_req[kQueries], sh_pos[kQueries], sh_cnt[kQueries], sh_own[kQueries];
    __shared__ int sh_U;
    __shared__ uint32_t sh_whole[kMaxUnion / kTileRegions / 32];   // bit i: tile i needs no mask

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    // group-major block order: the CTAs resident together gather from one group's cache
    const int n_qblocks = (int)gridDim.x / kG;
    const int g = (int)blockIdx.x / n_qblocks;
    const int q0 = ((int)blockIdx.x - g * n_qblocks) * kQueries;
    // softmax threads (warps 4..11) fetch their Q row half now; it goes to TMEM after set-up
    uint4 qreg[12];
    if (warp >= 4) {
        const int r = (warp & 3) * 32 + lane, q = q0 + (r >> 4);
        const uint4 *src = reinterpret_cast<const uint4 *>(
            p.q + ((int64_t)q * kHQ + g * kHeadsPerGroup + (r & 15)) * kD + ((warp - 4) >> 2) * 96);
#pragma unroll
        for (int k = 0; k < 12; ++k) qreg[k] = q < p.nq ? __ldg(src + k) : make_uint4(0u, 0u, 0u, 0u);
    }

    // ---- the block's queries: request, position, own region, selection count
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
        sh_own[tid] = pos >= 0 ? pos / kRegion : -1;
        sh_cnt[tid] = req >= 0 ? c : 0;
    }
    __syncthreads();
    // served here: every query of the block valid and of one request, and a small union
    int R = -1, maxc = 0, max_own = -1;
    bool share = true;
    for (int w = 0; w < kQueries; ++w) {
        if (q0 + w >= p.nq) continue;
        if (sh_req[w] < 0 || (R >= 0 && sh_req[w] != R)) share = false;
        R = sh_req[w];
        maxc = max(maxc, sh_cnt[w]);
        max_own = max(max_own, sh_own[w]);
    }
    share = share && R >= 0 && maxc > 0;
    const int words = share ? min(kMaxWords, (max_own + 1 + 31) / 32) : 0;
    if (share) {
        // ---- the union of the selections (region bitmap), each query's entries kept
        for (int i = tid; i < words; i += kThreads) bitmap[i] = 0u;
        __syncthreads();
        if (warp < kQueries && q0 + warp < p.nq) {
            const int c = sh_cnt[warp];
            const int32_t *src = p.sel_idx + ((int64_t)(q0 + warp) * kG + g) * p.k;
            int rv[kMaxK / 32];                             // all loads in flight at once
#pragma unroll
            for (int k = 0; k < kMaxK / 32; ++k) rv[k] = lane + 32 * k < c ? __ldg(src + lane + 32 * k) : -1;
#pragma unroll
            for (int k = 0; k < kMaxK / 32; ++k) {
                const int i = lane + 32 * k;
                if (i >= c) break;
                int r = rv[k];
                if (r < 0 || r > sh_own[warp] || r / 8 >= p.max_pages || (r >> 5) >= words) {
                    set_error(kErrAttnIndex);
                    r = -1;
                }
                sels[warp * kMaxK + i] = r;
                if (r >= 0) atomicOr(&bitmap[r >> 5], 1u << (r & 31));
            }
        }
        __syncthreads();
        const int wpt = (words + kThreads - 1) / kThreads;
        const int w0 = tid * wpt;
        uint32_t n = 0;
        for (int i = 0; i < wpt; ++i)
            if (w0 + i < words) n += __popc(bitmap[w0 + i]);
        const uint32_t incl = topkc::block_scan_incl<kThreads>(n, scan_ws);
        const uint32_t total = scan_ws[kThreads / 32 - 1];
        share = total > 0 && total <= 2u * (uint32_t)maxc && total <= (uint32_t)kMaxUnion;
        if (share) {
            uint32_t pos = incl - n;
            for (int i = 0; i < wpt; ++i) {
                if (w0 + i >= words) break;
                rank[w0 + i] = pos;
                uint32_t b = bitmap[w0 + i];
                while (b) {
                    const int bit = __ffs(b) - 1;
                    b &= b - 1;
                    uni[pos++] = (w0 + i) * 32 + bit;
                }
            }
        }
        if (tid == 0) sh_U = (int)total;
        __syncthreads();
    }
    if (p.row_shared && tid < kQueries && q0 + tid < p.nq) p.row_shared[(int64_t)(q0 + tid) * kG + g] = share ? 1 : 0;
    if (!share) return;                                   // block-uniform: the per-row kernel serves it
    const int U = sh_U;
    // ---- each union region's first cache row (through the block table, all lookups in flight
    // at once; a bad page reads zeros), and membership: bit 8 (u % 4) + w of word u / 4 when
    // query w selected union region u, whose union rank comes from the bitmap
    static_assert(3 * kThreads >= kMaxUnion, "three block-table lookups per thread");
    {
        int64_t page[3];
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int u = tid + k * kThreads;
            page[k] = u < U ? __ldg(p.block_table + (int64_t)R * p.max_pages + uni[u] / 8) : 0;
        }
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int u = tid + k * kThreads;
            if (u >= U) break;
            int y = kv_rows;
            if (page[k] >= 0 && page[k] < p.n_pages)
                y = (int)((page[k] * kG + g) * kPage + (uni[u] % 8) * kRegion);
            else
                set_error(kErrAttnIndex);
            urow[u] = y;
        }
    }
    for (int i = tid; i < (U + 3) / 4; i += kThreads) umask[i] = 0u;
    __syncthreads();
    if (warp < kQueries && q0 + warp < p.nq) {
        const int c = sh_cnt[warp];
        for (int i = lane; i < c; i += 32) {
            const int r = sels[warp * kMaxK + i];
            if (r < 0) continue;
            const uint32_t b = bitmap[r >> 5];
            const int u = (int)(rank[r >> 5] + __popc(b & ((1u << (r & 31)) - 1u)));
            atomicOr(&umask[u >> 2], 1u << ((u & 3) * 8 + warp));
        }
    }
    __syncthreads();
    // ---- tiles that need no mask: all 8 regions in the union, selected by every query of the
    // block, and wholly at or before the earliest position
    if (warp < kMaxUnion / kTileRegions / 32) {
        uint32_t qmask = 0u;
        int min_pos = INT_MAX;
        for (int w = 0; w < kQueries; ++w)
            if (q0 + w < p.nq) {
                qmask |= 1u << w;
                min_pos = min(min_pos, sh_pos[w]);
            }
        const int t = warp * 32 + lane;
        bool whole = (t + 1) * kTileRegions <= U;
        for (int jr = 0; jr < kTileRegions && whole; ++jr) {
            const int u = t * kTileRegions + jr;
            whole = ((umask[u >> 2] >> ((u & 3) * 8)) & qmask) == qmask && uni[u] * kRegion + kRegion - 1 <= min_pos;
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, whole);
        if (lane == 0) sh_whole[warp] = bits;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_empty[b], 8);
            mbar_init(&p_full[b], 8);
            mbar_init(&p_free[b], 1);
        }
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        for (int b = 0; b < 8; ++b) mbar_init(&x_full[b], 2);
        mbar_init(q_ready, 8);
        mbar_init(mma_drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    fence_proxy_async();                                  // the reused scratch, for the async proxy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_tiles = (U + kTileRegions - 1) / kTileRegions;
    bool ok = true;

    if (warp == 0 || warp == 2) {
        // ---------------- TMA producers: warp 0 loads K, warp 2 loads V; lane j < 8 issues
        // region j of each tile (one 3 KiB box)
        const bool is_k = warp == 0;
        const CUtensorMap *map = is_k ? &tmap_k : &tmap_v;
        uint8_t *ring = is_k ? ks : vs;
        uint64_t *full = is_k ? k_full : v_full, *empty = is_k ? k_empty : v_empty;
        if (lane == 0) prefetch_tensormap(map);
        int issued = 0;                                   // tiles whose loads went out
        for (int i = 0; i < n_tiles && ok; ++i) {
            const int s = i % kStages;
            int got = 1;
            if (lane == 0) {
                got = mbar_wait_sleep(&empty[s], ((i / kStages) & 1) ^ 1) ? 1 : 0;
                if (got) mbar_arrive_expect_tx(&full[s], kTileBytes);
            }
            ok = __shfl_sync(0xffffffffu, got, 0) != 0;
            if (!ok) break;
            if (lane < kTileRegions) {
                const int u = i * kTileRegions + lane;
                const int y = u < U ? urow[u] : kv_rows;        // past the union: zeros
                uint8_t *dst = ring + s * kTileBytes + lane * kRegionBox;
                tma_load_3d(dst, map, 0, y, 0, &full[s]);
            }
            issued = i + 1;
        }
        // drain: none of this warp's loads is in flight when the CTA exits, after a wait that
        // gave up as well (the last phase issued into every stage; complete already otherwise)
        __syncwarp();
        if (lane == 0)
            for (int s = 0; s < kStages && s < issued; ++s) {
                const int last = issued - 1 - (issued - 1 - s) % kStages;
                mbar_wait(&full[s], (last / kStages) & 1);
            }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one lane): S(i), then O += P(i-2) V(i-2): S runs two tiles
        // ahead, so that the tensor pipe has S(i) queued while the softmax of tile i-1 runs
        if (lane == 0) {
            constexpr uint32_t kIdS = idesc_bf16(128, 64, false), kIdO = idesc_bf16(128, kD, true);
            // K: K-major, 8-token atoms 3 KiB apart; V: MN-major, 64-dim blocks 1 KiB apart
            const uint32_t k_lo0 = desc_lo(smem_u32(ks), 16), v_lo0 = desc_lo(smem_u32(vs), 1024);
            constexpr uint32_t kHi = desc_hi(kRegionBox);
            ok = mbar_wait(q_ready, 0);                   // Q in TMEM
            auto issue_pv = [&](int j) {
                const int s = j % kStages, pb = j & 1;
                ok = ok && mbar_wait(&p_full[pb], (j >> 1) & 1) &&
                     mbar_wait(&v_full[s], (j / kStages) & 1);
                if (!ok) return;
                tc_fence_after();
                const uint32_t vlo = v_lo0 + (uint32_t)s * (kTileBytes >> 4);
                const uint32_t pa = tmem + kPCol + pb * 32;
                // 16 tokens (two regions) per instruction
                if (j > 0) mma_ts<true>(tmem + kOCol, pa, vlo, kHi, kIdO);
                else mma_ts<false>(tmem + kOCol, pa, vlo, kHi, kIdO);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk)
                    mma_ts<true>(tmem + kOCol, pa + kk * 8, vlo + kk * (2 * kRegionBox >> 4), kHi, kIdO);
                umma_commit(&p_free[pb]);                       // P(j) read
                umma_commit(&v_empty[s]);                       // V(j) read
                umma_commit(&o_done[j & 1]);                    // O holds the tiles up to j
            };
            for (int i = 0; i < n_tiles + 2 && ok; ++i) {
                if (i >= n_tiles) {                             // the last two P V
                    if (i >= 2) issue_pv(i - 2);
                    continue;
                }
                const int s = i % kStages, sb = i & 1;
                ok = mbar_wait(&k_full[s], (i / kStages) & 1) &&
                     mbar_wait(&s_empty[sb], ((i >> 1) & 1) ^ 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t klo = k_lo0 + (uint32_t)s * (kTileBytes >> 4), sd = tmem + sb * 64;
                // 16 dims per instruction, Q from TMEM
                mma_ts<false>(sd, tmem + kQCol, klo, kHi, kIdS);
#pragma unroll
                for (int kk = 1; kk < kD / 16; ++kk)
                    mma_ts<true>(sd, tmem + kQCol + kk * 8, klo + (((kk >> 2) * 1024 + (kk & 3) * 32) >> 4), kHi, kIdS);
                umma_commit(&s_full[sb]);
                umma_commit(&k_empty[s]);                       // K(i) read
                if (i >= 2) issue_pv(i - 2);
            }
            // drain: no MMA of this CTA is in flight when TMEM is released, after a wait that
            // gave up as well
            umma_commit(mma_drain);
            mbar_wait(mma_drain, 0);
        }
    } else if (warp >= 4) {
        // ---------------- softmax warps 4..11: TMEM lane quarter warp % 4 (row r = query, head),
        // column half (warps 4..7 the tile's first 32 tokens, 8..11 the last 32).  The two warps
        // of a row agree on its running max through xch (one mbarrier per quarter and buffer);
        // each keeps the sum of its own columns.
        const int quarter = warp & 3, half = (warp - 4) >> 2;
        const int r = quarter * 32 + lane;
        const int qq = r >> 4, h = r & 15;
        const int q = q0 + qq;
        const bool qv = q < p.nq;
        const int pos = qv ? sh_pos[qq] : -1;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        const float sc = p.scale_log2;
        const float2 sc2 = make_float2(sc, sc), one2 = make_float2(1.0f, 1.0f);
        {
            // Q: this warp's half of row r (96 dims, two per column) into TMEM, A of S = Q K^T
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                float qc[16];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint4 v = qreg[4 * j + k];
                    qc[4 * k + 0] = __uint_as_float(v.x);
                    qc[4 * k + 1] = __uint_as_float(v.y);
                    qc[4 * k + 2] = __uint_as_float(v.z);
                    qc[4 * k + 3] = __uint_as_float(v.w);
                }
                tmem_st16(trow + kQCol + half * 48 + 16 * j, qc);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        float mrow = -INFINITY, lrow = 0.0f;
        uint32_t whole_bits = 0u;
        auto exchange = [&](int i, float mine) -> float {    // the partner warp's value for row r
            const int b = i & 1;
            xch[(b * 2 + half) * 128 + r] = mine;
            __syncwarp();
            if (lane == 0) mbar_arrive(&x_full[quarter * 2 + b]);
            ok = __all_sync(0xffffffffu, mbar_wait(&x_full[quarter * 2 + b], (i >> 1) & 1));
            return ok ? xch[(b * 2 + (half ^ 1)) * 128 + r] : 0.0f;
        };
        for (int i = 0; i < n_tiles && ok; ++i) {
            const int sb = i & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (i >> 1) & 1));
            if (!ok) break;
            tc_fence_after();
            float sv[32];
            tmem_ld32(trow + sb * 64 + half * 32, sv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[sb]);       // the MMA may write S(i + 2) here
            // mask: a union region this row's query selected, tokens at or before its position
            // (token e of a region is kept when e <= lim); most tiles need none
            if ((i & 31) == 0) whole_bits = sh_whole[i >> 5];
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if ((whole_bits >> (i & 31)) & 1u) {               // block-uniform
#pragma unroll
                for (int j = 0; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], sv[j]);
            } else {
                int lim[4];
#pragma unroll
                for (int jr = 0; jr < 4; ++jr) {
                    const int u = i * kTileRegions + half * 4 + jr;
                    const bool member = u < U && ((umask[u >> 2] >> ((u & 3) * 8 + qq)) & 1u);
                    lim[jr] = member ? pos - uni[u] * kRegion : -1;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    sv[j] = (j & 7) <= lim[j >> 3] ? sv[j] : -INFINITY;
                    m4[j & 3] = fmaxf(m4[j & 3], sv[j]);
                }
            }
            const float mine = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sc;   // sc > 0
            const float mx = fmaxf(mine, exchange(i, mine));
            if (!ok) break;
            // lazy rescaling: the reference max moves only when the tile's max exceeds it by more
            // than the slack (P stays below 2^slack): the same softmax, rarely rescaled.  Both
            // warps of a row take the same decision from the same values.
            const bool grow = mx > mrow + attn::kSlack;
            float alpha = 1.0f;
            if (grow) {
                alpha = ex2(mrow - mx);
                mrow = mx;
            }
            const float nref = (mrow == -INFINITY) ? 0.0f : -mrow;
            const float2 nref2 = make_float2(nref, nref);
            float2 s2a = make_float2(0.0f, 0.0f), s2b = s2a;
            float pk[16];                                   // P(i): bf16 pairs (tokens 2c, 2c + 1)
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float2 t = ffma2(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nref2);
                const float2 e = make_float2(ex2(t.x), ex2(t.y));
                if (c & 1) s2b = ffma2(e, one2, s2b);
                else s2a = ffma2(e, one2, s2a);
                pk[c] = __uint_as_float(pack_bf16x2(e.x, e.y));
            }
            lrow = lrow * alpha + ((s2a.x + s2a.y) + (s2b.x + s2b.y));
            if (__any_sync(0xffffffffu, grow && i > 0)) {
                // O holds the tiles before i once their P V has completed: scale this warp's
                // 96 columns of it in TMEM
                ok = __all_sync(0xffffffffu, mbar_wait_sleep(&o_done[(i - 1) & 1], ((i - 1) >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 3; ++c) {
                    float o[32];
                    const uint32_t ta = trow + kOCol + half * 96 + 32 * c;
                    tmem_ld32(ta, o);
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] *= alpha;
                    tmem_st32(ta, o);
                }
            }
            // P(i) into its TMEM buffer once P V has read the tile two back from it
            ok = __all_sync(0xffffffffu, mbar_wait_sleep(&p_free[sb], ((i >> 1) & 1) ^ 1));
            if (!ok) break;
            tc_fence_after();
            tmem_st16(trow + kPCol + sb * 32 + half * 16, pk);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sb]);
        }
        // ---- output: O / l (bf16, this warp's 96 columns) and the LSE, once the last P V has
        // completed; l is the sum of both halves'
        if (ok) lrow += exchange(n_tiles, lrow);
        if (ok && n_tiles > 0)
            ok = __all_sync(0xffffffffu, mbar_wait_sleep(&o_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1));
        if (ok) {
            tc_fence_after();
            const float inv = lrow > 0.0f ? 1.0f / lrow : 0.0f;
            __nv_bfloat16 *dst = p.out + ((int64_t)q * kHQ + g * kHeadsPerGroup + h) * kD + half * 96;
#pragma unroll 1
            for (int c = 0; c < 3; ++c) {
                float o[32];
                tmem_ld32(trow + kOCol + half * 96 + 32 * c, o);
                if (qv) {
#pragma unroll
                    for (int k8 = 0; k8 < 4; ++k8) {
                        uint4 w;
                        w.x = pack_bf16x2(o[8 * k8 + 0] * inv, o[8 * k8 + 1] * inv);
                        w.y = pack_bf16x2(o[8 * k8 + 2] * inv, o[8 * k8 + 3] * inv);
                        w.z = pack_bf16x2(o[8 * k8 + 4] * inv, o[8 * k8 + 5] * inv);
                        w.w = pack_bf16x2(o[8 * k8 + 6] * inv, o[8 * k8 + 7] * inv);
                        reinterpret_cast<uint4 *>(dst + 32 * c)[k8] = w;
                    }
                }
            }
            if (qv && p.lse && half == 0)
                p.lse[(int64_t)q * kHQ + g * kHeadsPerGroup + h] =
                    lrow > 0.0f ? (mrow + log2f(lrow)) * 0.69314718055994531f : -INFINITY;
        }
    }
    // every role done (or gave up): release TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_free(tmem, kTmemCols);
}

}  // namespace attntc
}  // namespace dsa
