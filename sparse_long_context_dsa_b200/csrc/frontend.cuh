// Indexer front end ([P2] Step-5-Preview 如何实现1M长上下文 §索引器打分: the indexer projects
// the hidden state to index_q / index_k / index_z, then normalises and applies RoPE to part of
// the dimensions), as a tcgen05 bf16 GEMM with the norm, the rotation and the gates fused into
// its epilogue.  Reading of the unstated constants: per-head RMSNorm (eps 1e-6, a learned
// weight per side), rotate-half RoPE on the first 64 of 256 dims (pairs i, i + 32, angle
// pos * 10000^(-i/32)), z = sigmoid.
//
//   out[t][j] = sum_i W[j][i] h[t][i]      (bf16 x bf16 -> fp32, j < 5,136: 16 x 256 q rows,
//                                           4 x 256 k rows, 16 gate rows)
// Layout of the work: a unit is 128 tokens (M, the TMEM lanes) x one 256-row block of W (N):
// a q head, a k group, or the gate rows (the block's other 240 rows lie past W and read as
// zero).  Persistent CTAs, one per SM: a TMA warp streams 128 x 64 hidden and 256 x 64 weight
// tiles (128-byte swizzle) through a 4-stage ring, one thread issues 4 tcgen05.mma.kind::f16
// (M = 128, N = 256, K = 16) per stage into one of two 256-column TMEM accumulators, and four
// epilogue warps (one token row per thread) take the row's 256 values: the sum of squares, then
// x * rsqrt(mean + eps) * gamma, the rotation of the first 64 (angles reduced in double), bf16
// stores of 512 contiguous bytes; gate units take sigmoid of the first 16 columns.
#pragma once

#include "common.cuh"

namespace dsa {
namespace fe {

constexpr int kBM = 128;                  // tokens per unit
constexpr int kBN = 256;                  // weight rows per unit
constexpr int kBK = 64;                   // hidden elements per stage (128 bytes of bf16)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;    // 16 KiB
constexpr int kBBytes = kBN * kBK * 2;    // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kHeadUnits = kHI + kG;      // 20 blocks of 256 rows: q heads, then k groups
constexpr int kUnitsPerTile = kHeadUnits + 1;   // + the gate block
constexpr int kRows = kHeadUnits * kDI + kHI;   // 5,136 weight rows
constexpr int kRot = 64;                  // rotated dims of a 256-d head
constexpr int kThreads = 192;             // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kTmemCols = 512;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 2 * kDI * 4 + 32 * 8 + 256;
static_assert(kSmemBytes <= 232448, "one CTA per SM");

// tcgen05 instruction descriptor, kind::f16: BF16 x BF16 -> F32, both operands K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kIdesc = umma_idesc_bf16(kBM, kBN);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

struct Params {
    const __nv_bfloat16 *gamma_q;   // [256]
    const __nv_bfloat16 *gamma_k;   // [256]
    const int32_t *pos;             // [T]
    __nv_bfloat16 *index_q;         // [T][16][256]
    __nv_bfloat16 *index_k;         // [T][4][256]
    float *z;                       // [T][16]
    int n_tok;
    int n_k;                        // k-steps: ceil(hid / 64)
    int n_units;                    // ceil(T / 128) * 21
};

__global__ void __launch_bounds__(kThreads, 1)
    frontend_kernel(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w,
                    const Params p)
{
    pdl_trigger();   // the next kernel may launch; it waits for this one itself
    pdl_wait();      // the previous kernel's results are visible from here on
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *gam = reinterpret_cast<float *>(smem + kStages * kStageBytes);    // [2][256]: q, k
    double *inv_freq = reinterpret_cast<double *>(gam + 2 * kDI);            // [32]
    uint64_t *bars = reinterpret_cast<uint64_t *>(inv_freq + 32);
    uint64_t *full = bars, *empty = bars + kStages;                           // [kStages]
    uint64_t *acc_full = bars + 2 * kStages, *acc_empty = acc_full + 2;      // [2]
    uint64_t *mma_drain = acc_empty + 2;                                     // the MMA issuer's last commit
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(mma_drain, 1);
        fence_mbar_init();
    }
    for (int i = threadIdx.x; i < kDI; i += kThreads) {
        gam[i] = __bfloat162float(p.gamma_q[i]);
        gam[kDI + i] = __bfloat162float(p.gamma_k[i]);
    }
    if (threadIdx.x < kRot / 2) inv_freq[threadIdx.x] = pow(10000.0, -(double)threadIdx.x / (kRot / 2));
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        // ---------------- TMA producer (one lane)
        if (lane == 0) {
            prefetch_tensormap(&map_h);
            prefetch_tensormap(&map_w);
            int it = 0, issued = 0;                           // issued: stages whose loads went out
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
                const int m = u / kUnitsPerTile, n = u % kUnitsPerTile;
                for (int kk = 0; kk < p.n_k; ++kk, ++it) {
                    const int s = it % kStages;
                    ok = mbar_wait_sleep(&empty[s], ((it / kStages) & 1) ^ 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    uint8_t *dst = smem + s * kStageBytes;
                    tma_load_2d(dst, &map_h, kk * kBK, m * kBM, &full[s]);
                    tma_load_2d(dst + kABytes, &map_w, kk * kBK, n * kBN, &full[s]);
                    issued = it + 1;
                }
            }
            // drain: none of these loads is in flight when the CTA exits, after a wait that gave
            // up as well (the last phase issued into every stage; complete already otherwise)
            for (int s = 0; s < kStages && s < issued; ++s) {
                const int last = issued - 1 - (issued - 1 - s) % kStages;
                mbar_wait(&full[s], (last / kStages) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one lane)
        if (lane == 0) {
            int it = 0, ui = 0;
            for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++ui) {
                const int buf = ui & 1;
                ok = mbar_wait_sleep(&acc_empty[buf], ((ui >> 1) & 1) ^ 1);
                if (!ok) break;
                tc_fence_after();
                for (int kk = 0; kk < p.n_k; ++kk, ++it) {
                    const int s = it % kStages;
                    ok = mbar_wait_sleep(&full[s], (it / kStages) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t da = umma_desc_sw128(smem_u32(smem + s * kStageBytes));
                    const uint64_t db = umma_desc_sw128(smem_u32(smem + s * kStageBytes + kABytes));
#pragma unroll
                    for (int k16 = 0; k16 < kBK / 16; ++k16)      // 32 bytes of K per instruction
                        umma_bf16(tmem + buf * kBN, da + (uint64_t)(k16 * 2), db + (uint64_t)(k16 * 2), kIdesc,
                                  kk > 0 || k16 > 0);
                    umma_commit(&empty[s]);                       // the stage may be overwritten
                }
                if (!ok) break;
                umma_commit(&acc_full[buf]);                      // the unit's accumulator is ready
            }
            // drain: no MMA of this CTA is in flight when TMEM is released
            umma_commit(mma_drain);
            mbar_wait(mma_drain, 0);
        }
    } else {
        // ---------------- epilogue: warps 2..5; TMEM lane quarter sp = warp % 4 (the hardware's
        // lane-access rule): token rows 32 sp .. 32 sp + 31 of the unit, one per thread
        const int sp = warp & 3;
        auto store32 = [](__nv_bfloat16 *dst, const float (&v)[32]) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 w;
                w.x = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
                w.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
                w.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
                w.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
                reinterpret_cast<uint4 *>(dst)[c] = w;
            }
        };
        int ui = 0;
        for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++ui) {
            const int m = u / kUnitsPerTile, n = u % kUnitsPerTile;
            const int buf = ui & 1;
            const int t = m * kBM + 32 * sp + lane;
            const bool tv = t < p.n_tok;
            // this token's rotation angles, reduced to [-pi, pi] in double before the float sincos
            float cs[kRot / 2], sn[kRot / 2];
            if (n < kHeadUnits) {
                const double pos = tv ? (double)p.pos[t] : 0.0;
                constexpr double kTwoPi = 6.283185307179586476925286766559;
#pragma unroll
                for (int i = 0; i < kRot / 2; ++i) {
                    double th = pos * inv_freq[i];
                    th -= kTwoPi * rint(th / kTwoPi);
                    sincosf((float)th, &sn[i], &cs[i]);
                }
            }
            ok = mbar_wait_sleep(&acc_full[buf], (ui >> 1) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t ta = tmem + ((uint32_t)(32 * sp) << 16) + buf * kBN;
            auto release = [&]() {                                // the MMA may refill this accumulator
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
            };
            if (n == kHeadUnits) {
                // gate rows: z = sigmoid of columns 0..15
                float v[32];
                tmem_ld32(ta, v);
                release();
                if (tv) {
                    float4 *zd = reinterpret_cast<float4 *>(p.z + (int64_t)t * kHI);
#pragma unroll
                    for (int c = 0; c < kHI / 4; ++c)
                        zd[c] = make_float4(1.0f / (1.0f + expf(-v[4 * c])), 1.0f / (1.0f + expf(-v[4 * c + 1])),
                                            1.0f / (1.0f + expf(-v[4 * c + 2])), 1.0f / (1.0f + expf(-v[4 * c + 3])));
                }
                continue;
            }
            // pass 1: the head vector's sum of squares
            float ss = 0.0f;
#pragma unroll 1
            for (int c = 0; c < kDI / 32; ++c) {
                float v[32];
                tmem_ld32(ta + 32 * c, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
            }
            const float inv = 1.0f / sqrtf(ss * (1.0f / kDI) + 1e-6f);
            const float *g = gam + (n < kHI ? 0 : kDI);
            __nv_bfloat16 *dst = n < kHI ? p.index_q + ((int64_t)t * kHI + n) * kDI
                                         : p.index_k + ((int64_t)t * kG + (n - kHI)) * kDI;
            // pass 2: normalise, rotate dims 0..63 in pairs (i, i + 32), store
            {
                float a[32], b[32];
                tmem_ld32x2(ta, ta + 32, a, b);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float ya = a[i] * inv * g[i], yb = b[i] * inv * g[32 + i];
                    a[i] = ya * cs[i] - yb * sn[i];
                    b[i] = yb * cs[i] + ya * sn[i];
                }
                if (tv) {
                    store32(dst, a);
                    store32(dst + 32, b);
                }
            }
#pragma unroll 1
            for (int c = 2; c < kDI / 32; ++c) {
                float v[32];
                tmem_ld32(ta + 32 * c, v);
                if (c == kDI / 32 - 1) release();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = v[j] * inv * g[32 * c + j];
                if (tv) store32(dst + 32 * c, v);
            }
        }
    }
    // every role done (or gave up): release TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_free(tmem, kTmemCols);
}

}  // namespace fe
}  // namespace dsa
