// libdsa: the C-ABI entry points declared in include/dsa.h.  Host code here only checks
// arguments, sizes grids, encodes TMA tensor maps and launches the kernels of
// compress.cuh, indexer.cuh, topk.cuh and attention.cuh (one translation unit, so the
// per-device error word is a single symbol).
#include <algorithm>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <utility>
#include <string>

#include "../../include/dsa.h"
#include "attention.cuh"
#include "attention_cluster.cuh"
#include "attention_tc.cuh"
#include "common.cuh"
#include "compress.cuh"
#include "copy.cuh"
#include "frontend.cuh"
#include "gemm_indexer.cuh"
#include "indexer.cuh"
#include "selftest.cuh"
#include "topk.cuh"
#include "topk_cluster.cuh"
#include "topk_rows.cuh"

namespace {

thread_local std::string g_last_error;

dsa_status_t fail(dsa_status_t st, const std::string &msg)
{
    g_last_error = msg;
    return st;
}

dsa_status_t cuda_fail(cudaError_t e, const char *what)
{
    return fail(DSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define DSA_REQUIRE(cond, msg)                                  \
    do {                                                        \
        if (!(cond)) return fail(DSA_ERR_INVALID_ARG, (msg));   \
    } while (0)

#define DSA_CUDA(call, what)                                    \
    do {                                                        \
        cudaError_t e_ = (call);                                \
        if (e_ != cudaSuccess) return cuda_fail(e_, (what));    \
    } while (0)

// Every pointer argument must be memory the current device can dereference: device memory
// of this device, managed memory, or pinned / registered host memory.  Pageable host memory
// is refused (a kernel touching it would fault) unless the device reads pageable memory
// coherently (cudaDevAttrPageableMemoryAccess).  Checked on the host before any launch.
struct Ptr {
    const void *p;
    const char *name;
};

dsa_status_t check_reachable(std::initializer_list<Ptr> ptrs)
{
    int dev = 0;
    DSA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    int pageable = -1;
    for (const Ptr &x : ptrs) {
        if (!x.p) continue;                       // NULL is each call's own business
        cudaPointerAttributes a;
        const cudaError_t e = cudaPointerGetAttributes(&a, x.p);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, (std::string("cudaPointerGetAttributes(") + x.name + ")").c_str());
        }
        if (a.type == cudaMemoryTypeDevice && a.device != dev)
            return fail(DSA_ERR_INVALID_ARG, std::string(x.name) + " is device memory of GPU " +
                                                 std::to_string(a.device) + ", the call runs on GPU " +
                                                 std::to_string(dev));
        if (a.type != cudaMemoryTypeUnregistered) continue;
        if (pageable < 0) {
            DSA_CUDA(cudaDeviceGetAttribute(&pageable, cudaDevAttrPageableMemoryAccess, dev),
                     "cudaDeviceGetAttribute(PageableMemoryAccess)");
        }
        if (!pageable)
            return fail(DSA_ERR_INVALID_ARG, std::string(x.name) +
                                                 " is pageable host memory, which this GPU cannot read: pass device "
                                                 "memory or pinned host memory (cudaHostAlloc / cudaHostRegister)");
    }
    return DSA_OK;
}

#define DSA_REACHABLE(...)                                      \
    do {                                                        \
        dsa_status_t r_ = check_reachable({__VA_ARGS__});       \
        if (r_ != DSA_OK) return r_;                            \
    } while (0)

// A KV group range: 1, 2 or 4 consecutive groups starting at g0.
dsa_status_t group_range_args(int g0, int ng)
{
    DSA_REQUIRE(ng == 1 || ng == 2 || ng == 4, "ng must be 1, 2 or 4");
    DSA_REQUIRE(g0 >= 0 && g0 + ng <= dsa::kG, "groups g0 .. g0 + ng - 1 must lie in 0 .. 3");
    return DSA_OK;
}

constexpr int kGemmMinQueries = 64;   // FP8 prefill chunks at least this long use the GEMM
constexpr int kSharedMinQueries = 32; // prefill attention calls at least this long share selections

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device facts, checked on every call (cheap attribute queries).
dsa_status_t device_info(int &sm_count)
{
    int dev = 0;
    DSA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    int major = 0;
    DSA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "cudaDeviceGetAttribute");
    if (major != 10) return fail(DSA_ERR_UNSUPPORTED, "libdsa is built for sm_100a (B200); device is sm_" +
                                                          std::to_string(major) + "x");
    DSA_CUDA(cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev), "cudaDeviceGetAttribute");
    return DSA_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

dsa_status_t encode(CUtensorMap *map, CUtensorMapDataType dt, int rank, const void *base, const cuuint64_t *dims,
                    const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapL2promotion l2,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string((int)r) + ")");
    return DSA_OK;
}

dsa_status_t launched(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return DSA_OK;
}

// Every kernel is launched with programmatic stream serialization (it may start while the
// previous kernel of the stream finishes; each kernel waits for it before touching global
// memory), optionally as clusters of cluster_x CTAs.
template <typename... KArgs, typename... Args>
dsa_status_t launch_k(const char *what, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      dsa_stream_t stream, unsigned cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return launched(what);
}

// K/V cache viewed as [rows = n_pages*ng*64][3][64] bf16 (ng KV groups per page, 4 unless
// the call holds a group range): one region = box {64, 3, 8}.
dsa_status_t kv_map(CUtensorMap *m, const void *cache, int64_t n_pages, int ng = dsa::kG)
{
    const cuuint64_t dims[3] = {64, 3, (cuuint64_t)n_pages * ng * dsa::kPage};
    const cuuint64_t strides[2] = {128, (cuuint64_t)dsa::kD * 2};
    const cuuint32_t box[3] = {64, 3, (cuuint32_t)dsa::kRegion};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, cache, dims, strides, box, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// 3-D view (64 dims, n_pages * 4 * 64 rows, 3 blocks) of a K/V cache with the row stride 384 B
// and the block stride 128 B (a stride order the tensor map accepts): one box {64, 8, 3} is a
// whole region, landing as [3 blocks][8 rows][128 B] with the 128-byte swizzle, the tcgen05
// shared-selection attention's operand tiles.
dsa_status_t kv_map_blocks(CUtensorMap *m, const void *cache, int64_t n_pages)
{
    const cuuint64_t dims[3] = {64, (cuuint64_t)n_pages * dsa::kG * dsa::kPage, 3};
    const cuuint64_t strides[2] = {(cuuint64_t)dsa::kD * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)dsa::kRegion, 3};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, cache, dims, strides, box, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

struct TopkLayout {
    size_t hist, ctr, sure, cand, total;
};

TopkLayout topk_layout(int nq, int64_t ld, int k, int ng = dsa::kG)
{
    const size_t rows = (size_t)nq * ng;
    TopkLayout L;
    L.hist = 0;
    L.ctr = round_up(rows * dsa::topk::kBins * 4, 256);
    L.sure = L.ctr + round_up(rows * 16, 256);
    L.cand = L.sure + round_up(rows * (size_t)k * 4, 256);
    L.total = L.cand + round_up(rows * (size_t)ld * 8, 256);
    return L;
}

// attention split policy: few rows -> split each selection into chunks of 16 regions
struct AttnPlan {
    int rps, n_splits;
    size_t ws;
};

// The split is decided on all four groups' rows, also for a call that holds fewer groups,
// so a group shard runs exactly the splits of the 4-group call (and its rows come out bit
// for bit the same); the workspace counts the call's own rows (nq * ng).
AttnPlan attn_plan(int nq, int k, int sm_count, int ng = dsa::kG)
{
    AttnPlan a;
    const int rows = nq * dsa::kG;
    if (rows >= 2 * sm_count) {
        a.rps = k;
        a.n_splits = 1;
        a.ws = 0;
    } else {
        // about 2 CTAs per SM over all rows, at least 2 regions (one pair) per CTA and at
        // most kD splits (the combine kernel holds one split weight per thread)
        const int want = std::max(1, (2 * sm_count + rows - 1) / rows);
        int rps = (k + want - 1) / want;
        rps = std::max(2, (rps + 1) & ~1);
        while ((k + rps - 1) / rps > dsa::kD) rps += 2;
        a.rps = rps;
        a.n_splits = (k + a.rps - 1) / a.rps;
        const size_t n = (size_t)nq * ng * a.n_splits * 16;
        a.ws = round_up(n * dsa::kD * 4, 256) + round_up(n * 2 * 4, 256);
    }
    return a;
}

// The clustered attention kernel (splits merged in the kernel) serves rows that get one
// cluster each with every cluster resident at once: rows <= the number of such clusters the
// device holds together (queried once per process and shape; 0 when the kernel cannot take
// its cluster size).  Selections (k <= 512): 16-CTA clusters, one CTA per SM; windows of up
// to 80 regions: 8-CTA clusters, two CTAs per SM.
template <class Sh, int kMinBlocks, bool kWin>
struct ClusterAttn {
    static constexpr auto fn =
        dsa::attnc::sparse_attn_cluster_kernel<Sh::kSplits, Sh::kRegionsPerCta, kMinBlocks, kWin>;
    static int capacity()
    {
        static std::once_flag once;
        static int cap = 0;
        std::call_once(once, [] {
            if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::kSmemBytes) !=
                    cudaSuccess ||
                cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
                cudaGetLastError();
                return;
            }
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(Sh::kSplits, 1, 1);
            cfg.blockDim = dim3(dsa::attnc::kThreads, 1, 1);
            cfg.dynamicSmemBytes = Sh::kSmemBytes;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = Sh::kSplits;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
                cudaGetLastError();
                return;
            }
            cap = n;
        });
        return cap;
    }
    static dsa_status_t launch(const CUtensorMap &mk, const CUtensorMap &mv, const dsa::attn::Params &p, int nq,
                               dsa_stream_t stream)
    {
        return launch_k("sparse_attn_cluster_kernel", fn,
                        dim3(Sh::kSplits, (unsigned)(nq * ((int)1 << p.gshift))), dim3(dsa::attnc::kThreads),
                        Sh::kSmemBytes, stream, (unsigned)Sh::kSplits, mk, mv, p);
    }
};
using DecodeAttn = ClusterAttn<dsa::attnc::Decode, 1, false>;
using WindowAttn = ClusterAttn<dsa::attnc::Window, 2, true>;
int cluster_attn_capacity() { return DecodeAttn::capacity(); }

// Regions a window of `window` tokens can touch: its first token may sit anywhere in a region.
int window_regions(int window) { return window / dsa::kRegion + 2; }

// window == 0: attention over the selection (sel_idx, sel_count, k); window > 0: over each
// query's last `window` tokens (k = window_regions(window), no selection).
dsa_status_t attn_common(const void *q, const void *k_cache, const void *v_cache, int64_t n_pages,
                         const int32_t *block_table, int max_pages, const int32_t *q_req, int n_req,
                         const int32_t *q_pos, int nq, const int32_t *sel_idx, const int32_t *sel_count, int k,
                         void *out, float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream, int window = 0,
                         int g0 = 0, int ng = dsa::kG, const void *new_k = nullptr, const void *new_v = nullptr)
{
    DSA_REQUIRE(nq >= 0, "nq must be >= 0");
    DSA_REQUIRE(window > 0 || (k >= 1 && k <= DSA_MAX_TOPK), "k out of [1, DSA_MAX_TOPK]");
    DSA_REQUIRE(n_pages >= 1 && n_pages <= (INT32_MAX / (dsa::kG * dsa::kPage)), "n_pages out of range");
    DSA_REQUIRE(max_pages >= 1, "max_pages must be >= 1");
    DSA_REQUIRE(n_req >= 1, "n_req must be >= 1");
    if (nq == 0) return DSA_OK;
    DSA_REQUIRE(q && k_cache && v_cache && block_table && q_pos && out, "NULL pointer");
    DSA_REQUIRE(window > 0 || (sel_idx && sel_count), "NULL pointer");
    DSA_REQUIRE(aligned(q, 16) && aligned(k_cache, 16) && aligned(v_cache, 16) && aligned(out, 4),
                "q, k_cache, v_cache must be 16-byte aligned, out 4-byte aligned");
    DSA_REACHABLE({q, "q"}, {k_cache, "k_cache"}, {v_cache, "v_cache"}, {block_table, "block_table"},
                  {q_req, "q_req"}, {q_pos, "q_pos"}, {sel_idx, "sel_idx"}, {sel_count, "sel_count"}, {out, "out"},
                  {lse, "lse"}, {ws, "ws"});
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    // (decided on all four groups' rows, as the split above: a group shard runs the kernels
    // of the 4-group call)
    const bool clustered =
        window == 0 && k <= dsa::attnc::kMaxK && (int64_t)nq * dsa::kG <= cluster_attn_capacity();
    // window layers: one 8-CTA cluster per row while every row's cluster is resident at once
    const bool clustered_window = window > 0 && ng == dsa::kG && k <= dsa::attnc::Window::kMaxK &&
                                  (int64_t)nq * dsa::kG <= WindowAttn::capacity();
    // prefill chunks: 8 neighbouring queries per CTA share one stream of their selections' union
    const bool shared = window == 0 && !clustered && ng == dsa::kG && q_req != nullptr && nq >= kSharedMinQueries &&
                        k <= dsa::attntc::kMaxK &&
                        (int64_t)max_pages * dsa::kPage / dsa::kRegion <= (int64_t)dsa::attntc::kMaxWords * 32;
    const AttnPlan plan = attn_plan(nq, k, sms, ng);
    const size_t need_ws = plan.ws + (shared ? round_up((size_t)nq * dsa::kG, 256) : 0);
    if (need_ws > 0 && !clustered && !clustered_window) {
        if (!ws || ws_bytes < need_ws || !aligned(ws, 256))
            return fail(DSA_ERR_WORKSPACE, "attention workspace too small or not 256-byte aligned (need " +
                                               std::to_string(need_ws) + " bytes)");
    }
    CUtensorMap mk, mv;
    if ((st = kv_map(&mk, k_cache, n_pages, ng)) != DSA_OK) return st;
    if ((st = kv_map(&mv, v_cache, n_pages, ng)) != DSA_OK) return st;

    dsa::attn::Params p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.block_table = block_table;
    p.q_req = q_req;
    p.q_pos = q_pos;
    p.sel_idx = sel_idx;
    p.sel_count = sel_count;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.lse = lse;
    const size_t n = (size_t)nq * ng * plan.n_splits * 16;
    p.part_o = plan.ws ? static_cast<float *>(ws) : nullptr;
    p.part_ml = plan.ws ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + round_up(n * dsa::kD * 4, 256))
                        : nullptr;
    p.n_pages = n_pages;
    p.max_pages = max_pages;
    p.n_req = n_req;
    p.nq = nq;
    p.k = k;
    p.rps = plan.rps;
    p.n_splits = plan.n_splits;
    p.window = window;
    p.scale_log2 = dsa::attn::kLog2e / sqrtf((float)dsa::kD);
    p.gshift = ng == 4 ? 2 : ng == 2 ? 1 : 0;
    p.g0 = g0;
    if (new_k) {                       // the append folded in: only the clustered window kernel takes it
        if (!clustered_window) return fail(DSA_ERR_UNSUPPORTED, "window append without the clustered kernel");
        p.new_k = static_cast<const __nv_bfloat16 *>(new_k);
        p.new_v = static_cast<const __nv_bfloat16 *>(new_v);
        p.k_cache = static_cast<__nv_bfloat16 *>(const_cast<void *>(k_cache));
        p.v_cache = static_cast<__nv_bfloat16 *>(const_cast<void *>(v_cache));
    }

    if (clustered) return DecodeAttn::launch(mk, mv, p, nq, stream);
    if (clustered_window) return WindowAttn::launch(mk, mv, p, nq, stream);
    if (shared) {
        // 8 neighbouring queries of one request with a small union: tcgen05 tiles of 128 rows
        p.row_shared = static_cast<uint8_t *>(ws) + plan.ws;
        static std::once_flag sh_once;
        static cudaError_t sh_err = cudaSuccess;
        std::call_once(sh_once, [] {
            sh_err = cudaFuncSetAttribute(dsa::attntc::sparse_attn_tc_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsa::attntc::kSmemBytes);
        });
        DSA_CUDA(sh_err, "cudaFuncSetAttribute(sparse_attn_tc_kernel)");
        CUtensorMap rk, rv;
        if ((st = kv_map_blocks(&rk, k_cache, n_pages)) != DSA_OK) return st;
        if ((st = kv_map_blocks(&rv, v_cache, n_pages)) != DSA_OK) return st;
        const unsigned blocks = (unsigned)((nq + dsa::attntc::kQueries - 1) / dsa::attntc::kQueries) * dsa::kG;
        if ((st = launch_k("sparse_attn_tc_kernel", dsa::attntc::sparse_attn_tc_kernel, dim3(blocks),
                           dim3(dsa::attntc::kThreads), dsa::attntc::kSmemBytes, stream, 0, rk, rv, p,
                           (int)(n_pages * dsa::kG * dsa::kPage))) != DSA_OK)
            return st;
        // then the rows it left to the per-row kernel (the others return at once)
    }
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::attn::sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)dsa::attn::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(sparse_attn_kernel)");
    dim3 grid((unsigned)(plan.n_splits * nq * ng));
    if ((st = launch_k("sparse_attn_kernel", dsa::attn::sparse_attn_kernel, grid, dim3(dsa::attn::kThreads),
                       dsa::attn::kSmemBytes, stream, 0, mk, mv, p)) != DSA_OK)
        return st;
    if (plan.n_splits > 1) {
        if ((st = launch_k("combine_kernel", dsa::attn::combine_kernel, dim3(nq * ng * 16),
                           dim3(dsa::attn::kCombineThreads), 0, stream, 0, p)) != DSA_OK)
            return st;
    }
    return DSA_OK;
}

// Workspace of the prefill GEMM path: e4m3 query codes [nq][16][256], their scales
// [nq][16], the validated own region of every query and the largest one of every tile.
size_t gemm_ws_size(int nq)
{
    if (nq < kGemmMinQueries) return 0;
    const size_t tiles = (size_t)(nq + dsa::gemm::kQPerTile - 1) / dsa::gemm::kQPerTile;
    return round_up((size_t)nq * dsa::kHI * dsa::kDI, 256) + round_up((size_t)nq * dsa::kHI * 4, 256) +
           round_up((size_t)nq * 4, 256) + round_up(tiles * 4, 256);
}

dsa_status_t indexer_gemm_path(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos,
                               int nq, const uint8_t *summaries, const float *scales, int64_t n_slots,
                               const int64_t *sum_base, float *scores, int64_t ld, void *ws, int sms,
                               dsa_stream_t stream)
{
    uint8_t *w = static_cast<uint8_t *>(ws);
    uint8_t *codes = w;
    float *qscale = reinterpret_cast<float *>(w + round_up((size_t)nq * dsa::kHI * dsa::kDI, 256));
    int32_t *q_own = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(qscale) +
                                                 round_up((size_t)nq * dsa::kHI * 4, 256));
    int32_t *tile_own = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(q_own) + round_up((size_t)nq * 4, 256));
    const int n_mtiles = (nq + dsa::gemm::kQPerTile - 1) / dsa::gemm::kQPerTile;
    const int qblocks = (nq * dsa::kHI + 3) / 4;            // 4 warps per block: (q, h) pairs, then tiles
    const int grid_q = std::max(qblocks, (n_mtiles + 3) / 4);
    dsa_status_t st;
    if ((st = launch_k("gemm quantize_kernel", dsa::gemm::quantize_kernel, dim3(grid_q), dim3(128), 0, stream, 0,
                       static_cast<const __nv_bfloat16 *>(index_q), q_req, q_pos, sum_base, ld, n_slots, nq, codes,
                       qscale, q_own, tile_own, n_mtiles)) != DSA_OK)
        return st;

    CUtensorMap map_q, map_s;
    {
        // codes [nq][16 heads][256]: a box of 128 bytes of d x one group's 4 heads x 64 queries
        const cuuint64_t dims[3] = {(cuuint64_t)dsa::kDI, (cuuint64_t)dsa::kHI, (cuuint64_t)nq};
        const cuuint64_t strides[2] = {(cuuint64_t)dsa::kDI, (cuuint64_t)dsa::kDI * dsa::kHI};
        const cuuint32_t box[3] = {128, (cuuint32_t)dsa::gemm::kHeads, (cuuint32_t)dsa::gemm::kQPerTile};
        if ((st = encode(&map_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, dims, strides, box,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B)) != DSA_OK)
            return st;
    }
    {
        // summaries [4 * n_slots][256]: a box of 128 bytes x 128 regions
        const cuuint64_t dims[2] = {(cuuint64_t)dsa::kDI, (cuuint64_t)n_slots * dsa::kG};
        const cuuint64_t strides[1] = {(cuuint64_t)dsa::kDI};
        const cuuint32_t box[2] = {128, (cuuint32_t)dsa::gemm::kBM};
        if ((st = encode(&map_s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, summaries, dims, strides, box,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B)) != DSA_OK)
            return st;
    }
    CUtensorMap map_sc;
    {
        // scales [4 * n_slots] fp32 as one line: a block's 128 scales from a 16-byte aligned start
        const cuuint64_t dims[1] = {(cuuint64_t)n_slots * dsa::kG};
        const cuuint64_t strides[1] = {(cuuint64_t)n_slots * dsa::kG * 4};   // unused at rank 1
        const cuuint32_t box[1] = {(cuuint32_t)dsa::gemm::kScaleBox};
        if ((st = encode(&map_sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, scales, dims, strides, box,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_SWIZZLE_NONE)) != DSA_OK)
            return st;
    }
    dsa::gemm::Params p{};
    p.qscale = qscale;
    p.gate = gate;
    p.q_own = q_own;
    p.tile_own = tile_own;
    p.scales = scales;
    p.sum_base = sum_base;
    p.scores = scores;
    p.ld = ld;
    p.n_slots = n_slots;
    p.nq = nq;
    p.n_mtiles = n_mtiles;
    // persistent grid: at most one CTA per SM (512 TMEM columns, ~225 KiB of smem each)
    const int64_t blocks_bound = (int64_t)dsa::kG * n_mtiles * ((ld + dsa::gemm::kBM - 1) / dsa::gemm::kBM);
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::gemm::gemm_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)dsa::gemm::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(gemm_scores_kernel)");
    return launch_k("gemm_scores_kernel", dsa::gemm::gemm_scores_kernel,
                    dim3((unsigned)std::min<int64_t>(sms, std::max<int64_t>(1, blocks_bound))),
                    dim3(dsa::gemm::kThreads), dsa::gemm::kSmemBytes, stream, 0, map_q, map_s, map_sc, p);
}

// Workspace path of the top-k: histogram, threshold-bin gather and last-CTA selection
// (scales to many rows; scratch from the caller's workspace).
int gshift_of(int ng) { return ng == 4 ? 2 : ng == 2 ? 1 : 0; }

dsa_status_t topk_workspace_path(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq, int k,
                                 int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes, dsa_stream_t stream,
                                 int ng = dsa::kG)
{
    const TopkLayout L = topk_layout(nq, ld_scores, k, ng);
    if (!ws || ws_bytes < L.total || reinterpret_cast<uintptr_t>(ws) % 256 != 0)
        return fail(DSA_ERR_WORKSPACE, "top-k workspace too small or not 256-byte aligned (need " +
                                           std::to_string(L.total) + " bytes)");
    uint8_t *w = static_cast<uint8_t *>(ws);
    dsa::topk::Ws tw;
    tw.hist = reinterpret_cast<uint32_t *>(w + L.hist);
    tw.ctr = reinterpret_cast<uint32_t *>(w + L.ctr);
    tw.sure = reinterpret_cast<int32_t *>(w + L.sure);
    tw.cand = reinterpret_cast<uint2 *>(w + L.cand);
    tw.gshift = gshift_of(ng);
    DSA_CUDA(cudaMemsetAsync(w, 0, L.sure, stream), "cudaMemsetAsync(top-k histograms)");
    const int rows = nq * ng;
    const dim3 grid((unsigned)((ld_scores + dsa::topk::kChunk - 1) / dsa::topk::kChunk), (unsigned)rows);
    dsa_status_t st;
    if ((st = launch_k("topk hist_kernel", dsa::topk::hist_kernel, grid, dim3(dsa::topk::kThreads), 0, stream, 0,
                       scores, ld_scores, q_pos, k, tw)) != DSA_OK)
        return st;
    const size_t dyn = dsa::topk::kCandStage * 8 + round_up((size_t)((ld_scores + 1 + 31) / 32) * 4, 16);
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::topk::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(dsa::topk::kCandStage * 8 + (dsa::topk::kMaxRegions / 32 + 16) * 4));
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(topk select_kernel)");
    return launch_k("topk select_kernel", dsa::topk::select_kernel, grid, dim3(dsa::topk::kSelectThreads), dyn,
                    stream, 0, scores, ld_scores, q_pos, k, tw, sel_idx, sel_count);
}

// Cluster size for the cluster path: enough CTAs that each holds <= kPartMax keys in smem
// (power of two, at most 8); 0 when a row is too long for it.
int cluster_size_for(int64_t ld)
{
    int cl = 1;
    while ((int64_t)cl * dsa::topkc::kPartMax < ld) cl *= 2;
    return cl <= dsa::topkc::kMaxCluster ? cl : 0;
}

dsa_status_t topk_cluster_path(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq, int k,
                               int32_t *sel_idx, int32_t *sel_count, int cl, dsa_stream_t stream, int ng = dsa::kG)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::topkc::topk_cluster_kernel<true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsa::topkc::kSmemBytes);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(dsa::topkc::topk_cluster_kernel<false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsa::topkc::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(topk_cluster_kernel)");
    const dim3 grid((unsigned)cl, (unsigned)(nq * ng), 1);
    if (cl == 1)
        return launch_k("topk_cluster_kernel", dsa::topkc::topk_cluster_kernel<true>, grid, dim3(dsa::topkc::kThreads),
                        dsa::topkc::kSmemBytes, stream, 1u, scores, ld_scores, q_pos, k, sel_idx, sel_count,
                        static_cast<const float *>(nullptr), (int64_t)0, gshift_of(ng));
    return launch_k("topk_cluster_kernel", dsa::topkc::topk_cluster_kernel<false>, grid, dim3(dsa::topkc::kThreads),
                    dsa::topkc::kSmemBytes, stream, (unsigned)cl, scores, ld_scores, q_pos, k, sel_idx, sel_count,
                    static_cast<const float *>(nullptr), (int64_t)0, gshift_of(ng));
}

// Many rows of at most 65,536 scores: one CTA per row, no scratch.
dsa_status_t topk_rows_path(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq, int k,
                            int32_t *sel_idx, int32_t *sel_count, dsa_stream_t stream, int ng = dsa::kG)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::topkr::topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)dsa::topkr::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(topk_rows_kernel)");
    return launch_k("topk_rows_kernel", dsa::topkr::topk_rows_kernel, dim3((unsigned)(nq * ng)),
                    dim3(dsa::topkr::kThreads), dsa::topkr::kSmemBytes, stream, 0, scores, ld_scores, q_pos, k,
                    sel_idx, sel_count, gshift_of(ng));
}

// The top-k of nq queries x ng group rows: few long rows on clusters, many rows of up to
// 65,536 scores one CTA each, longer many-row calls through the workspace.
dsa_status_t topk_dispatch(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq, int k,
                           int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes, dsa_stream_t stream, int ng)
{
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    const int rows = nq * ng;
    const int cl = cluster_size_for(ld_scores);
    if (cl > 0 && (int64_t)rows * cl <= 2 * sms)
        return topk_cluster_path(scores, ld_scores, q_pos, nq, k, sel_idx, sel_count, cl, stream, ng);
    if (ld_scores <= dsa::topkr::kMaxLd)
        return topk_rows_path(scores, ld_scores, q_pos, nq, k, sel_idx, sel_count, stream, ng);
    return topk_workspace_path(scores, ld_scores, q_pos, nq, k, sel_idx, sel_count, ws, ws_bytes, stream, ng);
}

// Scratch of dsa_topk_regions_noalloc: one static array per GPU that loads the library.
static __device__ __align__(256) uint8_t g_topk_static_scratch[DSA_TOPK_STATIC_SCRATCH_BYTES];

// Device address of g_topk_static_scratch on `dev` (looked up once per device with that
// device current; in host code the symbol itself is only a host-side stand-in).
dsa_status_t static_scratch(int dev, void **ptr)
{
    constexpr int kMaxDevices = 64;
    static void *addr[kMaxDevices] = {};
    static std::mutex mu;
    if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device ordinal out of range");
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        DSA_CUDA(cudaGetSymbolAddress(&p, g_topk_static_scratch), "cudaGetSymbolAddress(top-k static scratch)");
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return DSA_OK;
}

}  // namespace

extern "C" {

int dsa_version(void) { return DSA_VERSION; }

const char *dsa_last_error(void) { return g_last_error.c_str(); }

size_t dsa_get_last_error(char *buf, size_t len)
{
    const size_t n = g_last_error.size();
    if (buf && len > 0) {
        const size_t m = std::min(n, len - 1);
        std::memcpy(buf, g_last_error.data(), m);
        buf[m] = '\0';
    }
    return n;
}

dsa_status_t dsa_check_device(dsa_stream_t stream)
{
    DSA_CUDA(cudaStreamSynchronize(stream), "cudaStreamSynchronize");
    unsigned word = 0;
    DSA_CUDA(cudaMemcpyFromSymbol(&word, dsa::g_error_word, sizeof(word)), "read error word");
    if (word == 0) return DSA_OK;
    const unsigned zero = 0;
    DSA_CUDA(cudaMemcpyToSymbol(dsa::g_error_word, &zero, sizeof(zero)), "clear error word");
    std::string msg = "device error word 0x" + [&] {
        char b[16];
        snprintf(b, sizeof b, "%x", word);
        return std::string(b);
    }() + ":";
    if (word & dsa::kErrCompressIndex) msg += " compress src_row/dst_slot out of range;";
    if (word & dsa::kErrIndexerQuery) msg += " indexer query out of range (q_req, own > ld, slots);";
    if (word & dsa::kErrTopkRow) msg += " top-k own region beyond ld_scores;";
    if (word & dsa::kErrAttnIndex) msg += " attention region/page index out of range;";
    if (word & dsa::kErrWaitTimeout) msg += " bounded wait timed out;";
    if (word & dsa::kErrTopkInternal) msg += " top-k internal inconsistency;";
    return fail(DSA_ERR_DEVICE, msg);
}

namespace {
dsa_status_t compress_impl(const void *index_k, int64_t row_stride, int64_t n_rows, const int64_t *src_row,
                           const int64_t *dst_slot, int n_regions, uint8_t *summaries, float *scales, int64_t n_slots,
                           dsa_stream_t stream, int g0, int ng)
{
    DSA_REQUIRE(n_regions >= 0, "n_regions must be >= 0");
    if (n_regions == 0) return DSA_OK;
    DSA_REQUIRE(index_k && src_row && dst_slot && summaries && scales, "NULL pointer");
    DSA_REQUIRE(row_stride >= (int64_t)(g0 + ng) * dsa::kDI && row_stride % 8 == 0,
                "row_stride must cover the groups' 256-element vectors and be a multiple of 8");
    DSA_REQUIRE(n_rows >= dsa::kRegion && n_slots >= 1, "n_rows >= 8 and n_slots >= 1 required");
    DSA_REQUIRE(aligned(index_k, 16) && aligned(summaries, 8) && aligned(scales, 4), "misaligned pointer");
    DSA_REACHABLE({index_k, "index_k"}, {src_row, "src_row"}, {dst_slot, "dst_slot"}, {summaries, "summaries"},
                  {scales, "scales"});
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    const int grid = (int)std::min<int64_t>(n_regions, (int64_t)sms * 16);
    // one warp per group: warp gl compresses group g0 + gl into pool row gl
    return launch_k("compress_regions_kernel", dsa::compress_regions_kernel, dim3(grid), dim3(32 * ng), 0, stream, 0,
                    static_cast<const __nv_bfloat16 *>(index_k) + (size_t)g0 * dsa::kDI, row_stride, n_rows, src_row,
                    dst_slot, n_regions, summaries, scales, n_slots);
}
}  // namespace

dsa_status_t dsa_compress_regions(const void *index_k, int64_t row_stride, int64_t n_rows, const int64_t *src_row,
                                  const int64_t *dst_slot, int n_regions, uint8_t *summaries, float *scales,
                                  int64_t n_slots, dsa_stream_t stream)
{
    return compress_impl(index_k, row_stride, n_rows, src_row, dst_slot, n_regions, summaries, scales, n_slots, stream,
                         0, dsa::kG);
}

dsa_status_t dsa_compress_regions_groups(const void *index_k, int64_t row_stride, int64_t n_rows,
                                         const int64_t *src_row, const int64_t *dst_slot, int n_regions, int g0,
                                         int ng, uint8_t *summaries, float *scales, int64_t n_slots,
                                         dsa_stream_t stream)
{
    dsa_status_t st = group_range_args(g0, ng);
    if (st != DSA_OK) return st;
    return compress_impl(index_k, row_stride, n_rows, src_row, dst_slot, n_regions, summaries, scales, n_slots, stream,
                         g0, ng);
}

// The streaming scan of dsa_indexer_scores; chunk_max (nullable) receives the largest score of
// every 32-region chunk, [nq][4][cm_stride].
dsa_status_t scan_path(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos, int nq,
                       const uint8_t *summaries, const float *scales, int64_t n_slots, const int64_t *sum_base,
                       int n_req, float *scores, int64_t ld_scores, uint32_t flags, int sms, dsa_stream_t stream,
                       float *chunk_max = nullptr, int64_t cm_stride = 0, int g0 = 0, int ng = dsa::kG)
{
    dsa_status_t st;
    CUtensorMap map;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)dsa::kDI, (cuuint64_t)n_slots * ng};
        const cuuint64_t strides[1] = {(cuuint64_t)dsa::kDI};
        const cuuint32_t box[2] = {128, (cuuint32_t)dsa::idx::kChunk};
        if ((st = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, summaries, dims, strides, box,
                         (CUtensorMapL2promotion)DSA_SCAN_L2_PROMOTION)) != DSA_OK)
            return st;
    }
    dsa::idx::Params p{};
    p.index_q = static_cast<const __nv_bfloat16 *>(index_q);
    p.gate = gate;
    p.q_req = q_req;
    p.q_pos = q_pos;
    p.scales = scales;
    p.sum_base = sum_base;
    p.scores = scores;
    p.chunk_max = chunk_max;
    p.cm_stride = cm_stride;
    p.n_slots = n_slots;
    p.ld = ld_scores;
    // stages per query: the (chunk, group) slabs of its row, four per stage
    const int64_t chunks = (ld_scores + dsa::idx::kChunk - 1) / dsa::idx::kChunk;
    p.units_per_query = (int)((chunks * ng + dsa::idx::kSlabs - 1) / dsa::idx::kSlabs);
    p.total_units = (int64_t)nq * p.units_per_query;
    p.groups = ng;
    p.gshift = gshift_of(ng);
    p.g0 = g0;
    p.nq = nq;
    p.n_req = n_req;
    p.flags = flags;

    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::idx::scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)dsa::idx::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(scan_kernel)");
    const int grid = (int)std::min<int64_t>(p.total_units, (int64_t)sms * dsa::idx::kCtasPerSm);
    return launch_k("scan_kernel", dsa::idx::scan_kernel, dim3(grid), dim3(dsa::idx::kThreads), dsa::idx::kSmemBytes,
                    stream, 0, map, p);
}

size_t dsa_indexer_workspace_size(int nq, int64_t ld_scores)
{
    (void)ld_scores;
    return gemm_ws_size(nq);
}

dsa_status_t dsa_indexer_scores(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos,
                                int nq, const uint8_t *summaries, const float *scales, int64_t n_slots,
                                const int64_t *sum_base, int n_req, float *scores, int64_t ld_scores, uint32_t flags,
                                void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    DSA_REQUIRE(nq >= 0, "nq must be >= 0");
    DSA_REQUIRE((flags & ~DSA_Q_FP8) == 0, "unknown flag");
    DSA_REQUIRE(ld_scores >= 1 && ld_scores <= (1ll << 26), "ld_scores out of [1, 2^26]");
    DSA_REQUIRE(n_slots >= 1 && n_slots <= (1ll << 28), "n_slots out of [1, 2^28]");
    DSA_REQUIRE(n_req >= 1, "n_req must be >= 1");
    if (nq == 0) return DSA_OK;
    DSA_REQUIRE(index_q && gate && q_req && q_pos && summaries && scales && sum_base && scores, "NULL pointer");
    DSA_REQUIRE(aligned(index_q, 16) && aligned(summaries, 16), "index_q and summaries must be 16-byte aligned");
    DSA_REACHABLE({index_q, "index_q"}, {gate, "gate"}, {q_req, "q_req"}, {q_pos, "q_pos"}, {summaries, "summaries"},
                  {scales, "scales"}, {sum_base, "sum_base"}, {scores, "scores"}, {ws, "ws"});
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;

    if ((flags & DSA_Q_FP8) && n_req == 1 && nq >= kGemmMinQueries && ws && ws_bytes >= gemm_ws_size(nq) &&
        aligned(ws, 256) && aligned(scales, 16))
        return indexer_gemm_path(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, scores,
                                 ld_scores, ws, sms, stream);
    return scan_path(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, n_req, scores, ld_scores,
                     flags, sms, stream);
}

size_t dsa_topk_workspace_size(int nq, int64_t ld_scores, int k)
{
    if (nq <= 0 || ld_scores < 1 || k < 1) return 0;
    return topk_layout(nq, ld_scores, k).total;
}

dsa_status_t dsa_topk_regions(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq, int k,
                              int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    DSA_REQUIRE(nq >= 0, "nq must be >= 0");
    DSA_REQUIRE(k >= 1 && k <= DSA_MAX_TOPK, "k out of [1, DSA_MAX_TOPK]");
    DSA_REQUIRE(ld_scores >= 1 && ld_scores < dsa::topk::kMaxRegions, "ld_scores out of [1, 2^20)");
    if (nq == 0) return DSA_OK;
    DSA_REQUIRE(scores && q_pos && sel_idx && sel_count, "NULL pointer");
    DSA_REACHABLE({scores, "scores"}, {q_pos, "q_pos"}, {sel_idx, "sel_idx"}, {sel_count, "sel_count"}, {ws, "ws"});
    return topk_dispatch(scores, ld_scores, q_pos, nq, k, sel_idx, sel_count, ws, ws_bytes, stream, dsa::kG);
}

dsa_status_t dsa_topk_regions_noalloc(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq, int k,
                                      int32_t *sel_idx, int32_t *sel_count, dsa_stream_t stream)
{
    DSA_REQUIRE(nq >= 0, "nq must be >= 0");
    DSA_REQUIRE(k >= 1 && k <= DSA_MAX_TOPK, "k out of [1, DSA_MAX_TOPK]");
    DSA_REQUIRE(ld_scores >= 1 && ld_scores < dsa::topk::kMaxRegions, "ld_scores out of [1, 2^20)");
    if (nq == 0) return DSA_OK;
    DSA_REQUIRE(scores && q_pos && sel_idx && sel_count, "NULL pointer");
    DSA_REACHABLE({scores, "scores"}, {q_pos, "q_pos"}, {sel_idx, "sel_idx"}, {sel_count, "sel_count"});
    const size_t need = topk_layout(nq, ld_scores, k).total;
    if (need > DSA_TOPK_STATIC_SCRATCH_BYTES)
        return fail(DSA_ERR_UNSUPPORTED, "dsa_topk_regions_noalloc: this call needs " + std::to_string(need) +
                                             " bytes of scratch, the static buffer holds " +
                                             std::to_string((size_t)DSA_TOPK_STATIC_SCRATCH_BYTES) +
                                             " (use dsa_topk_regions with a workspace)");
    int dev = 0;
    DSA_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    void *ws = nullptr;
    dsa_status_t st = static_scratch(dev, &ws);
    if (st != DSA_OK) return st;
    return topk_workspace_path(scores, ld_scores, q_pos, nq, k, sel_idx, sel_count, ws, need, stream);
}

// ---- decode selection in one call: the scan writes chunk maxima, the cluster top-k reads them
namespace {
int64_t cm_stride_of(int64_t ld) { return ((ld + 31) / 32 + 7) / 8 * 8; }
}  // namespace

size_t dsa_decode_select_workspace_size(int nq, int64_t ld_scores, int k)
{
    if (nq <= 0 || ld_scores < 1) return 0;
    const size_t cm = round_up((size_t)nq * dsa::kG * (size_t)cm_stride_of(ld_scores) * 4, 256);
    return cm + dsa_topk_workspace_size(nq, ld_scores, k);
}

namespace {
// Scores and selection of the KV groups g0 .. g0 + ng - 1 (all four: g0 = 0, ng = 4); the
// arguments are checked by the callers.
dsa_status_t decode_select_impl(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos,
                                int nq, const uint8_t *summaries, const float *scales, int64_t n_slots,
                                const int64_t *sum_base, int n_req, float *scores, int64_t ld_scores, uint32_t flags,
                                int k, int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes,
                                dsa_stream_t stream, int g0, int ng)
{
    const size_t need_ws = dsa_decode_select_workspace_size(nq, ld_scores, k);
    if (!ws || ws_bytes < need_ws || !aligned(ws, 256))
        return fail(DSA_ERR_WORKSPACE, "decode-select workspace too small or not 256-byte aligned (need " +
                                           std::to_string(need_ws) + " bytes)");
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    const int64_t cm_stride = cm_stride_of(ld_scores);
    float *chunk_max = static_cast<float *>(ws);
    const size_t cm = round_up((size_t)nq * dsa::kG * (size_t)cm_stride * 4, 256);
    const int cl = cluster_size_for(ld_scores);
    const bool maxima = k <= 512 && cl > 1 && (int64_t)nq * ng * cl <= 2 * sms;
    if ((st = scan_path(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, n_req, scores,
                        ld_scores, flags, sms, stream, maxima ? chunk_max : nullptr, cm_stride, g0, ng)) != DSA_OK)
        return st;
    if (!maxima)
        return topk_dispatch(scores, ld_scores, q_pos, nq, k, sel_idx, sel_count, static_cast<uint8_t *>(ws) + cm,
                             ws_bytes - cm, stream, ng);
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::topkc::topk_cluster_kernel<false, true>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsa::topkc::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(topk_cluster_kernel)");
    return launch_k("topk_cluster_kernel", dsa::topkc::topk_cluster_kernel<false, true>,
                    dim3((unsigned)cl, (unsigned)(nq * ng), 1), dim3(dsa::topkc::kThreads),
                    dsa::topkc::kSmemBytes, stream, (unsigned)cl, scores, ld_scores, q_pos, k, sel_idx, sel_count,
                    static_cast<const float *>(chunk_max), cm_stride, gshift_of(ng));
}

// Checks of the arguments dsa_decode_select and dsa_decode_select_groups share.
dsa_status_t decode_select_args(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos,
                                int nq, const uint8_t *summaries, const float *scales, int64_t n_slots,
                                const int64_t *sum_base, int n_req, float *scores, int64_t ld_scores, uint32_t flags,
                                int k, int32_t *sel_idx, int32_t *sel_count, void *ws)
{
    DSA_REQUIRE(nq >= 0, "nq must be >= 0");
    DSA_REQUIRE((flags & ~DSA_Q_FP8) == 0, "unknown flag");
    DSA_REQUIRE(ld_scores >= 1 && ld_scores <= (1ll << 26), "ld_scores out of [1, 2^26]");
    DSA_REQUIRE(n_slots >= 1 && n_slots <= (1ll << 28), "n_slots out of [1, 2^28]");
    DSA_REQUIRE(n_req >= 1, "n_req must be >= 1");
    DSA_REQUIRE(k >= 1 && k <= DSA_MAX_TOPK, "k out of [1, DSA_MAX_TOPK]");
    if (nq == 0) return DSA_OK;
    DSA_REQUIRE(index_q && gate && q_req && q_pos && summaries && scales && sum_base && scores && sel_idx && sel_count,
                "NULL pointer");
    DSA_REQUIRE(aligned(index_q, 16) && aligned(summaries, 16), "index_q and summaries must be 16-byte aligned");
    DSA_REACHABLE({index_q, "index_q"}, {gate, "gate"}, {q_req, "q_req"}, {q_pos, "q_pos"}, {summaries, "summaries"},
                  {scales, "scales"}, {sum_base, "sum_base"}, {scores, "scores"}, {sel_idx, "sel_idx"},
                  {sel_count, "sel_count"}, {ws, "ws"});
    return DSA_OK;
}
}  // namespace

dsa_status_t dsa_decode_select(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos,
                               int nq, const uint8_t *summaries, const float *scales, int64_t n_slots,
                               const int64_t *sum_base, int n_req, float *scores, int64_t ld_scores, uint32_t flags,
                               int k, int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes,
                               dsa_stream_t stream)
{
    dsa_status_t st = decode_select_args(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, n_req,
                                         scores, ld_scores, flags, k, sel_idx, sel_count, ws);
    if (st != DSA_OK || nq == 0) return st;
    return decode_select_impl(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, n_req, scores,
                              ld_scores, flags, k, sel_idx, sel_count, ws, ws_bytes, stream, 0, dsa::kG);
}

dsa_status_t dsa_decode_select_groups(const void *index_q, const float *gate, const int32_t *q_req,
                                      const int32_t *q_pos, int nq, int g0, int ng, const uint8_t *summaries,
                                      const float *scales, int64_t n_slots, const int64_t *sum_base, int n_req,
                                      float *scores, int64_t ld_scores, uint32_t flags, int k, int32_t *sel_idx,
                                      int32_t *sel_count, void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    dsa_status_t st = group_range_args(g0, ng);
    if (st != DSA_OK) return st;
    st = decode_select_args(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, n_req, scores,
                            ld_scores, flags, k, sel_idx, sel_count, ws);
    if (st != DSA_OK || nq == 0) return st;
    return decode_select_impl(index_q, gate, q_req, q_pos, nq, summaries, scales, n_slots, sum_base, n_req, scores,
                              ld_scores, flags, k, sel_idx, sel_count, ws, ws_bytes, stream, g0, ng);
}

dsa_status_t dsa_copy(void *dst, const void *src, size_t bytes, dsa_stream_t stream)
{
    if (bytes == 0) return DSA_OK;
    DSA_REQUIRE(dst && src, "NULL pointer");
    DSA_REACHABLE({dst, "dst"}, {src, "src"});
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    const size_t per_block = 256 * 16 * 4;                 // about 4 uint4 per thread
    const unsigned blocks = (unsigned)std::min<size_t>((bytes + per_block - 1) / per_block, (size_t)sms * 4);
    return launch_k("copy_kernel", dsa::copy_kernel, dim3(std::max(1u, blocks)), dim3(256), 0, stream, 0,
                    static_cast<uint8_t *>(dst), static_cast<const uint8_t *>(src), bytes);
}

size_t dsa_attn_workspace_size(int nq, int k)
{
    if (nq <= 0 || k < 1) return 0;
    int sms = 0;
    if (device_info(sms) != DSA_OK) sms = 148;
    // split partials, and the per-row flags of the shared-selection prefill kernel
    return attn_plan(nq, k, sms).ws + round_up((size_t)nq * dsa::kG, 256);
}

dsa_status_t dsa_sparse_attn_decode(const void *q, const void *k_cache, const void *v_cache, int64_t n_pages,
                                    const int32_t *block_table, int max_pages, const int32_t *q_pos, int batch,
                                    const int32_t *sel_idx, const int32_t *sel_count, int k, void *out, float *lse,
                                    void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    return attn_common(q, k_cache, v_cache, n_pages, block_table, max_pages, nullptr, batch, q_pos, batch, sel_idx,
                       sel_count, k, out, lse, ws, ws_bytes, stream);
}

size_t dsa_attn_groups_workspace_size(int nq, int k, int ng)
{
    if (nq <= 0 || k < 1 || !(ng == 1 || ng == 2 || ng == 4)) return 0;
    int sms = 0;
    if (device_info(sms) != DSA_OK) sms = 148;
    return attn_plan(nq, k, sms, ng).ws;
}

dsa_status_t dsa_sparse_attn_decode_groups(const void *q, const void *k_cache, const void *v_cache, int64_t n_pages,
                                           const int32_t *block_table, int max_pages, const int32_t *q_pos, int batch,
                                           int g0, int ng, const int32_t *sel_idx, const int32_t *sel_count, int k,
                                           void *out, float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    dsa_status_t st = group_range_args(g0, ng);
    if (st != DSA_OK) return st;
    return attn_common(q, k_cache, v_cache, n_pages, block_table, max_pages, nullptr, batch, q_pos, batch, sel_idx,
                       sel_count, k, out, lse, ws, ws_bytes, stream, 0, g0, ng);
}

dsa_status_t dsa_indexer_frontend(const void *hidden, int hid, int n_tok, const void *w, const void *gamma_q,
                                  const void *gamma_k, const int32_t *pos, void *index_q, void *index_k, float *z,
                                  dsa_stream_t stream)
{
    DSA_REQUIRE(n_tok >= 0, "n_tok must be >= 0");
    DSA_REQUIRE(hid >= 8 && hid % 8 == 0 && hid <= (1 << 20), "hid must be a multiple of 8 in [8, 2^20]");
    if (n_tok == 0) return DSA_OK;
    DSA_REQUIRE(hidden && w && gamma_q && gamma_k && pos && index_q && index_k && z, "NULL pointer");
    DSA_REQUIRE(aligned(hidden, 16) && aligned(w, 16) && aligned(index_q, 16) && aligned(index_k, 16) &&
                    aligned(z, 16),
                "hidden, w, index_q, index_k and z must be 16-byte aligned");
    DSA_REACHABLE({hidden, "hidden"}, {w, "w"}, {gamma_q, "gamma_q"}, {gamma_k, "gamma_k"}, {pos, "pos"},
                  {index_q, "index_q"}, {index_k, "index_k"}, {z, "z"});
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    CUtensorMap map_h, map_w;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)hid, (cuuint64_t)n_tok};
        const cuuint64_t strides[1] = {(cuuint64_t)hid * 2};
        const cuuint32_t box[2] = {(cuuint32_t)dsa::fe::kBK, (cuuint32_t)dsa::fe::kBM};
        if ((st = encode(&map_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, hidden, dims, strides, box,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B)) != DSA_OK)
            return st;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)hid, (cuuint64_t)dsa::fe::kRows};
        const cuuint64_t strides[1] = {(cuuint64_t)hid * 2};
        const cuuint32_t box[2] = {(cuuint32_t)dsa::fe::kBK, (cuuint32_t)dsa::fe::kBN};
        if ((st = encode(&map_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w, dims, strides, box,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B)) != DSA_OK)
            return st;
    }
    dsa::fe::Params p{};
    p.gamma_q = static_cast<const __nv_bfloat16 *>(gamma_q);
    p.gamma_k = static_cast<const __nv_bfloat16 *>(gamma_k);
    p.pos = pos;
    p.index_q = static_cast<__nv_bfloat16 *>(index_q);
    p.index_k = static_cast<__nv_bfloat16 *>(index_k);
    p.z = z;
    p.n_tok = n_tok;
    p.n_k = (hid + dsa::fe::kBK - 1) / dsa::fe::kBK;
    p.n_units = (n_tok + dsa::fe::kBM - 1) / dsa::fe::kBM * dsa::fe::kUnitsPerTile;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(dsa::fe::frontend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)dsa::fe::kSmemBytes);
    });
    DSA_CUDA(attr_err, "cudaFuncSetAttribute(frontend_kernel)");
    return launch_k("frontend_kernel", dsa::fe::frontend_kernel, dim3((unsigned)std::min(sms, p.n_units)),
                    dim3(dsa::fe::kThreads), dsa::fe::kSmemBytes, stream, 0, map_h, map_w, p);
}

namespace {
// The window call runs on the clustered kernel (splits merged in the kernel, one launch).
bool window_clustered(int nq, int window)
{
    return window_regions(window) <= dsa::attnc::Window::kMaxK && (int64_t)nq * dsa::kG <= WindowAttn::capacity();
}
}  // namespace

int dsa_window_decode_launches(int nq, int window)
{
    if (nq <= 0 || window < 1) return 0;
    if (window_clustered(nq, window)) return 1;                            // the append folded in
    int sms = 0;
    if (device_info(sms) != DSA_OK) sms = 148;
    return 1 + (attn_plan(nq, window_regions(window), sms).n_splits > 1 ? 2 : 1);
}

size_t dsa_window_attn_workspace_size(int nq, int window)
{
    if (nq <= 0 || window < 1) return 0;
    int sms = 0;
    if (device_info(sms) != DSA_OK) sms = 148;
    return attn_plan(nq, window_regions(window), sms).ws;
}

dsa_status_t dsa_window_attn(const void *q, const void *k_cache, const void *v_cache, int64_t n_pages,
                             const int32_t *block_table, int max_pages, int n_req, const int32_t *q_req,
                             const int32_t *q_pos, int nq, int window, void *out, float *lse, void *ws,
                             size_t ws_bytes, dsa_stream_t stream)
{
    DSA_REQUIRE(window >= 1 && window <= (1 << 20), "window out of [1, 2^20]");
    return attn_common(q, k_cache, v_cache, n_pages, block_table, max_pages, q_req, q_req ? n_req : nq, q_pos, nq,
                       nullptr, nullptr, window_regions(window), out, lse, ws, ws_bytes, stream, window);
}

dsa_status_t dsa_window_decode(void *k_cache, void *v_cache, int64_t n_pages, const int32_t *block_table,
                               int max_pages, int n_req, const int32_t *q_req, const int32_t *q_pos, int nq,
                               const void *new_k, const void *new_v, const void *q, int window, void *out,
                               float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    DSA_REQUIRE(window >= 1 && window <= (1 << 20), "window out of [1, 2^20]");
    DSA_REQUIRE(nq >= 0, "nq must be >= 0");
    if (nq == 0) return DSA_OK;
    DSA_REQUIRE(new_k && new_v, "NULL pointer");
    DSA_REQUIRE(aligned(new_k, 16) && aligned(new_v, 16), "new rows must be 16-byte aligned");
    DSA_REACHABLE({new_k, "new_k"}, {new_v, "new_v"});
    if (!window_clustered(nq, window)) {
        // the two calls it stands for
        dsa_status_t st = dsa_kv_append(k_cache, v_cache, n_pages, block_table, max_pages, n_req, q_req, q_pos, nq,
                                        new_k, new_v, stream);
        if (st != DSA_OK) return st;
        return dsa_window_attn(q, k_cache, v_cache, n_pages, block_table, max_pages, n_req, q_req, q_pos, nq, window,
                               out, lse, ws, ws_bytes, stream);
    }
    return attn_common(q, k_cache, v_cache, n_pages, block_table, max_pages, q_req, q_req ? n_req : nq, q_pos, nq,
                       nullptr, nullptr, window_regions(window), out, lse, ws, ws_bytes, stream, window, 0, dsa::kG,
                       new_k, new_v);
}

dsa_status_t dsa_kv_append(void *k_cache, void *v_cache, int64_t n_pages, const int32_t *block_table, int max_pages,
                           int n_req, const int32_t *q_req, const int32_t *q_pos, int n, const void *new_k,
                           const void *new_v, dsa_stream_t stream)
{
    DSA_REQUIRE(n >= 0, "n must be >= 0");
    DSA_REQUIRE(n_pages >= 1 && n_pages <= (INT32_MAX / (dsa::kG * dsa::kPage)), "n_pages out of range");
    DSA_REQUIRE(max_pages >= 1, "max_pages must be >= 1");
    if (n == 0) return DSA_OK;
    DSA_REQUIRE(k_cache && v_cache && block_table && q_pos && new_k && new_v, "NULL pointer");
    DSA_REQUIRE(q_req == nullptr || n_req >= 1, "n_req must be >= 1");
    DSA_REQUIRE(aligned(k_cache, 16) && aligned(v_cache, 16) && aligned(new_k, 16) && aligned(new_v, 16),
                "caches and new rows must be 16-byte aligned");
    DSA_REACHABLE({k_cache, "k_cache"}, {v_cache, "v_cache"}, {block_table, "block_table"}, {q_req, "q_req"},
                  {q_pos, "q_pos"}, {new_k, "new_k"}, {new_v, "new_v"});
    return launch_k("kv_append_kernel", dsa::kv_append_kernel, dim3((unsigned)n), dim3(256), 0, stream, 0,
                    static_cast<__nv_bfloat16 *>(k_cache), static_cast<__nv_bfloat16 *>(v_cache), n_pages,
                    block_table, max_pages, q_req, q_req ? n_req : n, q_pos, n,
                    static_cast<const __nv_bfloat16 *>(new_k), static_cast<const __nv_bfloat16 *>(new_v));
}

dsa_status_t dsa_sparse_attn_prefill(const void *q, const void *k_cache, const void *v_cache, int64_t n_pages,
                                     const int32_t *block_table, int max_pages, int n_req, const int32_t *q_req,
                                     const int32_t *q_pos, int nq, const int32_t *sel_idx, const int32_t *sel_count,
                                     int k, void *out, float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream)
{
    DSA_REQUIRE(q_req != nullptr || nq == 0, "q_req must not be NULL");
    return attn_common(q, k_cache, v_cache, n_pages, block_table, max_pages, q_req, n_req, q_pos, nq, sel_idx,
                       sel_count, k, out, lse, ws, ws_bytes, stream);
}

dsa_status_t dsa_selftest_wait_timeout(int64_t limit_cycles, dsa_stream_t stream)
{
    DSA_REQUIRE(limit_cycles >= 1 && limit_cycles <= dsa::kWaitLimitCycles,
                "limit_cycles out of [1, 2^31]");
    int sms = 0;
    dsa_status_t st = device_info(sms);
    if (st != DSA_OK) return st;
    return launch_k("wait_timeout_kernel", dsa::wait_timeout_kernel, dim3(1), dim3(64), 0, stream, 0,
                    (long long)limit_cycles);
}

}  // extern "C"
