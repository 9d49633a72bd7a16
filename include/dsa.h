/*
 * dsa.h: C-ABI of libdsa, DSA region-sparse GQA on NVIDIA B200 (sm_100a).
 *
 * DSA is the sparse attention of Step-5-Preview's 23 full-attention layers.  Pages
 * cited (title, site):
 *   [P1] Step-5-Preview 百万 token 长上下文: 滑窗 + DSA (kwkr.cn/news/601179)
 *   [P2] Step-5-Preview 如何实现1M长上下文？滑窗+DSA稀疏注意力混合机制完整揭秘 (yfxerp.com/news/376439)
 *   [P3] 100 万 token 上下文实测：Step 5 Preview 一次能吞下多大的工程 (kwkr.cn/news/593658)
 *
 * The method has four steps, one call each (plus the fused decode selection):
 *   dsa_compress_regions     A1  8-token regions -> 256-d e4m3 summaries     [P1 §DSA ②][P2 §区域压缩CSA]
 *   dsa_indexer_scores       A2  16-head indexer score per (query, region)   [P1 §DSA ③][P2 §索引器打分]
 *   dsa_topk_regions         A3  own region + top-(k-1), ties -> lower index [P2 §索引器打分]
 *   dsa_sparse_attn_decode   A4  exact GQA over the selected regions         [P1 §DSA ④][P3 §一]
 *   dsa_sparse_attn_prefill  A4  the same for a chunk of prefill queries     [P3 §一 sparse_attention_prefill]
 * and, for the window layers beside the DSA layers:
 *   dsa_kv_append            new tokens' K/V into their page slots (a ring with a cyclic table)
 *   dsa_window_attn          GQA over each query's last `window` tokens      [P1 §滑窗注意力][P2 §第一招]
 * and the indexer's front end, upstream of A1/A2:
 *   dsa_indexer_frontend     hidden state -> index_q, index_k, gates        [P2 §索引器打分]
 *
 * Conventions (every call):
 *   - Pointers are DEVICE pointers unless stated otherwise, owned by the caller.  Every
 *     pointer argument is checked on the host (cudaPointerGetAttributes) before anything is
 *     launched: device memory of another GPU, and pageable host memory on a GPU that cannot
 *     read pageable memory, return DSA_ERR_INVALID_ARG (a kernel touching them would fault).
 *     Pinned or registered host memory and managed memory are accepted.  The
 *     library never allocates device memory; scratch comes from a caller-provided
 *     workspace `ws` of at least the size the matching *_workspace_size() returns,
 *     aligned to 256 bytes.  Workspace contents need not be initialised and are
 *     clobbered.  Calls that share a workspace must not overlap on the GPU.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and never synchronise it.  The return value reflects the synchronous
 *     host-side argument checks and the launch; errors that only the kernels can see
 *     (an index read from device memory out of range, a bounded wait that gave up)
 *     set a per-device error word that dsa_check_device() reads and clears.
 *   - All tensors are dense row-major with the shapes given; bf16 is IEEE bfloat16,
 *     e4m3 is the OCP FP8 E4M3 ("fn") byte format.
 *   - dsa_last_error() returns a thread-local message for the last failed call.
 *
 * Shapes: G = 4 KV groups, HI = 16 indexer heads (head h in group h/4), DI = 256,
 * HQ = 64 query heads (head h uses KV group h/16), D = 192, regions of 8 tokens,
 * K/V pages of 64 tokens (8 regions).
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_VERSION 100          /* 1.0.0 */

#define DSA_REGION_TOKENS 8      /* [P1 §DSA ①] REGION_BLOCK_SIZE */
#define DSA_GROUPS 4             /* [P3 §一] num_attention_groups; [P2 §索引器打分] num_provider_groups */
#define DSA_PROXY_DIM 256        /* [P2 §第二招] proxy_dim */
#define DSA_INDEX_HEADS 16       /* [P1 §DSA ③] 16-head sparse indexer */
#define DSA_Q_HEADS 64           /* [P3 §一] num_attention_heads */
#define DSA_HEAD_DIM 192         /* [P3 §三] 2 x 4 x 192 x 2 bytes per token per layer */
#define DSA_PAGE_TOKENS 64       /* K/V page size of the paged cache ([P3 §一] block_table) */
#define DSA_MAX_TOPK 2048        /* largest k accepted (the method uses 512, [P2 §第二招]) */

/* flags for dsa_indexer_scores */
#define DSA_Q_FP8 1u             /* quantise index_q per (query, head) to e4m3 (absmax/448
                                    scale) before scoring: an FP8 x FP8 contraction */

typedef struct CUstream_st *dsa_stream_t;   /* identical to cudaStream_t */

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,     /* a host-visible argument is out of range or NULL */
    DSA_ERR_UNSUPPORTED = 2,     /* the device is not sm_100 or a size exceeds a limit */
    DSA_ERR_WORKSPACE = 3,       /* ws too small or not 256-byte aligned */
    DSA_ERR_CUDA = 4,            /* a CUDA runtime call failed (launch, attribute, ...) */
    DSA_ERR_DEVICE = 5           /* a kernel flagged an error (dsa_check_device) */
} dsa_status_t;

/* Library version (DSA_VERSION of the build). */
int dsa_version(void);

/* Message for the last non-OK status returned on this host thread ("" if none).
 * The pointer stays valid until the next call on this thread. */
const char *dsa_last_error(void);

/* The same message copied into a caller buffer, for callers that keep no pointer into the
 * library: writes at most len - 1 bytes of it and a terminating NUL into buf (nothing when
 * len is 0; buf may then be NULL) and returns the message's full length, so a return value
 * >= len means it was cut short. */
size_t dsa_get_last_error(char *buf, size_t len);

/* Synchronises `stream`, then reads and clears the error word that kernels of this
 * library set on the current device.  Returns DSA_OK or DSA_ERR_DEVICE (message via
 * dsa_last_error), or DSA_ERR_CUDA if the synchronisation itself failed. */
dsa_status_t dsa_check_device(dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* A1 region compression.  [P1 §DSA ②] every complete 8-token region is collapsed into a
 * 256-d summary stored as FP8; [P2 §区域压缩CSA] only full regions are summarised, a
 * tail of fewer than 8 tokens waits.  For region i and group g:
 *   m_j   = fp32( sum_{t=0..7} index_k[src_row[i]+t][g][j] / 8 )   (sum in fp64, t = 0..7)
 *   scale = fp32( max_j |m_j| / 448 )
 *   code_j = e4m3_RNE_satfinite( fp32(m_j / scale) ),  all 0 when scale = 0
 * index_k   bf16  [n_rows][row_stride]; token row t of group g is index_k[t*row_stride + g*256 + j]
 *           (row_stride >= 1024 elements, a multiple of 8)
 * src_row   int64 [n_regions]   first row of region i (rows src_row[i] .. +7, must be < n_rows)
 * dst_slot  int64 [n_regions]   pool slot written for region i (0 <= slot < n_slots)
 * summaries e4m3  [4][n_slots][256]   (group-major pool)
 * scales    fp32  [4][n_slots]
 * Out-of-range src_row/dst_slot values are skipped and flag DSA_ERR_DEVICE.  Regions
 * written to the same slot in one call race.  n_regions == 0 is a no-op. */
dsa_status_t dsa_compress_regions(const void *index_k, int64_t row_stride, int64_t n_rows,
                                  const int64_t *src_row, const int64_t *dst_slot, int n_regions,
                                  uint8_t *summaries, float *scales, int64_t n_slots,
                                  dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* A2 indexer scores.  [P1 §DSA ③][P2 §索引器打分] the 16-head indexer scores each query
 * against every region summary of its request; regions and heads map onto the 4 KV
 * groups (heads 4g..4g+3 score group g):
 *   score[q][g][r] = sum_{h=4g}^{4g+3} gate[q][h] * ReLU(index_q[q][h] . s_{r,g}) / 16,
 *   s_{r,g} = e4m3 value of summaries[g][sum_base[b]+r] * scales[g][sum_base[b]+r],
 * for r = 0 .. own-1 where own = q_pos[q] / 8 (the regions complete before the query's
 * own region; the own region itself is forced by dsa_topk_regions, not scored).
 * Entries r >= own are not written.  Accumulation is fp32 on the tensor cores.
 * index_q   bf16  [nq][16][256]
 * gate      fp32  [nq][16]
 * q_req     int32 [nq]      request of each query (index into sum_base)
 * q_pos     int32 [nq]      0-based position of the query token
 * sum_base  int64 [n_req]   pool slot of region 0 of each request
 * scores    fp32  [nq][4][ld_scores]
 * flags     0 or DSA_Q_FP8
 * A query whose own > ld_scores, q_req out of [0, n_req) or sum_base[b]+own > n_slots
 * is skipped and flags DSA_ERR_DEVICE.
 * Two kernels serve the call.  A call with DSA_Q_FP8 over one request's chunk (n_req == 1,
 * nq >= 64) and a workspace of dsa_indexer_workspace_size(nq, ld) bytes (256-byte
 * aligned, owned by the caller, not kept after the stream reaches the end of the call)
 * and 16-byte aligned scales runs as a tcgen05 FP8 x FP8 GEMM per group; every other call
 * (decode batches, several requests, bf16 queries, ws == NULL or unaligned scales) runs
 * the streaming scan, which needs no workspace.  Both compute the same scores up to fp32
 * summation order. */
size_t dsa_indexer_workspace_size(int nq, int64_t ld_scores);
dsa_status_t dsa_indexer_scores(const void *index_q, const float *gate, const int32_t *q_req,
                                const int32_t *q_pos, int nq, const uint8_t *summaries,
                                const float *scales, int64_t n_slots, const int64_t *sum_base,
                                int n_req, float *scores, int64_t ld_scores, uint32_t flags,
                                void *ws, size_t ws_bytes, dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* A3 top-k region selection.  [P2 §索引器打分] a radix-style top-k keeps the best regions
 * and always includes the query's own region; [P2 §第二招] at most k = 512 per query.
 * Per (query q, group g), own = q_pos[q] / 8: the own region plus the k-1 best of the
 * regions r < own ordered by (score descending, region index ascending); equal values
 * (+0 and -0 included) tie.  Output ascending region indices:
 *   sel_idx   int32 [nq][4][k]   first sel_count entries valid, the rest -1
 *   sel_count int32 [nq][4]      min(k, own + 1)
 * scores    fp32  [nq][4][ld_scores]; only entries r < own are read.  NaN scores are
 *           not supported (their rank is unspecified).
 * 1 <= k <= DSA_MAX_TOPK.  A query with own > ld_scores flags DSA_ERR_DEVICE and gets
 * count 0. */
size_t dsa_topk_workspace_size(int nq, int64_t ld_scores, int k);
dsa_status_t dsa_topk_regions(const float *scores, int64_t ld_scores, const int32_t *q_pos, int nq,
                              int k, int32_t *sel_idx, int32_t *sel_count, void *ws,
                              size_t ws_bytes, dsa_stream_t stream);

/* Allocation-free top-k (no counterpart in the pages: a library convenience).  Same
 * computation and results as dsa_topk_regions, for callers that cannot allocate device
 * memory at the point of the call: code running while another component owns the
 * device allocator (a serving runtime whose memory pool is fully reserved), or a
 * plain-C host without a device allocator of its own.  The caller passes only inputs
 * and outputs; the scratch lives in one static device array inside libdsa,
 * DSA_TOPK_STATIC_SCRATCH_BYTES (8 MiB) per GPU, held by every GPU that loads the library
 * until the process exits.  A call needs dsa_topk_workspace_size(nq, ld_scores, k)
 * bytes of it (a 1M-token request, k = 512: about 4.3 MB); larger calls return
 * DSA_ERR_UNSUPPORTED.  No cudaMalloc/cudaFree or allocating routine is called.
 *   - The first call on a device resolves the array's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 *   - Every call on a device shares the one array and it keeps the previous call's
 *     contents (the call clears what must start at zero itself): calls whose kernels
 *     overlap on the GPU (different streams, concurrent graphs) race and must be
 *     serialised by the caller. */
#define DSA_TOPK_STATIC_SCRATCH_BYTES (8u << 20)
dsa_status_t dsa_topk_regions_noalloc(const float *scores, int64_t ld_scores, const int32_t *q_pos,
                                      int nq, int k, int32_t *sel_idx, int32_t *sel_count,
                                      dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* A2 + A3 in one call, for decode: the streaming scan of dsa_indexer_scores followed by the
 * selection of dsa_topk_regions, with the same arguments and exactly their outputs (the
 * scores in `scores`, the selection in sel_idx/sel_count).  The scan also writes, into the
 * workspace, the largest score of every chunk of 32 regions, and for few long rows (k <= 512,
 * rows of up to 131,072 regions, one cluster per row) the selection bounds its threshold
 * from those maxima and reads only the chunks that can hold a selected region; other calls
 * select as dsa_topk_regions does.  Compression of filled regions ([P2 §区域压缩CSA]) is not
 * part of it.  ws: dsa_decode_select_workspace_size(nq, ld_scores, k) bytes, 256-byte
 * aligned, owned by the caller, free again once the stream has passed the call; a smaller or
 * unaligned one returns DSA_ERR_WORKSPACE.  Invalid queries flag DSA_ERR_DEVICE as in the
 * two calls. */
size_t dsa_decode_select_workspace_size(int nq, int64_t ld_scores, int k);
dsa_status_t dsa_decode_select(const void *index_q, const float *gate, const int32_t *q_req, const int32_t *q_pos,
                               int nq, const uint8_t *summaries, const float *scales, int64_t n_slots,
                               const int64_t *sum_base, int n_req, float *scores, int64_t ld_scores, uint32_t flags,
                               int k, int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes,
                               dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* Byte copy by a kernel, for staging a step's inputs: dst and src are any addresses the
 * current device can reach (device memory, or pinned host memory, which unified addressing
 * maps at the same address).  Launched like every call of this library, it joins the
 * stream's kernel chain without a copy-engine operation in between.  Regions must not
 * overlap.  bytes == 0 is a no-op. */
dsa_status_t dsa_copy(void *dst, const void *src, size_t bytes, dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* A4 sparse GQA attention.  [P1 §DSA ④] exact attention over only the selected regions'
 * real K/V; [P3 §一] the selected regions are gathered from the paged cache through the
 * block_table.  For query q (request b = q_req[q], position p = q_pos[q]) and head h
 * (group g = h/16): T = union of tokens 8r..8r+7 over r in sel_idx[q][g][0..cnt), kept
 * where t <= p (the causal mask inside the own region);
 *   out[q][h] = sum_{t in T} softmax_t(q[q][h] . K_t / sqrt(192)) V_t   (bf16, fp32 math)
 *   lse[q][h] = ln sum_{t in T} exp(q[q][h] . K_t / sqrt(192))          (-inf if T empty)
 * q           bf16  [nq][64][192]  (already rotated)
 * k_cache     bf16  [n_pages][4][64][192]; token t of request b is row t%64 of page
 * v_cache     bf16  [n_pages][4][64][192]   block_table[b*max_pages + t/64]
 * block_table int32 [n_req][max_pages]
 * sel_idx     int32 [nq][4][k], sel_count int32 [nq][4]  (as written by dsa_topk_regions)
 * out         bf16  [nq][64][192]
 * lse         fp32  [nq][64] or NULL
 * A selected region beyond the block table, a page index outside [0, n_pages) or a
 * q_req outside [0, n_req) is skipped and flags DSA_ERR_DEVICE.  An empty T gives
 * out = 0.  decode: one query per request, q_req = identity (nq = n_req = batch).
 * Kernels: rows of one or two decode requests run as one 16-CTA cluster per row with the
 * splits merged in the kernel; prefill calls of >= 32 queries first try the shared-selection
 * kernel (8 neighbouring queries of a request stream the union of their selections once,
 * kept when the union is at most twice the longest selection, [P5]); every other row runs
 * the per-row kernel (split across CTAs, with a merge kernel, when there are few rows).
 * The results do not depend on the kernel.  Workspace: dsa_attn_workspace_size(nq, k)
 * bytes (split partials and one flag per row; it depends on the current device's SM
 * count), 256-byte aligned, owned by the caller; a smaller one returns DSA_ERR_WORKSPACE
 * when a kernel needs it. */
size_t dsa_attn_workspace_size(int nq, int k);
dsa_status_t dsa_sparse_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                                    int64_t n_pages, const int32_t *block_table, int max_pages,
                                    const int32_t *q_pos, int batch, const int32_t *sel_idx,
                                    const int32_t *sel_count, int k, void *out, float *lse,
                                    void *ws, size_t ws_bytes, dsa_stream_t stream);
dsa_status_t dsa_sparse_attn_prefill(const void *q, const void *k_cache, const void *v_cache,
                                     int64_t n_pages, const int32_t *block_table, int max_pages,
                                     int n_req, const int32_t *q_req, const int32_t *q_pos, int nq,
                                     const int32_t *sel_idx, const int32_t *sel_count, int k,
                                     void *out, float *lse, void *ws, size_t ws_bytes,
                                     dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* The window layers.  [P1 §滑窗注意力] 69 of the 92 layers read only the most recent 512
 * tokens; [P2 §第一招] their cache is a ring buffer keeping each request's last 512 tokens
 * (a new token overwrites the slot of the token 512 before it) and decode attends inside
 * the window.  A ring is a paged cache whose block table maps a request's virtual pages
 * cyclically onto a few physical pages: with 8 pages of 64 tokens (block_table[b][v] =
 * ring page (v mod 8) of b) token t lands on the slot of token t - 512.
 *
 * dsa_kv_append: writes token i's K and V rows (new_k, new_v bf16 [n][4][192]) to row
 * q_pos[i] % 64 of page block_table[b*max_pages + q_pos[i]/64], b = q_req[i] (q_req NULL:
 * b = i).  Caches as for dsa_sparse_attn_decode.  A position beyond the block table or a
 * page outside [0, n_pages) is skipped and flags DSA_ERR_DEVICE.  Tokens of one call must
 * not share a slot.
 *
 * dsa_window_attn: for query q (request b = q_req[q], or q when q_req is NULL; position
 * p = q_pos[q]) and head h (group g = h/16), T = { t : max(0, p - window + 1) <= t <= p },
 * read through the block table:
 *   out[q][h] = sum_{t in T} softmax_t(q[q][h] . K_t / sqrt(192)) V_t   (bf16, fp32 math)
 *   lse[q][h] = ln sum_{t in T} exp(q[q][h] . K_t / sqrt(192))          (NULL: not written)
 * The caller keeps every token of the window in the cache (a ring of at least `window`
 * tokens).  1 <= window <= 2^20.  A window of at most 624 tokens, with every (query,
 * group) row's 8-CTA cluster resident at once, runs in one kernel that merges the row's
 * splits in distributed shared memory; other calls run on the per-row attention kernel
 * (split across CTAs, with a merge kernel, when there are few rows).  Workspace
 * dsa_window_attn_workspace_size(nq, window) bytes, 256-byte aligned (0: none needed).
 * Errors as for the sparse calls.
 *
 * dsa_window_decode: one window-layer decode step, dsa_kv_append(new_k, new_v at q_pos)
 * followed by dsa_window_attn over the window that now ends at the appended token, with the
 * same arguments, results and errors as the two calls.  Where dsa_window_attn would run
 * its clustered kernel the append is folded into it (one launch: the CTA that holds a row's
 * newest region writes the token's K and V rows to the cache slot and attends them from
 * new_k / new_v); elsewhere it makes the two calls.  As for dsa_kv_append, the queries of one
 * call must be distinct requests (no query's window may hold another query's new token).
 *
 * dsa_window_decode_launches: the number of kernels dsa_window_decode(nq, window) launches
 * on the current device (1 where the append is folded in, else 2 or 3; 0 for nq <= 0 or
 * window < 1). */
dsa_status_t dsa_kv_append(void *k_cache, void *v_cache, int64_t n_pages, const int32_t *block_table,
                           int max_pages, int n_req, const int32_t *q_req, const int32_t *q_pos, int n,
                           const void *new_k, const void *new_v, dsa_stream_t stream);
size_t dsa_window_attn_workspace_size(int nq, int window);
dsa_status_t dsa_window_attn(const void *q, const void *k_cache, const void *v_cache, int64_t n_pages,
                             const int32_t *block_table, int max_pages, int n_req, const int32_t *q_req,
                             const int32_t *q_pos, int nq, int window, void *out, float *lse, void *ws,
                             size_t ws_bytes, dsa_stream_t stream);
dsa_status_t dsa_window_decode(void *k_cache, void *v_cache, int64_t n_pages, const int32_t *block_table,
                               int max_pages, int n_req, const int32_t *q_req, const int32_t *q_pos, int nq,
                               const void *new_k, const void *new_v, const void *q, int window, void *out,
                               float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream);
int dsa_window_decode_launches(int nq, int window);

/* ------------------------------------------------------------------------------ */
/* Indexer front end.  [P2 §索引器打分] the indexer projects the hidden state to index_q /
 * index_k / index_z, then normalises and applies RoPE to part of the dimensions.  The pages
 * give no constants; this library's reading, per token t at position pos[t]:
 *   a = W h_t                                  (W bf16 [5136][hid], fp32 accumulation; rows
 *                                               0..4095: 16 q heads x 256, 4096..5119: 4 k
 *                                               groups x 256, 5120..5135: 16 gates)
 *   each 256-d head vector x (q heads with gamma_q, k groups with gamma_k, bf16 [256]):
 *     y = x / sqrt(mean(x^2) + 1e-6) * gamma                                 (RMSNorm)
 *     dims 0..63 rotated in pairs (i, i + 32) by pos * 10000^(-i/32)         (partial RoPE)
 *   z_h = sigmoid(a_gate h)
 * hidden  bf16 [n_tok][hid] (hid a multiple of 8), pos int32 [n_tok]
 * index_q bf16 [n_tok][16][256], index_k bf16 [n_tok][4][256], z fp32 [n_tok][16]
 * (the layouts dsa_indexer_scores and dsa_compress_regions read).  All device pointers
 * 16-byte aligned except gamma_q, gamma_k and pos.  Runs as one tcgen05 bf16 GEMM with the
 * norm, rotation and gates in its epilogue; no workspace. */
dsa_status_t dsa_indexer_frontend(const void *hidden, int hid, int n_tok, const void *w, const void *gamma_q,
                                  const void *gamma_k, const int32_t *pos, void *index_q, void *index_k, float *z,
                                  dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* KV-group-sharded decode.  [P2 §索引器打分] the indexer's regions and heads map one to one
 * onto the 4 KV groups (num_provider_groups 4), and every step of the method is per group:
 * summaries, scores, selection and attention of group g touch only group g's data and its
 * heads (indexer heads 4g..4g+3, query heads 16g..16g+15).  A GPU that holds the groups
 * g0 .. g0+ng-1 (ng = 1, 2 or 4, g0 + ng <= 4; e.g. two GPUs with groups {0,1} and {2,3})
 * runs these calls on its own shard and produces exactly the rows of the 4-group calls for
 * its groups; the 16*ng heads of output per query are then gathered across GPUs by the
 * caller (one all-gather of 16 x 192 bf16 per group and query).  Layouts of a shard:
 *   summaries e4m3 [ng][n_slots][256], scales fp32 [ng][n_slots]   (local group gl = g - g0)
 *   k_cache / v_cache bf16 [n_pages][ng][64][192]
 *   scores fp32 [nq][ng][ld_scores], sel_idx int32 [nq][ng][k], sel_count int32 [nq][ng]
 *   out bf16 [nq][16*ng][192] (head 16*gl + i is query head 16*(g0+gl) + i), lse fp32 [nq][16*ng]
 * index_k, index_q, gate and q keep their full layouts; each call reads its groups' part.
 *
 * dsa_compress_regions_groups: dsa_compress_regions for groups g0..g0+ng-1 of index_k (row
 *   stride >= (g0+ng)*256) into the shard's pool.
 * dsa_decode_select_groups: dsa_decode_select for the shard; the workspace of
 *   dsa_decode_select_workspace_size(nq, ld_scores, k) bytes suffices.
 * dsa_sparse_attn_decode_groups: dsa_sparse_attn_decode for the shard; workspace
 *   dsa_attn_groups_workspace_size(nq, k, ng) bytes (0: none needed).
 * A group range outside these limits returns DSA_ERR_INVALID_ARG; all else as the 4-group
 * calls. */
dsa_status_t dsa_compress_regions_groups(const void *index_k, int64_t row_stride, int64_t n_rows,
                                         const int64_t *src_row, const int64_t *dst_slot, int n_regions,
                                         int g0, int ng, uint8_t *summaries, float *scales, int64_t n_slots,
                                         dsa_stream_t stream);
dsa_status_t dsa_decode_select_groups(const void *index_q, const float *gate, const int32_t *q_req,
                                      const int32_t *q_pos, int nq, int g0, int ng, const uint8_t *summaries,
                                      const float *scales, int64_t n_slots, const int64_t *sum_base,
                                      int n_req, float *scores, int64_t ld_scores, uint32_t flags, int k,
                                      int32_t *sel_idx, int32_t *sel_count, void *ws, size_t ws_bytes,
                                      dsa_stream_t stream);
size_t dsa_attn_groups_workspace_size(int nq, int k, int ng);
dsa_status_t dsa_sparse_attn_decode_groups(const void *q, const void *k_cache, const void *v_cache,
                                           int64_t n_pages, const int32_t *block_table, int max_pages,
                                           const int32_t *q_pos, int batch, int g0, int ng,
                                           const int32_t *sel_idx, const int32_t *sel_count, int k, void *out,
                                           float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* ------------------------------------------------------------------------------ */
/* Self-test of the failure detection (no counterpart in the pages).  Every mbarrier wait in
 * this library's kernels is bounded (2^31 SM cycles, about a second); a wait that runs out
 * sets the timeout bit of the per-device error word and lets its kernel return, so a stuck
 * pipeline becomes DSA_ERR_DEVICE from dsa_check_device() instead of a hung GPU.  This call
 * launches one small kernel whose barrier nothing ever completes, with the bound set to
 * limit_cycles (1 <= limit_cycles <= 2^31) for that kernel only: it returns after about that
 * many cycles and leaves the timeout bit set (dsa_check_device reports it and clears it).  The
 * kernel issues no copy or MMA and holds no tensor memory; other kernels keep their bound. */
dsa_status_t dsa_selftest_wait_timeout(int64_t limit_cycles, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
