/*
 * basiskv.h — C ABI of the BasisKV decode hot path on NVIDIA B200 (sm_100a).
 *
 * One decode step of a batch of sequences is four calls on one CUDA stream:
 *
 *   basiskv_append       (step 1-2) store each new token's raw key, Value latent
 *                        and key residual in the paged cache; refresh the
 *                        summary (mean predicted key) of every page it touched
 *                        (basiskv_prefill: the same for long appends, on the
 *                        tensor cores)
 *   basiskv_route        (step 3)   score every page of every sequence for every
 *                        query head against the summaries; keep the top-k pages
 *                        plus the sink page and the recent page
 *                        (basiskv_route_group: one selection per KV group)
 *   basiskv_decode_attn  (step 4)   exact attention of each query head over the
 *                        original keys of its selected pages, accumulating the
 *                        Value latents (rank-r output per head)
 *   basiskv_out_proj     (step 5)   y = sum_h o_h G_h through the fused factor
 *
 * basiskv_append_route does steps 1-3 in one call, the route's scoring running
 * beside the append (no second stream needed).  A step whose inputs and output
 * live in page-locked host memory brings the inputs in with basiskv_copy and
 * lets basiskv_out_proj store y on the host.
 *
 * Method: "BasisKV: Value Latents for Communication and Key Routing"
 * (weekinpapers.com/paper/2611.02583v1, Abstract) and the kongchang.com
 * explainer of it (sections on binding the Value latent to the output
 * projection and "用Value潜变量辅助Key路由" on key routing); decode-step order
 * and attention formula: machinelearning.ru "KV-кэширование", sections
 * "Фаза Decode" and "Математическая формализация"; paged cache: same page,
 * section "Форматы хранения и библиотеки".
 *
 * Conventions for every entry point
 *   - Pointers marked (device) are CUDA device pointers owned by the caller;
 *     the library never allocates, frees or retains them.  Pointers marked
 *     (host) are read during the call only.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work and return; results are ready when the stream is.
 *   - Host-side validation failures return an error status and launch
 *     nothing.  No C++ exception crosses the ABI.
 *   - Faults the kernels can detect (a block-table entry or selected page out
 *     of range, a sequence length that cannot hold the new tokens, a wait that
 *     timed out) are OR-ed into *err_flag (device int32, bit values
 *     BASISKV_DEVERR_*) and the offending page or sequence is skipped; no
 *     kernel traps.  The caller zeroes the flag and reads it when it likes.
 *   - Tensor layouts are dense row-major in the order written.  `dtype` in
 *     basiskv_config fixes the element type of k_raw, c_lat, r_res, q, the
 *     new tokens and every factor (fp32 or bf16); summaries, o_lat, y and
 *     scores are always fp32.
 *   - Query head h uses KV head g(h) = h / (Hq / Hkv).
 */
#ifndef BASISKV_H
#define BASISKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BASISKV_API __attribute__((visibility("default")))
#else
#define BASISKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* 1: append, route, decode_attn, out_proj and their helpers;
 * 2: adds basiskv_route_group and basiskv_prefill;
 * 3: decode_attn accepts sel = sel_cnt = NULL (the routing call's selection). */
#define BASISKV_ABI_VERSION 4

typedef enum {
  BASISKV_OK = 0,
  BASISKV_ERR_INVALID_ARG = 1,   /* a NULL pointer, a negative size, an inconsistent shape */
  BASISKV_ERR_UNSUPPORTED = 2,   /* a valid shape this build has no kernel for            */
  BASISKV_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed                 */
  BASISKV_ERR_WORKSPACE = 4      /* workspace NULL or smaller than basiskv_workspace_bytes */
} basiskv_status;

typedef enum { BASISKV_F32 = 0, BASISKV_BF16 = 1 } basiskv_dtype;

/* How basiskv_route_group folds the scores of a KV group's query heads. */
typedef enum { BASISKV_GROUP_SUM = 1, BASISKV_GROUP_MAX = 2 } basiskv_group_reduce;

/* Bits OR-ed into *err_flag by the kernels. */
#define BASISKV_DEVERR_BLOCK_TABLE 1   /* block_table entry outside [0, num_phys_pages)      */
#define BASISKV_DEVERR_SELECTION 2     /* sel entry outside [0, pages of the sequence)       */
#define BASISKV_DEVERR_SEQ_LEN 4       /* seq_len < n_new, or > max_pages * page_size         */
#define BASISKV_DEVERR_TIMEOUT 8       /* an in-kernel wait on a bulk copy gave up (~1 s)     */
#define BASISKV_DEVERR_WORKSPACE 16    /* a workspace counter was not zero: not zero-filled   */

/*
 * Shapes.  Supported by this build: head_dim in {64, 128}; page_size in
 * {16, 32, 64}; 1 <= rank_v <= 128; 1 <= rank_k <= 64;
 * Hq / Hkv in {1, 2, 4, 8}; 1 <= top_k and top_k + 2 <= 1024;
 * hidden a multiple of 16.  Anything else returns BASISKV_ERR_UNSUPPORTED.
 */
typedef struct {
  int32_t num_q_heads;   /* Hq                                          */
  int32_t num_kv_heads;  /* Hkv (KV heads; Hq % Hkv == 0)                */
  int32_t head_dim;      /* d                                           */
  int32_t rank_v;        /* r: Value-latent rank                         */
  int32_t rank_k;        /* s: key-residual rank                         */
  int32_t page_size;     /* P: tokens per page                           */
  int32_t hidden;        /* width of the layer output y                  */
  int32_t top_k;         /* k: routed pages per head, sink/recent excluded */
  int32_t dtype;         /* basiskv_dtype                                */
} basiskv_config;

/*
 * Paged cache (device).  A physical page holds, for every KV head, one
 * contiguous block per tensor:
 *   k_raw   [num_phys_pages][Hkv][P][d]   original keys (dtype)
 *   c_lat   [num_phys_pages][Hkv][P][r]   Value latents C = v A_g (dtype)
 *   r_res   [num_phys_pages][Hkv][P][s]   key residuals R = (k - C P_g) E_g (dtype)
 *   summary [num_phys_pages][Hkv][d]      mean predicted key of the page (fp32)
 * block_table [B][max_pages] maps logical page p of sequence b to a physical
 * page; seq_len [B] is each sequence's token count AFTER the step's append.
 * Sequence b has n_b = ceil(seq_len[b] / P) pages; the recent page n_b - 1
 * may be partial and only its first seq_len[b] - (n_b - 1) P slots are valid.
 */
typedef struct {
  void* k_raw;
  void* c_lat;
  void* r_res;
  float* summary;
  const int32_t* block_table;
  const int32_t* seq_len;
  int32_t num_phys_pages;
  int32_t max_pages;
} basiskv_cache;

/*
 * Factors (device, dtype).  A [Hkv][d][r] (Value -> latent), P [Hkv][r][d]
 * (latent -> predicted key), E [Hkv][d][s] (key residual basis),
 * Gt: the fused out-projection factor G_h = B_g(h) W_O,h, hidden * Hq * r
 * elements written by basiskv_fuse_out_factor.  Element (c, k), output column
 * c and k = h * r + i, K = Hq * r, sits at
 *   - bf16 with K % 64 == 0 and hidden % 128 == 0 (the tensor-core layout):
 *     ((c/128 * K/64 + k/64) * 128 + c%128) * 64 + ((k%64/8) ^ (c%8)) * 8 + k%8,
 *     i.e. 128 x 64 tiles, each a contiguous 16 KB block whose 128-byte rows
 *     hold their 16-byte chunks in XOR-swizzled order;
 *   - every other shape: c * K + k (row-major [hidden][Hq][r]).
 */
typedef struct {
  const void* A;
  const void* P;
  const void* E;
  const void* Gt;
} basiskv_factors;

/*
 * Steps 1-2.  Append n_new tokens to each of `batch` sequences.
 * k_new, v_new (device, dtype): [batch][n_new][Hkv][d]; token t of sequence b
 * lands at position seq_len[b] - n_new + t (the pages it needs must already be
 * in block_table).  Per token and KV head g: C = v A_g, R = (k - C P_g) E_g
 * (R from the unrounded C), accumulated in fp64 and rounded once to dtype;
 * the raw key is stored as given.  Then every touched page's summary is
 * recomputed over its valid tokens: S = mean(C) P_g + mean(R) E_g^T, rounded
 * to fp32.  n_new = 1 is the decode step; larger n_new is prefill.
 * factors->Gt is not read (it may be NULL).  With n_new = 1 the kernel lets a
 * programmatic dependent launch at its start: a kernel launched after this
 * call with programmatic stream serialization must execute griddepcontrol.wait
 * before it reads anything the append writes (ordinary launches are unaffected).
 * err_flag (device int32) may not be NULL.
 */
BASISKV_API basiskv_status basiskv_append(const basiskv_config* cfg, const basiskv_cache* cache,
                              const basiskv_factors* factors, const void* k_new,
                              const void* v_new, int32_t batch, int32_t n_new,
                              int32_t* err_flag, void* stream);

/*
 * Steps 1-2 for long appends (prefill) on the tcgen05 tensor cores, bf16 only.
 * Same arguments, layouts, results and error reporting as basiskv_append, with
 * one difference in precision: the three chained products (C = v A_g,
 * k - C P_g, R = (k - C P_g) E_g) accumulate in fp32 in tensor memory, and
 * the fp32 intermediate that feeds the next product is passed as a bf16 pair
 * (hi + lo, ~16 mantissa bits), so a stored C or R value may differ by one
 * bf16 ulp from basiskv_append's correctly rounded fp64 result where the two
 * straddle a rounding midpoint.  The summaries of every touched page are then
 * recomputed in fp64 from the stored C and R, as basiskv_append does.
 * Requires head_dim 128, rank_v a multiple of 16 in [16, 128], rank_k a
 * multiple of 16 in [16, 64] (else BASISKV_ERR_UNSUPPORTED); k_new and v_new
 * 16-byte aligned.  Work is split in tiles of 128 consecutive new tokens per
 * (sequence, KV head), so short appends leave most of the GPU idle.
 */
BASISKV_API basiskv_status basiskv_prefill(const basiskv_config* cfg, const basiskv_cache* cache,
                               const basiskv_factors* factors, const void* k_new,
                               const void* v_new, int32_t batch, int32_t n_new,
                               int32_t* err_flag, void* stream);

/*
 * Step 3.  Page routing for every (sequence, query head).
 * q (device, dtype) [batch][Hq][d].  score_p = q_h . S_p in fp32 over every
 * logical page.  If n_b <= top_k + 2 every page is selected; otherwise pages
 * 0 and n_b - 1 plus the top_k of pages 1..n_b-2 under the order (score
 * descending, page index ascending).
 * A NaN score ranks below every other score (NaN pages are kept only when
 * fewer than top_k others exist, lowest page index first).
 * Outputs (device): sel [batch][Hq][top_k + 2] int32 logical page indices in
 * ascending order, padded with -1; sel_cnt [batch][Hq] int32.  The call also
 * leaves in the workspace, per (sequence, KV head), the ascending union of the
 * pages its G query heads selected (with their physical page ids), which a
 * following basiskv_decode_attn with sel = sel_cnt = NULL attends over.
 * scores (device, optional, may be NULL): [batch][Hq][max_pages] fp32, the
 * score of every page p < n_b (others untouched).
 * With scores == NULL the call reads no summary of page 0 or of page n_b - 1
 * (both are kept whatever they score), so it does not depend on
 * basiskv_append of the same step, which only rewrites the recent page: the
 * two may run concurrently on different streams.
 * workspace (device): at least basiskv_workspace_bytes(cfg, batch, max_pages)
 * bytes, zero-filled once when it is allocated.  It holds per-call scratch
 * plus small counters that every route call leaves at zero again, so no
 * further clearing is needed between calls of one shape (a counter found out
 * of range sets BASISKV_DEVERR_WORKSPACE).  The counters' place depends on the
 * shape: before a workspace serves another (cfg, batch, max_pages), zero-fill
 * it again.  Calls sharing one workspace must not overlap.  Requires
 * num_phys_pages < 2^24.
 */
BASISKV_API basiskv_status basiskv_route(const basiskv_config* cfg, const basiskv_cache* cache,
                             const void* q, int32_t batch, int32_t* sel, int32_t* sel_cnt,
                             float* scores, void* workspace, size_t workspace_bytes,
                             int32_t* err_flag, void* stream);

/*
 * Step 3, per-KV-group variant.  The pages say only that routing picks key
 * pages whose original keys are then read (kongchang.com explainer, section
 * "用Value潜变量辅助Key路由"); under grouped-query attention the G = Hq/Hkv
 * query heads of a group share one key head (cloud.baidu.com article
 * "大模型KV缓存压缩架构解析", section "1. 分组查询注意力（GQA）").  This
 * call routes once per (sequence, KV group g): the group score of page p is
 * the sum (reduce = BASISKV_GROUP_SUM) or the maximum (BASISKV_GROUP_MAX,
 * a NaN head score wins) over h = gG .. gG+G-1 of q_h . S_p in fp32, and the
 * selection rule of basiskv_route is applied to that one row.  The pages are
 * written to the sel / sel_cnt rows of all G heads of the group, in
 * basiskv_route's layout, so basiskv_decode_attn reads top_k + 2 pages per
 * group (instead of the union of G per-head selections).
 * scores (device, optional): [batch][Hkv][max_pages] fp32 group scores.
 * Other arguments, concurrency and workspace as for basiskv_route.  Any other
 * value of `reduce` is BASISKV_ERR_INVALID_ARG.
 */
BASISKV_API basiskv_status basiskv_route_group(const basiskv_config* cfg, const basiskv_cache* cache,
                                   const void* q, int32_t batch, int32_t reduce, int32_t* sel,
                                   int32_t* sel_cnt, float* scores, void* workspace,
                                   size_t workspace_bytes, int32_t* err_flag, void* stream);

/*
 * Steps 1-3 of one decode step in one call: basiskv_append with n_new = 1
 * (k_new, v_new as there), then basiskv_route (reduce = 0) or
 * basiskv_route_group (reduce = BASISKV_GROUP_SUM / BASISKV_GROUP_MAX) with
 * scores = NULL, on one stream.  Results are those of the two calls in that
 * order.  The route's scoring kernel is launched as a programmatic dependent of
 * the append kernel and runs beside it: without a scores output it reads no
 * page the append writes (the recent page is kept whatever it scores), and it
 * waits for the append before it completes, so everything after this call on
 * the stream sees both.  Saves the second stream and the join a caller would
 * otherwise use to overlap the two.  Arguments and errors as for the two calls
 * (an invalid `reduce` returns BASISKV_ERR_INVALID_ARG); validation happens
 * before either kernel is launched.
 */
BASISKV_API basiskv_status basiskv_append_route(const basiskv_config* cfg, const basiskv_cache* cache,
                                                const basiskv_factors* factors, const void* k_new,
                                                const void* v_new, const void* q, int32_t batch, int32_t reduce,
                                                int32_t* sel, int32_t* sel_cnt, void* workspace,
                                                size_t workspace_bytes, int32_t* err_flag, void* stream);

/*
 * Step 4.  Exact sparse attention.  For each (b, h): over the valid tokens j
 * of the pages in sel[b][h][0 .. sel_cnt-1], s_j = q_h . K_j / sqrt(d) on the
 * original keys, w = softmax(s), o_lat[b][h] = sum_j w_j C_j (fp32, [batch][Hq][r]).
 * Pages selected by several query heads of one KV head are read once.
 * sel / sel_cnt (device): any selection in basiskv_route's layout (each row a
 * duplicate-free list of pages of its sequence; a page outside the sequence
 * sets BASISKV_DEVERR_SELECTION and is skipped).  With sel and sel_cnt both
 * NULL the call attends over the selection the last basiskv_route or
 * basiskv_route_group call on the same workspace (same cfg, batch and
 * max_pages) stored there, without rebuilding it; giving only one of them is
 * BASISKV_ERR_INVALID_ARG.  workspace as for basiskv_route (the same buffer
 * may be passed to both).  err_flag may not be NULL.
 * The split of the work depends only on the union sizes, so repeated calls
 * on the same inputs give bitwise identical o_lat.
 */
BASISKV_API basiskv_status basiskv_decode_attn(const basiskv_config* cfg, const basiskv_cache* cache,
                                   const void* q, int32_t batch, const int32_t* sel,
                                   const int32_t* sel_cnt, float* o_lat, void* workspace,
                                   size_t workspace_bytes, int32_t* err_flag, void* stream);

/*
 * basiskv_decode_attn without a workspace.  This entry point has no
 * counterpart in the paper: it exists for callers that cannot allocate
 * device memory (a plugin whose host engine owns every allocation, code that
 * runs while its stream is captured into a CUDA graph, a fixed memory budget
 * after start-up).  It computes exactly what basiskv_decode_attn computes for
 * a given selection, with the same arguments minus the workspace, using a
 * scratch array of 16 MiB that the library keeps in device memory on every
 * GPU where it is loaded, for the life of the process.
 *   - Arguments are checked exactly as basiskv_decode_attn checks them, in the
 *     same order; sel and sel_cnt may not be NULL (there is no routing
 *     workspace to take a selection from).
 *   - Shapes whose scratch (union lists, counters, split partials) exceeds
 *     16 MiB return BASISKV_ERR_WORKSPACE (with a message on stderr) and
 *     launch nothing; use basiskv_decode_attn then.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) in the context current then (the device's
 *     primary context for CUDA runtime callers) and keeps it; make that first
 *     call before any stream capture.  Calling from another context on the
 *     same device, or after cudaDeviceReset, is not supported.
 *   - Every call on a device shares the one array, whatever its shape.  Calls
 *     that may overlap on the GPU (different streams without ordering) race
 *     and corrupt each other's results; order them.  Each call writes all the
 *     scratch it reads (its first kernel zeroes the counters the second one
 *     uses), so the array needs no clearing, also between calls of different
 *     shapes.
 */
BASISKV_API basiskv_status basiskv_decode_attn_noalloc(const basiskv_config* cfg,
                                                       const basiskv_cache* cache, const void* q,
                                                       int32_t batch, const int32_t* sel,
                                                       const int32_t* sel_cnt, float* o_lat,
                                                       int32_t* err_flag, void* stream);

/*
 * Step 5.  y[b] = sum_h o_lat[b][h] G_h (fp32 [batch][hidden]) with G read from
 * factors->Gt.  The full Value width is never formed.  workspace as above.
 * y may be device memory or page-locked host memory that the runtime has
 * mapped into the device's address space (cudaHostAlloc / cudaMallocHost, or
 * cudaHostRegister with mapping, under unified addressing): the kernel then
 * stores the result straight into host memory, readable once the stream has
 * been synchronised.  Any other y (pageable host memory) returns
 * BASISKV_ERR_INVALID_ARG and launches nothing.
 */
BASISKV_API basiskv_status basiskv_out_proj(const basiskv_config* cfg, const basiskv_factors* factors,
                                const float* o_lat, int32_t batch, float* y, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * Weight preparation for step 5 (not per step).  Gt(c, h r + i) =
 * sum_j Bf[g(h)][i][j] W_O[h d + j][c], accumulated in fp64 and rounded once to
 * dtype, stored in the layout described with basiskv_factors.  Bf (device,
 * dtype) [Hkv][r][d]; W_O (device, dtype) [Hq d][hidden]; Gt (device, dtype)
 * hidden * Hq * r elements.
 */
BASISKV_API basiskv_status basiskv_fuse_out_factor(const basiskv_config* cfg, const void* Bf,
                                       const void* W_O, void* Gt, void* stream);

/*
 * Copies `bytes` from src to dst on `stream` with a kernel (the SMs' own loads
 * and stores, no copy engine): either side may be device memory or page-locked
 * host memory mapped into the device's address space, as for basiskv_out_proj's
 * y.  Meant for a decode step's small inputs (q, k_new, v_new: about 100 KB),
 * where a copy-engine transfer captured in a CUDA graph costs several times the
 * bytes' wire time.  Both pointers 16-byte aligned, ranges not overlapping;
 * host memory that is not mapped, a NULL pointer with bytes > 0 or a
 * misaligned pointer returns BASISKV_ERR_INVALID_ARG and launches nothing.
 * Asynchronous: the caller keeps src unchanged and does not read dst until the
 * stream has passed the copy.  bytes = 0 does nothing.
 */
BASISKV_API basiskv_status basiskv_copy(void* dst, const void* src, size_t bytes, void* stream);

/* Workspace bytes needed by route / decode_attn / out_proj for this shape. */
BASISKV_API size_t basiskv_workspace_bytes(const basiskv_config* cfg, int32_t batch, int32_t max_pages);

/* Static description of a status code (never NULL). */
BASISKV_API const char* basiskv_status_string(int32_t status);

/* BASISKV_ABI_VERSION of the loaded library. */
BASISKV_API int32_t basiskv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BASISKV_H */
