// C ABI entry points (include/basiskv.h): host-side validation, workspace
// layout and kernel dispatch.  Nothing here allocates device memory.
#include <stdio.h>

#include "kernels.cuh"
#include "union.cuh"

namespace bkv {

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------
constexpr int kMaxPagesLimit = 49152;  // route select keeps one key per page in shared memory

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int esize(const basiskv_config* c) { return c->dtype == BASISKV_BF16 ? 2 : 4; }

static basiskv_status check_config(const basiskv_config* c) {
  if (!c) return BASISKV_ERR_INVALID_ARG;
  if (c->num_q_heads <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0 || c->rank_v <= 0 ||
      c->rank_k <= 0 || c->page_size <= 0 || c->hidden <= 0 || c->top_k <= 0)
    return BASISKV_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads != 0) return BASISKV_ERR_INVALID_ARG;
  if (c->dtype != BASISKV_F32 && c->dtype != BASISKV_BF16) return BASISKV_ERR_INVALID_ARG;
  if (c->rank_v > c->head_dim || c->rank_k > c->head_dim) return BASISKV_ERR_INVALID_ARG;
  const int G = c->num_q_heads / c->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return BASISKV_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return BASISKV_ERR_UNSUPPORTED;
  if (c->page_size != 16 && c->page_size != 32 && c->page_size != 64) return BASISKV_ERR_UNSUPPORTED;
  if (c->rank_v > 128 || c->rank_k > 64) return BASISKV_ERR_UNSUPPORTED;
  if (c->top_k + 2 > 1024) return BASISKV_ERR_UNSUPPORTED;
  if (c->hidden % 16 != 0) return BASISKV_ERR_UNSUPPORTED;
  if (((size_t)c->num_q_heads * c->rank_v * esize(c)) % 16 != 0) return BASISKV_ERR_UNSUPPORTED;
  return BASISKV_OK;
}

static basiskv_status check_cache(const basiskv_config* c, const basiskv_cache* k, bool need_res,
                                  bool need_summary = true) {
  if (!k || !k->k_raw || !k->c_lat || !k->block_table || !k->seq_len) return BASISKV_ERR_INVALID_ARG;
  if (need_summary && !k->summary) return BASISKV_ERR_INVALID_ARG;
  if (need_res && !k->r_res) return BASISKV_ERR_INVALID_ARG;
  if (k->num_phys_pages <= 0 || k->max_pages <= 0) return BASISKV_ERR_INVALID_ARG;
  if (k->max_pages > kMaxPagesLimit || k->num_phys_pages > kMaxPhysPages) return BASISKV_ERR_UNSUPPORTED;
  if (!aligned16(k->k_raw) || !aligned16(k->c_lat) || (need_summary && !aligned16(k->summary)) ||
      (need_res && !aligned16(k->r_res)))
    return BASISKV_ERR_INVALID_ARG;
  (void)c;
  return BASISKV_OK;
}

// The address under which kernels reach `p`: p itself for device or managed
// memory, the mapping of page-locked host memory allocated or registered with
// the runtime; NULL for anything else (pageable host memory, unknown pointers).
static void* device_view(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();  // the error is not sticky: clear it so a later check does not see it
    return nullptr;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return const_cast<void*>(p);
  if (a.type == cudaMemoryTypeHost) return a.devicePointer;
  return nullptr;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Workspace: routing scores, the routing arrival counters, then the decode
// scratch of decode_plan() (union lists, counters, tile cursors, split results).
struct Workspace {
  size_t scores, rcnt, decode, total;
  DecodePlan plan;
};

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

static Workspace layout(const basiskv_config* c, int batch, int max_pages) {
  Workspace w{};
  w.plan = decode_plan(c->num_q_heads, c->num_kv_heads, c->page_size, c->rank_v, c->top_k, batch, max_pages,
                       c->dtype == BASISKV_BF16, c->head_dim, num_sms());
  w.scores = 0;
  w.rcnt = up256((size_t)batch * c->num_q_heads * max_pages * 4);
  w.decode = w.rcnt + up256((size_t)batch * c->num_kv_heads * 4);
  w.total = w.decode + w.plan.bytes;
  return w;
}

basiskv_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BASISKV_OK;
  fprintf(stderr, "basiskv: CUDA error %s\n", cudaGetErrorString(e));
  return BASISKV_ERR_CUDA;
}

// Validation shared by basiskv_decode_attn and basiskv_decode_attn_noalloc
// (sel and sel_cnt are both given, or both NULL).
basiskv_status check_decode_attn(const basiskv_config* cfg, const basiskv_cache* cache, const void* q, int32_t batch,
                                 const int32_t* sel, const int32_t* sel_cnt, const float* o_lat,
                                 const int32_t* err_flag) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if ((s = check_cache(cfg, cache, false, false)) != BASISKV_OK) return s;
  if (batch < 0) return BASISKV_ERR_INVALID_ARG;
  if (batch == 0) return BASISKV_OK;
  if (!q || !o_lat || !err_flag || (!sel) != (!sel_cnt)) return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(q)) return BASISKV_ERR_INVALID_ARG;
  return BASISKV_OK;
}

DecodePlan plan_decode_attn(const basiskv_config* cfg, int32_t batch, int32_t max_pages) {
  return decode_plan(cfg->num_q_heads, cfg->num_kv_heads, cfg->page_size, cfg->rank_v, cfg->top_k, batch, max_pages,
                     cfg->dtype == BASISKV_BF16, cfg->head_dim, num_sms());
}

// Union lists from sel (when given), then the attention kernel, into `scratch`
// laid out by `plan`.
basiskv_status run_decode_attn(const DecodePlan& plan, const basiskv_config* cfg, const basiskv_cache* cache,
                               const void* q, int32_t batch, const int32_t* sel, const int32_t* sel_cnt,
                               float* o_lat, char* scratch, int32_t* err_flag, void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  if (sel) {
    const UnionParams u{sel, sel_cnt, cache->block_table, cache->seq_len,
                        reinterpret_cast<uint32_t*>(scratch + plan.list_off),
                        reinterpret_cast<uint32_t*>(scratch + plan.ucount_off),
                        reinterpret_cast<int32_t*>(scratch + plan.cnt_off), err_flag, cfg->num_q_heads,
                        cfg->num_kv_heads, cfg->page_size, cache->max_pages, cache->num_phys_pages, cfg->top_k,
                        plan.ustride};
    cudaError_t e = launch_union(u, batch, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  DecodeArgs a{q, cache->k_raw, cache->c_lat, o_lat, err_flag, cfg->num_q_heads, cfg->num_kv_heads, cfg->head_dim,
               cfg->page_size, cfg->rank_v, cache->num_phys_pages, cfg->dtype == BASISKV_BF16};
  return cuda_status(launch_decode_attn(plan, a, scratch, batch, st));
}

}  // namespace bkv

using namespace bkv;

extern "C" {

int32_t basiskv_abi_version(void) { return BASISKV_ABI_VERSION; }

const char* basiskv_status_string(int32_t s) {
  switch (s) {
    case BASISKV_OK: return "ok";
    case BASISKV_ERR_INVALID_ARG: return "invalid argument";
    case BASISKV_ERR_UNSUPPORTED: return "unsupported shape";
    case BASISKV_ERR_CUDA: return "CUDA error";
    case BASISKV_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

size_t basiskv_workspace_bytes(const basiskv_config* cfg, int32_t batch, int32_t max_pages) {
  if (check_config(cfg) != BASISKV_OK || batch < 0 || max_pages <= 0) return 0;
  return layout(cfg, batch, max_pages).total;
}

basiskv_status basiskv_append(const basiskv_config* cfg, const basiskv_cache* cache,
                              const basiskv_factors* f, const void* k_new, const void* v_new,
                              int32_t batch, int32_t n_new, int32_t* err_flag, void* stream) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != BASISKV_OK) return s;
  if (batch == 0 || n_new == 0) return BASISKV_OK;
  if (!f || !f->A || !f->P || !f->E || !k_new || !v_new || !err_flag || batch < 0 || n_new < 0)
    return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(f->A) || !aligned16(f->P) || !aligned16(f->E)) return BASISKV_ERR_INVALID_ARG;
  if ((long long)n_new > (long long)cache->max_pages * cfg->page_size) return BASISKV_ERR_INVALID_ARG;
  const AppendParams p{k_new, v_new, f->A, f->P, f->E, cache->k_raw, cache->c_lat, cache->r_res,
                       cache->summary, cache->block_table, cache->seq_len, err_flag,
                       batch, n_new, cfg->num_kv_heads, cfg->head_dim, cfg->rank_v, cfg->rank_k,
                       cfg->page_size, cache->max_pages, cache->num_phys_pages};
  return cuda_status(launch_append(p, cfg->dtype == BASISKV_BF16, (cudaStream_t)stream));
}

basiskv_status basiskv_prefill(const basiskv_config* cfg, const basiskv_cache* cache,
                               const basiskv_factors* f, const void* k_new, const void* v_new,
                               int32_t batch, int32_t n_new, int32_t* err_flag, void* stream) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != BASISKV_OK) return s;
  if (!prefill_tc_supported(cfg->dtype == BASISKV_BF16, cfg->head_dim, cfg->rank_v, cfg->rank_k))
    return BASISKV_ERR_UNSUPPORTED;
  if (batch == 0 || n_new == 0) return BASISKV_OK;
  if (!f || !f->A || !f->P || !f->E || !k_new || !v_new || !err_flag || batch < 0 || n_new < 0)
    return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(f->A) || !aligned16(f->P) || !aligned16(f->E) || !aligned16(k_new) || !aligned16(v_new))
    return BASISKV_ERR_INVALID_ARG;
  if ((long long)n_new > (long long)cache->max_pages * cfg->page_size) return BASISKV_ERR_INVALID_ARG;
  const AppendParams p{k_new, v_new, f->A, f->P, f->E, cache->k_raw, cache->c_lat, cache->r_res,
                       cache->summary, cache->block_table, cache->seq_len, err_flag,
                       batch, n_new, cfg->num_kv_heads, cfg->head_dim, cfg->rank_v, cfg->rank_k,
                       cfg->page_size, cache->max_pages, cache->num_phys_pages};
  return cuda_status(launch_prefill_tc(p, num_sms(), (cudaStream_t)stream));
}

static basiskv_status route_common(const basiskv_config* cfg, const basiskv_cache* cache, const void* q,
                                   int32_t batch, int group_mode, int32_t* sel, int32_t* sel_cnt, float* scores,
                                   void* ws, size_t ws_bytes, int32_t* err_flag, void* stream,
                                   const AppendParams* append_first = nullptr) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if ((s = check_cache(cfg, cache, false)) != BASISKV_OK) return s;
  if (batch == 0) return BASISKV_OK;
  if (!q || !sel || !sel_cnt || !err_flag || batch < 0) return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(q) || (scores && !aligned16(scores))) return BASISKV_ERR_INVALID_ARG;
  const Workspace w = layout(cfg, batch, cache->max_pages);
  if (!ws || ws_bytes < w.total || !aligned16(ws)) return BASISKV_ERR_WORKSPACE;
  char* wsb = static_cast<char*>(ws);
  float* sc = scores ? scores : reinterpret_cast<float*>(wsb + w.scores);
  uint32_t* lists = reinterpret_cast<uint32_t*>(wsb + w.decode + w.plan.list_off);
  int32_t* acnt = reinterpret_cast<int32_t*>(wsb + w.decode + w.plan.cnt_off);
  RouteParams rp{q, cache->summary, cache->block_table, cache->seq_len, sc, sel, sel_cnt, err_flag,
                 batch, cfg->num_q_heads, cfg->num_kv_heads, cfg->page_size, cache->max_pages,
                 cache->num_phys_pages, cfg->top_k, scores ? 1 : 0, group_mode,
                 lists, reinterpret_cast<uint32_t*>(wsb + w.decode + w.plan.ucount_off),
                 reinterpret_cast<int32_t*>(wsb + w.rcnt), acnt, w.plan.ustride};
  if (append_first) {
    // the append, then the scoring as its programmatic dependent (it reads none of the append's pages)
    const cudaError_t e = launch_append(*append_first, cfg->dtype == BASISKV_BF16, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return cuda_status(launch_route(rp, cfg->head_dim, cfg->dtype == BASISKV_BF16, num_sms(), (cudaStream_t)stream,
                                  append_first != nullptr));
}

basiskv_status basiskv_route(const basiskv_config* cfg, const basiskv_cache* cache, const void* q,
                             int32_t batch, int32_t* sel, int32_t* sel_cnt, float* scores,
                             void* ws, size_t ws_bytes, int32_t* err_flag, void* stream) {
  return route_common(cfg, cache, q, batch, 0, sel, sel_cnt, scores, ws, ws_bytes, err_flag, stream);
}

basiskv_status basiskv_route_group(const basiskv_config* cfg, const basiskv_cache* cache, const void* q,
                                   int32_t batch, int32_t reduce, int32_t* sel, int32_t* sel_cnt,
                                   float* scores, void* ws, size_t ws_bytes, int32_t* err_flag, void* stream) {
  if (reduce != BASISKV_GROUP_SUM && reduce != BASISKV_GROUP_MAX) return BASISKV_ERR_INVALID_ARG;
  return route_common(cfg, cache, q, batch, reduce, sel, sel_cnt, scores, ws, ws_bytes, err_flag, stream);
}

basiskv_status basiskv_append_route(const basiskv_config* cfg, const basiskv_cache* cache,
                                    const basiskv_factors* f, const void* k_new, const void* v_new, const void* q,
                                    int32_t batch, int32_t reduce, int32_t* sel, int32_t* sel_cnt, void* ws,
                                    size_t ws_bytes, int32_t* err_flag, void* stream) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if ((s = check_cache(cfg, cache, true)) != BASISKV_OK) return s;
  if (reduce != 0 && reduce != BASISKV_GROUP_SUM && reduce != BASISKV_GROUP_MAX) return BASISKV_ERR_INVALID_ARG;
  if (batch == 0) return BASISKV_OK;
  if (!f || !f->A || !f->P || !f->E || !k_new || !v_new || !err_flag || batch < 0) return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(f->A) || !aligned16(f->P) || !aligned16(f->E)) return BASISKV_ERR_INVALID_ARG;
  const AppendParams ap{k_new, v_new, f->A, f->P, f->E, cache->k_raw, cache->c_lat, cache->r_res,
                        cache->summary, cache->block_table, cache->seq_len, err_flag,
                        batch, 1, cfg->num_kv_heads, cfg->head_dim, cfg->rank_v, cfg->rank_k,
                        cfg->page_size, cache->max_pages, cache->num_phys_pages};
  return route_common(cfg, cache, q, batch, reduce, sel, sel_cnt, nullptr, ws, ws_bytes, err_flag, stream, &ap);
}

basiskv_status basiskv_decode_attn(const basiskv_config* cfg, const basiskv_cache* cache,
                                   const void* q, int32_t batch, const int32_t* sel,
                                   const int32_t* sel_cnt, float* o_lat, void* ws, size_t ws_bytes,
                                   int32_t* err_flag, void* stream) {
  basiskv_status s = check_decode_attn(cfg, cache, q, batch, sel, sel_cnt, o_lat, err_flag);
  if (s != BASISKV_OK || batch == 0) return s;
  const Workspace w = layout(cfg, batch, cache->max_pages);
  if (!ws || ws_bytes < w.total || !aligned16(ws)) return BASISKV_ERR_WORKSPACE;
  return run_decode_attn(w.plan, cfg, cache, q, batch, sel, sel_cnt, o_lat, static_cast<char*>(ws) + w.decode,
                         err_flag, stream);
}

basiskv_status basiskv_out_proj(const basiskv_config* cfg, const basiskv_factors* f, const float* o_lat,
                                int32_t batch, float* y, void* ws, size_t ws_bytes, void* stream) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if (batch == 0) return BASISKV_OK;
  if (!f || !f->Gt || !o_lat || !y || batch < 0) return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(f->Gt) || !aligned16(o_lat) || !aligned16(y)) return BASISKV_ERR_INVALID_ARG;
  y = static_cast<float*>(device_view(y));  // device memory, or page-locked host memory the kernel writes
  if (!y || !aligned16(y)) return BASISKV_ERR_INVALID_ARG;
  (void)ws;
  (void)ws_bytes;
  const int K = cfg->num_q_heads * cfg->rank_v;
  if (cfg->dtype == BASISKV_BF16 && out_proj_mma_fits(batch, K, cfg->hidden))
    return cuda_status(launch_out_proj_mma(o_lat, f->Gt, y, batch, K, cfg->hidden, (cudaStream_t)stream));
  if (cfg->dtype == BASISKV_BF16 && gt_blocked(K, cfg->hidden))
    return cuda_status(launch_out_proj_tc(o_lat, f->Gt, y, nullptr, batch, K, cfg->hidden, num_sms(),
                                          (cudaStream_t)stream));
  OutProjParams p{o_lat, f->Gt, y, batch, K, cfg->hidden};
  return cuda_status(launch_out_proj_gemv(p, cfg->dtype == BASISKV_BF16, (cudaStream_t)stream));
}

basiskv_status basiskv_copy(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return BASISKV_OK;
  if (!dst || !src) return BASISKV_ERR_INVALID_ARG;
  if (!aligned16(dst) || !aligned16(src)) return BASISKV_ERR_INVALID_ARG;
  void* d = device_view(dst);
  const void* s = device_view(src);
  if (!d || !s || !aligned16(d) || !aligned16(s)) return BASISKV_ERR_INVALID_ARG;
  const uintptr_t a = reinterpret_cast<uintptr_t>(d), b = reinterpret_cast<uintptr_t>(s);
  if (a < b + bytes && b < a + bytes) return BASISKV_ERR_INVALID_ARG;  // overlapping ranges
  return cuda_status(launch_copy(d, s, bytes, num_sms(), (cudaStream_t)stream));
}

basiskv_status basiskv_fuse_out_factor(const basiskv_config* cfg, const void* Bf, const void* W_O,
                                       void* Gt, void* stream) {
  basiskv_status s = check_config(cfg);
  if (s != BASISKV_OK) return s;
  if (!Bf || !W_O || !Gt) return BASISKV_ERR_INVALID_ARG;
  const bool blocked = cfg->dtype == BASISKV_BF16 && gt_blocked(cfg->num_q_heads * cfg->rank_v, cfg->hidden);
  FuseParams p{Bf, W_O, Gt, cfg->num_q_heads, cfg->num_kv_heads, cfg->head_dim, cfg->rank_v, cfg->hidden,
               blocked ? 1 : 0};
  return cuda_status(launch_fuse(p, cfg->dtype == BASISKV_BF16, (cudaStream_t)stream));
}

}  // extern "C"
