// Parameter blocks and launchers shared between the kernel files and api.cu.
#pragma once

#include "common.cuh"

namespace bkv {

struct AppendParams {
  const void* k_new;
  const void* v_new;
  const void* A;
  const void* P;
  const void* E;
  void* k_raw;
  void* c_lat;
  void* r_res;
  float* summary;
  const int32_t* block_table;
  const int32_t* seq_len;
  int32_t* err;
  int batch, n_new, Hkv, d, r, s, page, max_pages, num_phys;
};
cudaError_t launch_append(const AppendParams& p, bool bf16, cudaStream_t st);
// many tokens per sequence on the tensor cores (bf16 only), then the touched pages' summaries
bool prefill_tc_supported(bool bf16, int d, int r, int s);
cudaError_t launch_prefill_tc(const AppendParams& p, int num_sms, cudaStream_t st);

struct RouteParams {
  const void* q;
  const float* summary;
  const int32_t* block_table;
  const int32_t* seq_len;
  float* scores;    // [B][Hq][max_pages] per head; [B][Hkv][max_pages] per group
  int32_t* sel;     // [B][Hq][top_k + 2]
  int32_t* sel_cnt; // [B][Hq]
  int32_t* err;
  int batch, Hq, Hkv, page, max_pages, num_phys, top_k;
  int all_pages;    // 0: skip the sink and recent pages (always kept; their scores are not needed)
  int group_mode;   // 0: one selection per query head; 1 / 2: one per KV group from the
                    // sum / maximum of its heads' scores, copied to every head of the group
  // the union lists the selection kernel leaves for the attention kernel (union.cuh)
  uint32_t* lists;  // [B][Hkv][ustride]
  uint32_t* ucount; // [B][Hkv] entries of each list (compact)
  int32_t* ucnt;    // [B][Hkv] per-group arrival counters, zero between calls
  int32_t* acnt;    // [B][Hkv] the attention kernel's split counters, zeroed with the lists
  int ustride;
};
// beside_append: the score kernel is launched as a programmatic dependent of
// the kernel before it, which must be the decode-step append (basiskv_append_route)
cudaError_t launch_route(const RouteParams& p, int d, bool bf16, int num_sms, cudaStream_t st,
                         bool beside_append = false);

// Union lists from a given selection (sel / sel_cnt rows of every head).
struct UnionParams {
  const int32_t* sel;
  const int32_t* sel_cnt;
  const int32_t* block_table;
  const int32_t* seq_len;
  uint32_t* lists;
  uint32_t* ucount;  // [B][Hkv] entries of each list (compact)
  int32_t* acnt;  // [B][Hkv] the attention kernel's split counters, zeroed here for the
                  //   attention launch that reads the lists
  int32_t* err;
  int Hq, Hkv, page, max_pages, num_phys, top_k, ustride;
};
cudaError_t launch_union(const UnionParams& u, int batch, cudaStream_t st);

struct AttnParams {
  const void* q;
  const void* k_raw;
  const void* c_lat;
  const uint32_t* lists;   // [B][Hkv][ustride] union lists (union.cuh)
  const uint32_t* ucount;  // [B][Hkv] entries of each list
  int32_t* cnt;            // [B Hkv] finished-split counters, zeroed when the lists are written
  float* part;             // [grid][G][r + 2] partial results, one per CTA
  float* o_lat;            // [B][Hq][r]
  int32_t* err;
  int Hq, Hkv, page, r, num_phys, tpp, ngroups, extra, ustride, umax;
  float qscale;  // log2(e) / sqrt(d)
};

// Grid and scratch layout of one decode_attn call; depends on the shape only,
// so the workspace query and every launch agree on it.  Both attention
// kernels: every group gets one CTA, and the `extra` remaining CTAs of one
// resident wave are shared out at run time in proportion to the groups'
// tiles; one partial result per CTA.
struct DecodePlan {
  int umax;       // max union pages per (sequence, KV head)
  int tpp;        // 16-token tiles per page
  int grid;       // CTAs of the attention launch
  int extra;      // CUDA-core kernel: grid - groups
  int ustride;    // words per union list
  int ring_slots; // tensor-core kernel: bulk-copy slots per warp
  size_t list_off, ucount_off, cnt_off, part_off, bytes;
};
DecodePlan decode_plan(int Hq, int Hkv, int page, int r, int top_k, int batch, int max_pages, bool bf16, int d,
                       int num_sms);

struct DecodeArgs {
  const void* q;
  const void* k_raw;
  const void* c_lat;
  float* o_lat;
  int32_t* err;
  int Hq, Hkv, d, page, r, num_phys;
  bool bf16;
};
// The attention kernel over the union lists already in the plan's scratch.
cudaError_t launch_decode_attn(const DecodePlan& pl, const DecodeArgs& a, void* scratch, int batch,
                               cudaStream_t st);

// Host helpers of the C ABI (api.cu) shared with the allocation-free entry point.
int num_sms();
basiskv_status cuda_status(cudaError_t e);
basiskv_status check_decode_attn(const basiskv_config* cfg, const basiskv_cache* cache, const void* q, int32_t batch,
                                 const int32_t* sel, const int32_t* sel_cnt, const float* o_lat,
                                 const int32_t* err_flag);
DecodePlan plan_decode_attn(const basiskv_config* cfg, int32_t batch, int32_t max_pages);
basiskv_status run_decode_attn(const DecodePlan& plan, const basiskv_config* cfg, const basiskv_cache* cache,
                               const void* q, int32_t batch, const int32_t* sel, const int32_t* sel_cnt,
                               float* o_lat, char* scratch, int32_t* err_flag, void* stream);

struct OutProjParams {
  const float* o;
  const void* Gt;
  float* y;
  int batch, K, hidden;
};
cudaError_t launch_out_proj_gemv(const OutProjParams& p, bool bf16, cudaStream_t st);
// bf16 shapes with K % 64 == 0 and hidden % 128 == 0 keep Gt in the blocked
// tensor-core layout (see out_proj_tc.cu); every other shape uses [hidden][K].
bool gt_blocked(int K, int hidden);
// small batches (<= 8) with the pre-tiled Gt: mma.sync kernel without cluster or tensor memory
bool out_proj_mma_fits(int batch, int K, int hidden);
cudaError_t launch_out_proj_mma(const float* o, const void* Gt, float* y, int batch, int K, int hidden,
                                cudaStream_t st);
cudaError_t launch_out_proj_tc(const float* o, const void* Gt, float* y, int32_t* err, int batch, int K, int hidden,
                               int num_sms, cudaStream_t st);

// bytes from src to dst by the SMs (either side device memory or mapped host memory)
cudaError_t launch_copy(void* dst, const void* src, size_t bytes, int num_sms, cudaStream_t st);

struct FuseParams {
  const void* Bf;
  const void* W_O;
  void* Gt;
  int Hq, Hkv, d, r, hidden;
  int blocked;  // write the tensor-core tile layout instead of [hidden][K]
};
cudaError_t launch_fuse(const FuseParams& p, bool bf16, cudaStream_t st);

}  // namespace bkv
