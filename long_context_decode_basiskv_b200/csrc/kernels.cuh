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
  const void* warm;   // optional: bytes to bring into L2 during a decode-step append (the fused factor)
  size_t warm_bytes;  // a multiple of 16
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
};
cudaError_t launch_route(const RouteParams& p, int d, bool bf16, int num_sms, cudaStream_t st);

struct AttnParams {
  const void* q;
  const void* k_raw;
  const void* c_lat;
  const int32_t* block_table;
  const int32_t* seq_len;
  const int32_t* sel;
  const int32_t* sel_cnt;
  int32_t* cnt;  // [B][Hkv] finished-split counters, zero between calls
  float* part;   // [B][Hq][nsplit][r + 2]
  float* o_lat;  // [B][Hq][r]
  int32_t* err;
  int Hq, Hkv, page, r, max_pages, num_phys, top_k, umax, tpp, eps, nsplit, nsplit_lo, rich_from;
  float qscale;  // log2(e) / sqrt(d)
};

// Tiles per split and scratch layout of one decode_attn call; depends on the
// shape only, so the workspace query and every launch agree on it.
struct DecodePlan {
  int umax;    // max union pages per (sequence, KV head)
  int tpp;     // 16-token tiles per page
  int eps;        // union pages per split, at most
  int nsplit;     // splits of the groups with the most (grid x extent; partial slots per head)
  int nsplit_lo;  // splits of groups b * Hkv + g < rich_from (nsplit or nsplit - 1)
  int rich_from;
  size_t cnt_off, part_off, bytes;
};
DecodePlan decode_plan(int Hq, int Hkv, int page, int r, int top_k, int batch, int max_pages, bool bf16, int d,
                       int num_sms);

struct DecodeArgs {
  const void* q;
  const void* k_raw;
  const void* c_lat;
  const int32_t* block_table;
  const int32_t* seq_len;
  const int32_t* sel;
  const int32_t* sel_cnt;
  float* o_lat;
  int32_t* err;
  int Hq, Hkv, d, page, r, max_pages, num_phys, top_k;
  bool bf16;
};
cudaError_t launch_decode_attn(const DecodePlan& pl, const DecodeArgs& a, void* scratch, int batch,
                               cudaStream_t st);

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

struct FuseParams {
  const void* Bf;
  const void* W_O;
  void* Gt;
  int Hq, Hkv, d, r, hidden;
  int blocked;  // write the tensor-core tile layout instead of [hidden][K]
};
cudaError_t launch_fuse(const FuseParams& p, bool bf16, cudaStream_t st);

}  // namespace bkv
