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

struct ScoreParams {
  const void* q;
  const float* summary;
  const int32_t* block_table;
  const int32_t* seq_len;
  float* scores;
  int32_t* err;
  int batch, Hq, Hkv, page, max_pages, num_phys;
  int page_batches;
};
struct SelectParams {
  const float* scores;
  const int32_t* seq_len;
  int32_t* sel;
  int32_t* sel_cnt;
  int Hq, page, max_pages, top_k;
};
cudaError_t launch_route(const ScoreParams& sp, const SelectParams& selp, int d, int G, bool bf16,
                         int num_sms, cudaStream_t st);

struct UnionParams {
  const int32_t* sel;
  const int32_t* sel_cnt;
  const int32_t* seq_len;
  int32_t* uni;
  int32_t* ucnt;
  int32_t* err;
  int Hq, Hkv, page, max_pages, top_k, umax;
};
struct AttnParams {
  const void* q;
  const void* k_raw;
  const void* c_lat;
  const int32_t* block_table;
  const int32_t* seq_len;
  const int32_t* uni;
  const int32_t* ucnt;
  float* part;
  int32_t* err;
  int Hq, Hkv, page, r, max_pages, num_phys, umax, pps, nsplit;
  float qscale;
  int nstages;  // set by the launcher
};
struct CombineParams {
  const float* part;
  const int32_t* ucnt;
  float* o_lat;
  int Hq, Hkv, r, pps, nsplit;
};
int attn_pages_per_split(int page);
int attn_nsplit(int umax, int page);
cudaError_t launch_decode_attn(const UnionParams& up, const AttnParams& ap, const CombineParams& cp,
                               int batch, int d, bool bf16, cudaStream_t st);

struct OutProjParams {
  const float* o;
  const void* Gt;
  float* y;
  int batch, K, hidden;
};
cudaError_t launch_out_proj_gemv(const OutProjParams& p, bool bf16, cudaStream_t st);
bool out_proj_tc_supported(int K, int hidden, int batch);
cudaError_t launch_out_proj_tc(const float* o, const void* Gt, float* y, int32_t* err, int batch, int K, int hidden,
                               int num_sms, cudaStream_t st);

struct FuseParams {
  const void* Bf;
  const void* W_O;
  void* Gt;
  int Hq, Hkv, d, r, hidden;
};
cudaError_t launch_fuse(const FuseParams& p, bool bf16, cudaStream_t st);

}  // namespace bkv
