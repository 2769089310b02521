// basiskv_decode_attn_noalloc: the sparse-attention call for callers that
// cannot allocate device memory.
//
// Some callers have no way to hand this library a workspace: a plugin whose
// enqueue hook runs inside a host engine that owns every device allocation,
// code that runs while a stream is being captured into a CUDA graph (where
// cudaMalloc is not allowed), or a deployment with a fixed memory budget
// that forbids allocation after start-up.  This entry point runs exactly the
// kernels of basiskv_decode_attn with a given selection (the union lists from
// it, then the attention kernel), but their scratch (the union lists, the
// per-group counters and tile cursors, the per-split partial results) lives in
// one file-scope __device__ array of fixed size that the library owns.  The
// caller still passes the inputs and the output.
//
// The array costs kNoAllocScratchBytes of memory on every GPU on which the
// library is loaded, until the process exits.
#include <stdio.h>

#include "kernels.cuh"

namespace bkv {

// Fixed scratch for basiskv_decode_attn_noalloc (16 MiB).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands for the symbol; the address the kernels need
// is looked up once per device, with that device current, in the context
// current then (the device's primary context for CUDA runtime callers).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_addr_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace bkv

using namespace bkv;

extern "C" BASISKV_API basiskv_status basiskv_decode_attn_noalloc(
    const basiskv_config* cfg, const basiskv_cache* cache, const void* q, int32_t batch,
    const int32_t* sel, const int32_t* sel_cnt, float* o_lat, int32_t* err_flag, void* stream) {
  // the checks of basiskv_decode_attn, in its order
  basiskv_status s = check_decode_attn(cfg, cache, q, batch, sel, sel_cnt, o_lat, err_flag);
  if (s != BASISKV_OK || batch == 0) return s;
  // there is no routing workspace whose union lists this call could read
  if (!sel) return BASISKV_ERR_INVALID_ARG;

  // the same scratch basiskv_decode_attn takes from its workspace
  const DecodePlan plan = plan_decode_attn(cfg, batch, cache->max_pages);
  if (plan.bytes > kNoAllocScratchBytes) {
    fprintf(stderr,
            "basiskv_decode_attn_noalloc: this shape needs %zu bytes of scratch, more than the "
            "fixed %zu; use basiskv_decode_attn with a workspace\n",
            plan.bytes, kNoAllocScratchBytes);
    return BASISKV_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    fprintf(stderr, "basiskv_decode_attn_noalloc: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
    return BASISKV_ERR_CUDA;
  }
  return run_decode_attn(plan, cfg, cache, q, batch, sel, sel_cnt, o_lat, static_cast<char*>(scratch), err_flag,
                         stream);
}
