// Shared device helpers for the BasisKV kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#include "basiskv.h"

namespace bkv {

constexpr int kWarp = 32;
constexpr unsigned kFull = 0xffffffffu;

// -------------------------------------------------------------------------
// element loads / stores
// -------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ double to_d(float x) { return (double)x; }
  static __device__ __forceinline__ float from_d(double x) { return __double2float_rn(x); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ double to_d(__nv_bfloat16 x) { return (double)__bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_d(double x) { return __double2bfloat16(x); }
};

// bf16 pair packed in a 32-bit word -> two floats (exact: bf16 is the top half of fp32)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Row swizzle of bf16 K and C pages for the tensor-core attention path: the
// 16-byte chunk c of page row j is stored at chunk c ^ (j & mask), which keeps
// 8 consecutive rows of one chunk column in 8 different bank groups.  mask is
// the largest of 7, 3, 1 that keeps every chunk inside its row.
__host__ __device__ __forceinline__ int swz_mask(int row_elems) {
  const int chunks = row_elems / 8;
  return (chunks % 8 == 0) ? 7 : (chunks % 4 == 0) ? 3 : (chunks % 2 == 0) ? 1 : 0;
}
__host__ __device__ __forceinline__ int swz(int x, int row, int mask) {
  return ((((x >> 3) ^ (row & mask)) << 3) | (x & 7));
}
// K and C pages are swizzled exactly when the tensor-core attention path runs
__host__ __device__ __forceinline__ bool kc_swizzled(bool bf16, int d, int r) {
  return bf16 && d % 16 == 0 && r % 16 == 0;
}

__device__ __forceinline__ void set_err(int32_t* flag, int32_t bits) {
  if (flag) atomicOr(flag, bits);
}

// -------------------------------------------------------------------------
// warp reductions
// -------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Sum N per-lane partial values over the 32 lanes, leaving each lane with
// the totals of the indices it owns.  Each butterfly stage halves the array:
// lanes with bit `o` set keep the upper half and receive the partner's upper
// half, the others keep the lower half.  For N <= 32 lane l ends with
// v[0] = total of index (l >> (5 - log2 N)); for N = 64 it holds the totals of
// indices 2l and 2l + 1 in v[0] and v[1].
template <int CUR, int O, int N>
struct TransposeReduce {
  static __device__ __forceinline__ void run(float (&v)[N], int lane) {
    if constexpr (O > 0) {
      constexpr int kKeep = (N > 32) ? N / 32 : 1;
      if constexpr (CUR > kKeep) {
        constexpr int H = CUR / 2;
        const bool upper = (lane & O) != 0;
#pragma unroll
        for (int j = 0; j < H; ++j) {
          const float send = upper ? v[j] : v[j + H];
          const float keep = upper ? v[j + H] : v[j];
          v[j] = keep + __shfl_xor_sync(kFull, send, O);
        }
        TransposeReduce<H, O / 2, N>::run(v, lane);
      } else {
#pragma unroll
        for (int j = 0; j < CUR; ++j) v[j] += __shfl_xor_sync(kFull, v[j], O);
        TransposeReduce<CUR, O / 2, N>::run(v, lane);
      }
    }
  }
};

template <int N>
__device__ __forceinline__ void transpose_reduce(float (&v)[N], int lane) {
  static_assert(N == 1 || N == 2 || N == 4 || N == 8 || N == 16 || N == 32 || N == 64,
                "transpose_reduce: N must be a power of two <= 64");
  TransposeReduce<N, 16, N>::run(v, lane);
}

// Exclusive scan of one int per thread over the block (blockDim.x a multiple of
// 32, at most 1024).  `warp_tot` is shared scratch of 32 ints; `total` gets the
// block sum.  Every thread of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = (lane < nw) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) warp_tot[lane] = t;  // inclusive totals
  }
  __syncthreads();
  const int before = (w > 0) ? warp_tot[w - 1] : 0;
  total = warp_tot[nw - 1];
  __syncthreads();  // warp_tot reused by the next scan
  return before + x - v;
}

// -------------------------------------------------------------------------
// mbarrier + bulk copy (TMA, 1-D) wrappers
// -------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`, giving up after ~`limit_cycles` SM clocks.
// Returns false on timeout (the caller records BASISKV_DEVERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  long long limit_cycles = 2000000000LL) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit_cycles) return false;
  }
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing on `bar` as transaction bytes; the data lands in this CTA only.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The same copy with an L2 eviction-priority hint (a policy from l2_evict_first()).
__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 policy for data read once: its lines are the first to be replaced, so
// data of normal priority (union lists, split partials, the out-projection
// factor where it fits) stays cached while such a stream passes through.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}


// Asynchronous 16-byte global -> shared copy (LDGSTS) that reads L2 only,
// tracked per thread with commit / wait groups; both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async16_cg(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// the same, writing zeros instead when !valid (nothing is read from src then)
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
// the same for one 4-byte word (both addresses 4-byte aligned)
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Order-preserving 32-bit key of a routing score: larger score, larger key;
// -0 == +0; NaN ranks below every other value (key 1).  Key 0 is kept for
// pages that do not compete.
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 1u;
  if (v == 0.f) v = 0.f;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Thread-block cluster helpers: this CTA's rank in its cluster; the cluster
// barrier split into arrive (release) and wait (acquire), executed by every
// thread of every CTA of the cluster; a load from another CTA's shared memory
// (ld_shared_cluster, below).
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The word at `local`'s offset in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t ld_shared_cluster(const uint32_t* local, uint32_t rank) {
  uint32_t remote, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}
__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }

// -------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the kernel before it on the stream is still
// running; it must execute grid_dep_wait() before it reads anything that
// kernel wrote.  A kernel calls allow_dependents() to let its dependent launch
// early.  Both instructions are no-ops when there is no such dependency.
// -------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }


// Raise a kernel's dynamic shared memory limit once per (device, kernel), so
// that later calls (including calls made while a stream is being captured
// into a CUDA graph) launch without touching function attributes.
inline cudaError_t ensure_smem(const void* func, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  auto key = std::make_pair(dev, func);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

}  // namespace bkv
