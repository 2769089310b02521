// Step 3 of the BasisKV decode step: key-page routing.
//
// The compressed cache predicts which key pages matter (kongchang.com
// explainer, section "用Value潜变量辅助Key路由"; BasisKV abstract): every page
// keeps its mean predicted key S_p, each query head scores all pages with
// q_h . S_p and keeps the top-k, plus the sink page 0 and the recent page.
//
// Kernel 1 (score): streams the fp32 summaries once.  A warp takes 8 pages of
// one (sequence, KV head); each lane loads its d/32 dimensions of the 8
// summary rows (8 independent 16-byte loads in flight per lane), forms the
// partial dot products with all G query heads of the group, and one
// transpose-reduction leaves one (page, head) score per lane.  The summary of
// a page is read once for the whole GQA group.  HBM-bound.
//
// Kernel 2 (select): one CTA per (sequence, query head) runs an exact radix
// select (4 passes of 8 bits) on order-preserving integer keys of the fp32
// scores, then resolves ties at the threshold by ascending page index and
// compacts the kept pages in ascending order with two block scans.
#include "kernels.cuh"

namespace bkv {



constexpr int kScoreThreads = 256;
constexpr int kPagesPerWarp = 8;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kScoreThreads) route_score_kernel(ScoreParams p) {
  constexpr int DPL = D / 32;
  constexpr int N = kPagesPerWarp * G;
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x / 32);
  const int wid = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const long long items = (long long)p.batch * p.Hkv * p.page_batches;

  for (long long it = wid; it < items; it += warps_total) {
    const int pb = (int)(it % p.page_batches);
    const int bg = (int)(it / p.page_batches);
    const int g = bg % p.Hkv, b = bg / p.Hkv;
    const int L = p.seq_len[b];
    int n = (L + p.page - 1) / p.page;
    if (n > p.max_pages) {
      if (pb == 0 && lane == 0) set_err(p.err, BASISKV_DEVERR_SEQ_LEN);
      n = p.max_pages;
    }
    const int p0 = pb * kPagesPerWarp;
    if (p0 >= n) continue;

    float qf[G][DPL];
    const T* qb = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * D;
#pragma unroll
    for (int hi = 0; hi < G; ++hi)
#pragma unroll
      for (int u = 0; u < DPL; ++u) qf[hi][u] = Elem<T>::to_f(qb[hi * D + lane * DPL + u]);

    int my_phys = -1;
    if (lane < kPagesPerWarp && p0 + lane < n) {
      my_phys = p.block_table[(size_t)b * p.max_pages + p0 + lane];
      if (my_phys < 0 || my_phys >= p.num_phys) {
        set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
        my_phys = -2;
      }
    }
    float sv[kPagesPerWarp][DPL];
#pragma unroll
    for (int i = 0; i < kPagesPerWarp; ++i) {
      const int ph = __shfl_sync(kFull, my_phys, i);
      if (ph >= 0) {
        const float* row = p.summary + ((size_t)ph * p.Hkv + g) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(row));
          sv[i][0] = v.x; sv[i][1] = v.y; sv[i][2] = v.z; sv[i][3] = v.w;
        } else {
          const float2 v = __ldg(reinterpret_cast<const float2*>(row));
          sv[i][0] = v.x; sv[i][1] = v.y;
        }
      } else {
#pragma unroll
        for (int u = 0; u < DPL; ++u) sv[i][u] = 0.f;
      }
    }
    float part[N];
#pragma unroll
    for (int i = 0; i < kPagesPerWarp; ++i)
#pragma unroll
      for (int hi = 0; hi < G; ++hi) {
        float a = 0.f;
#pragma unroll
        for (int u = 0; u < DPL; ++u) a = fmaf(qf[hi][u], sv[i][u], a);
        part[i * G + hi] = a;
      }
    transpose_reduce<N>(part, lane);

    float* out = p.scores + ((size_t)b * p.Hq + (size_t)g * G) * p.max_pages + p0;
    if constexpr (N <= 32) {
      constexpr int kDup = 32 / N;
      const int idx = lane / kDup;
      const int i = idx / G, hi = idx % G;
      const int ph = __shfl_sync(kFull, my_phys, i);
      if ((lane % kDup) == 0 && p0 + i < n)
        out[(size_t)hi * p.max_pages + i] = (ph == -2) ? -INFINITY : part[0];
    } else {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = 2 * lane + j;
        const int i = idx / G, hi = idx % G;
        const int ph = __shfl_sync(kFull, my_phys, i);
        if (p0 + i < n) out[(size_t)hi * p.max_pages + i] = (ph == -2) ? -INFINITY : part[j];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// selection
// ---------------------------------------------------------------------------


constexpr int kSelectThreads = 256;

// order-preserving map fp32 -> uint32 (larger score -> larger key); -0 == +0
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x == 0.f) x = 0.f;
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kSelectThreads) route_select_kernel(SelectParams p) {
  extern __shared__ __align__(16) uint32_t keys[];  // [max_pages]
  __shared__ int hist[256];
  __shared__ int warp_tot[32];
  __shared__ uint32_t s_digit;
  __shared__ int s_above;

  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31;
  const int L = p.seq_len[b];
  const int n = max(1, min((L + p.page - 1) / p.page, p.max_pages));
  const int kk = p.top_k;
  const size_t row = (size_t)b * p.Hq + h;
  int32_t* out = p.sel + row * (kk + 2);
  const float* sc = p.scores + row * p.max_pages;

  if (n <= kk + 2) {
    for (int i = tid; i < kk + 2; i += blockDim.x) out[i] = (i < n) ? i : -1;
    if (tid == 0) p.sel_cnt[row] = n;
    return;
  }

  const int ncand = n - 2;  // pages 1 .. n-2
  for (int i = tid; i < ncand; i += blockDim.x) keys[1 + i] = order_key(sc[1 + i]);
  __syncthreads();

  uint32_t prefix = 0, pmask = 0;
  int rem = kk;  // how many of the matching keys are still to be taken
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < ncand; base += blockDim.x) {
      const int i = base + tid;
      uint32_t digit = 0xffffffffu;
      if (i < ncand) {
        const uint32_t key = keys[1 + i];
        if ((key & pmask) == prefix) digit = (key >> shift) & 0xffu;
      }
      const unsigned same = __match_any_sync(kFull, digit);
      if (digit != 0xffffffffu && lane == __ffs(same) - 1) atomicAdd(&hist[digit], __popc(same));
    }
    __syncthreads();
    if (tid < 32) {
      // lane owns digits 8*lane .. 8*lane+7; count of matching keys above each digit
      int loc[8];
      int sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        loc[j] = hist[8 * tid + j];
        sum += loc[j];
      }
      int above = 0;  // sum over lanes with higher digits
      int x = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(kFull, x, o);
        if (tid + o < 32) x += y;
      }
      above = x - sum;  // inclusive suffix minus own
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (above < rem && rem <= above + loc[j]) {
          s_digit = (uint32_t)(8 * tid + j);
          s_above = above;
        }
        above += loc[j];
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    pmask |= 0xffu << shift;
    rem -= s_above;
    __syncthreads();
  }
  const uint32_t thr = prefix;  // key of the k-th largest candidate
  // rem = how many candidates equal to thr are kept (lowest page index first)

  // pass A: rank of each equal-to-threshold candidate in page order
  const int per = (n + kSelectThreads - 1) / kSelectThreads;
  const int lo = tid * per, hi = min(n, lo + per);
  int eq_local = 0;
  for (int pg = lo; pg < hi; ++pg)
    if (pg >= 1 && pg <= n - 2 && keys[pg] == thr) ++eq_local;
  int tot;
  int eq_rank = block_exclusive_scan(eq_local, warp_tot, tot);
  // pass B: keep flags and their count
  int take_local = 0;
  {
    int er = eq_rank;
    for (int pg = lo; pg < hi; ++pg) {
      bool take;
      if (pg == 0 || pg == n - 1) {
        take = true;
      } else {
        const uint32_t key = keys[pg];
        take = key > thr || (key == thr && er < rem);
        if (key == thr) ++er;
      }
      take_local += take ? 1 : 0;
    }
  }
  int pos = block_exclusive_scan(take_local, warp_tot, tot);
  {
    int er = eq_rank;
    for (int pg = lo; pg < hi; ++pg) {
      bool take;
      if (pg == 0 || pg == n - 1) {
        take = true;
      } else {
        const uint32_t key = keys[pg];
        take = key > thr || (key == thr && er < rem);
        if (key == thr) ++er;
      }
      if (take) out[pos++] = pg;
    }
  }
  for (int i = tot + tid; i < kk + 2; i += blockDim.x) out[i] = -1;
  if (tid == 0) p.sel_cnt[row] = tot;
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
template <typename T, int D>
static cudaError_t launch_score_g(const ScoreParams& p, int G, int grid, cudaStream_t st) {
  switch (G) {
    case 1: route_score_kernel<T, D, 1><<<grid, kScoreThreads, 0, st>>>(p); break;
    case 2: route_score_kernel<T, D, 2><<<grid, kScoreThreads, 0, st>>>(p); break;
    case 4: route_score_kernel<T, D, 4><<<grid, kScoreThreads, 0, st>>>(p); break;
    case 8: route_score_kernel<T, D, 8><<<grid, kScoreThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_route(const ScoreParams& sp, const SelectParams& selp, int d, int G, bool bf16,
                         int num_sms, cudaStream_t st) {
  const long long items = (long long)sp.batch * sp.Hkv * sp.page_batches;
  const long long warps = (items + 0);
  long long blocks = (warps + (kScoreThreads / 32) - 1) / (kScoreThreads / 32);
  const long long cap = (long long)num_sms * (2048 / kScoreThreads);
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaError_t e;
  if (bf16) {
    e = (d == 128) ? launch_score_g<__nv_bfloat16, 128>(sp, G, (int)blocks, st)
                   : launch_score_g<__nv_bfloat16, 64>(sp, G, (int)blocks, st);
  } else {
    e = (d == 128) ? launch_score_g<float, 128>(sp, G, (int)blocks, st)
                   : launch_score_g<float, 64>(sp, G, (int)blocks, st);
  }
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)sp.max_pages * sizeof(uint32_t);
  e = ensure_smem((const void*)route_select_kernel, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(sp.Hq, sp.batch);
  route_select_kernel<<<grid, kSelectThreads, smem, st>>>(selp);
  return cudaGetLastError();
}

}  // namespace bkv
