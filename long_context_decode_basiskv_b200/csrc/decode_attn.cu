// Step 4 of the BasisKV decode step: exact attention on the routed pages.
//
// Only the selected key pages are read back, and the QK scores on them are
// exact (BasisKV abstract; kongchang.com explainer, section
// "用Value潜变量辅助Key路由"); the attention formula is the textbook one
// (machinelearning.ru "KV-кэширование", section "Математическая формализация"),
// restricted to the selected tokens, with the weights applied to the rank-r
// Value latents instead of full-width values.
//
// Three launches:
//  union    one CTA per (sequence, KV head): merges the G query heads'
//           selections into one ascending page list with a G-bit head mask
//           per page, so a page chosen by several heads of a group is read once.
//  attn     one CTA per (sequence, KV head, split of the union).  Each of its
//           warps streams its own 16-token tiles (raw K rows and C rows,
//           contiguous in the page block) through a private ring of shared
//           memory stages filled by 1-D bulk copies (cp.async.bulk, mbarrier
//           completion, no multicast).  Per tile and per head in the mask it
//           forms 16 exact scores, updates an online softmax (running max and
//           sum, base 2) and accumulates p * C.  Warps then merge in shared
//           memory and the CTA writes one partial (max, sum, acc[r]) per head.
//  combine  one CTA per (sequence, query head): log-sum-exp merge of the splits.
// HBM-bound: every byte of the union's pages is read once.
#include "kernels.cuh"

namespace bkv {

constexpr int kTile = 16;          // tokens per tile
constexpr int kAttnWarps = 4;      // warps per CTA
constexpr int kMaxStages = 4;      // ring depth per warp (fewer when shared memory is short)
constexpr int kTilesPerSplit = 32; // tiles of union pages handled by one CTA

// ---------------------------------------------------------------------------
// union of the group's selections
// ---------------------------------------------------------------------------


__global__ void __launch_bounds__(256) union_kernel(UnionParams p) {
  extern __shared__ __align__(16) uint32_t words[];  // [ceil(max_pages / 4)] byte masks
  __shared__ int warp_tot[32];
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int G = p.Hq / p.Hkv;
  const int L = p.seq_len[b];
  const int n = min((L + p.page - 1) / p.page, p.max_pages);
  const int nw = (n + 3) / 4;
  for (int i = tid; i < nw; i += blockDim.x) words[i] = 0u;
  __syncthreads();
  for (int hi = 0; hi < G; ++hi) {
    const size_t row = (size_t)b * p.Hq + g * G + hi;
    const int cnt = min(p.sel_cnt[row], p.top_k + 2);
    for (int i = tid; i < cnt; i += blockDim.x) {
      const int pg = p.sel[row * (p.top_k + 2) + i];
      if (pg < 0 || pg >= n) {
        set_err(p.err, BASISKV_DEVERR_SELECTION);
        continue;
      }
      atomicOr(&words[pg >> 2], (1u << hi) << ((pg & 3) * 8));
    }
  }
  __syncthreads();
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int lo = tid * per, hi = min(n, lo + per);
  int c = 0;
  for (int pg = lo; pg < hi; ++pg) c += ((words[pg >> 2] >> ((pg & 3) * 8)) & 0xffu) ? 1 : 0;
  int tot;
  int pos = block_exclusive_scan(c, warp_tot, tot);
  int32_t* out = p.uni + ((size_t)b * p.Hkv + g) * p.umax;
  for (int pg = lo; pg < hi; ++pg) {
    const uint32_t m = (words[pg >> 2] >> ((pg & 3) * 8)) & 0xffu;
    if (m) {
      if (pos < p.umax) out[pos] = (int32_t)((uint32_t)pg | (m << 24));
      ++pos;
    }
  }
  if (tid == 0) {
    if (tot > p.umax) set_err(p.err, BASISKV_DEVERR_SELECTION);
    p.ucnt[(size_t)b * p.Hkv + g] = min(tot, p.umax);
  }
}

// ---------------------------------------------------------------------------
// split attention
// ---------------------------------------------------------------------------


template <typename T, int D>
struct TileLoad {
  static constexpr int DPL = D / 32;
  // lane's DPL consecutive elements of row j
  static __device__ __forceinline__ void row(const T* tile, int j, int lane, float (&out)[DPL]) {
    const T* src = tile + j * D + lane * DPL;
    if constexpr (sizeof(T) == 2 && DPL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(src);
      out[0] = bf16lo(w.x); out[1] = bf16hi(w.x); out[2] = bf16lo(w.y); out[3] = bf16hi(w.y);
    } else if constexpr (sizeof(T) == 2 && DPL == 2) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
      out[0] = bf16lo(w); out[1] = bf16hi(w);
    } else if constexpr (sizeof(T) == 4 && DPL == 4) {
      const float4 w = *reinterpret_cast<const float4*>(src);
      out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;
    } else {
      const float2 w = *reinterpret_cast<const float2*>(src);
      out[0] = w.x; out[1] = w.y;
    }
  }
};

template <typename T, int D, int G, int RPL>
__global__ void __launch_bounds__(kAttnWarps * 32) attn_kernel(AttnParams p) {
  constexpr int DPL = D / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = p.r;
  const int U = p.ucnt[(size_t)b * p.Hkv + g];
  const int e0 = split * p.pps;
  if (e0 >= U) return;  // whole CTA idle (uniform)
  const int e1 = min(U, e0 + p.pps);
  const int L = p.seq_len[b];
  const int n = min((L + p.page - 1) / p.page, p.max_pages);  // union entries are < n
  const int last_valid = L - (n - 1) * p.page;
  const int tpp = p.page / kTile;
  const int ntiles = (e1 - e0) * tpp;

  const uint32_t k_bytes = kTile * D * sizeof(T);
  const uint32_t c_bytes = kTile * r * sizeof(T);
  const uint32_t stage_bytes = (k_bytes + c_bytes + 127u) & ~127u;
  const int kStages = p.nstages;
  unsigned char* ring = smem + (size_t)w * kStages * stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kAttnWarps * kStages * stage_bytes) + w * kStages;

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int32_t* uni = p.uni + ((size_t)b * p.Hkv + g) * p.umax;
  const T* kbase = static_cast<const T*>(p.k_raw);
  const T* cbase = static_cast<const T*>(p.c_lat);

  // tile t of this split -> source pointers, valid tokens, head mask
  auto desc = [&](int t, const T*& kp, const T*& cp, int& valid, uint32_t& mask) {
    const int e = e0 + t / tpp, sub = t - (t / tpp) * tpp;
    const uint32_t ent = (uint32_t)uni[e];
    const int pg = (int)(ent & 0xffffffu);
    mask = ent >> 24;
    valid = (pg == n - 1) ? min(kTile, max(0, last_valid - sub * kTile)) : kTile;
    kp = nullptr;
    cp = nullptr;
    if (pg >= n) {
      valid = 0;
      return;
    }
    const int phys = p.block_table[(size_t)b * p.max_pages + pg];
    if (phys < 0 || phys >= p.num_phys) {
      valid = 0;
      if (lane == 0) set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
      return;
    }
    const size_t row0 = ((size_t)phys * p.Hkv + g) * p.page + (size_t)sub * kTile;
    kp = kbase + row0 * D;
    cp = cbase + row0 * r;
  };

  auto issue = [&](int i) {  // i-th tile of this warp into stage i % kStages
    const T* kp;
    const T* cp;
    int valid;
    uint32_t mask;
    desc(w + i * kAttnWarps, kp, cp, valid, mask);
    if (lane == 0) {
      uint64_t* bar = &bars[i % kStages];
      unsigned char* st = ring + (size_t)(i % kStages) * stage_bytes;
      fence_proxy_async_smem();
      if (valid > 0) {
        mbar_arrive_expect_tx(bar, k_bytes + c_bytes);
        bulk_g2s(st, kp, k_bytes, bar);
        bulk_g2s(st + k_bytes, cp, c_bytes, bar);
      } else {
        mbar_arrive_expect_tx(bar, 0);
      }
    }
  };

  // per-head query (pre-scaled for base-2 softmax) and running state
  float qf[G][DPL];
  {
    const T* qb = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * D;
#pragma unroll
    for (int hi = 0; hi < G; ++hi)
#pragma unroll
      for (int u = 0; u < DPL; ++u) qf[hi][u] = Elem<T>::to_f(qb[hi * D + lane * DPL + u]) * p.qscale;
  }
  float m_run[G], l_run[G], acc[G][RPL];
#pragma unroll
  for (int hi = 0; hi < G; ++hi) {
    m_run[hi] = -INFINITY;
    l_run[hi] = 0.f;
#pragma unroll
    for (int u = 0; u < RPL; ++u) acc[hi][u] = 0.f;
  }

  const int my_count = (ntiles > w) ? (ntiles - w + kAttnWarps - 1) / kAttnWarps : 0;
  const int pre = min(kStages, my_count);
  for (int i = 0; i < pre; ++i) issue(i);

  bool ok = true;
  for (int i = 0; i < my_count; ++i) {
    const int st_idx = i % kStages;
    const uint32_t parity = (uint32_t)((i / kStages) & 1);
    if (!mbar_wait_bounded(&bars[st_idx], parity)) {
      if (lane == 0) set_err(p.err, BASISKV_DEVERR_TIMEOUT);
      // let the copies already in flight land before the CTA leaves
      for (int j = i + 1; j < min(my_count, i + kStages); ++j)
        mbar_wait_bounded(&bars[j % kStages], (uint32_t)((j / kStages) & 1), 200000000LL);
      ok = false;
      break;
    }
    const T* kp;
    const T* cp;
    int valid;
    uint32_t mask;
    desc(w + i * kAttnWarps, kp, cp, valid, mask);
    if (valid > 0) {
      const T* ks = reinterpret_cast<const T*>(ring + (size_t)st_idx * stage_bytes);
      const T* cs = reinterpret_cast<const T*>(ring + (size_t)st_idx * stage_bytes + k_bytes);
      float kf[kTile][DPL];
#pragma unroll
      for (int j = 0; j < kTile; ++j) TileLoad<T, D>::row(ks, j, lane, kf[j]);
      // latents of slots past the valid tokens of a partial page are never
      // written: zero them so that 0 * (stale bits) cannot inject NaN
      float cf[kTile][RPL];
#pragma unroll
      for (int j = 0; j < kTile; ++j)
#pragma unroll
        for (int u = 0; u < RPL; ++u) {
          const int dim = u * 32 + lane;
          cf[j][u] = (dim < r && j < valid) ? Elem<T>::to_f(cs[j * r + dim]) : 0.f;
        }
      const bool tok_ok = (lane >> 1) < valid;
#pragma unroll
      for (int hi = 0; hi < G; ++hi) {
        if (!((mask >> hi) & 1u)) continue;  // warp-uniform
        float s[kTile];
#pragma unroll
        for (int j = 0; j < kTile; ++j) {
          float a = 0.f;
#pragma unroll
          for (int u = 0; u < DPL; ++u) a = fmaf(qf[hi][u], kf[j][u], a);
          s[j] = a;
        }
        transpose_reduce<kTile>(s, lane);  // lane holds token (lane >> 1)
        const float sj = tok_ok ? s[0] : -INFINITY;
        float mx = sj;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        const float m_new = fmaxf(m_run[hi], mx);
        const float corr = exp2f(m_run[hi] - m_new);
        const float pj = exp2f(sj - m_new);
        l_run[hi] = l_run[hi] * corr + ((lane & 1) ? 0.f : pj);
#pragma unroll
        for (int u = 0; u < RPL; ++u) acc[hi][u] *= corr;
#pragma unroll
        for (int j = 0; j < kTile; ++j) {
          const float pb = __shfl_sync(kFull, pj, 2 * j);
#pragma unroll
          for (int u = 0; u < RPL; ++u) acc[hi][u] = fmaf(pb, cf[j][u], acc[hi][u]);
        }
        m_run[hi] = m_new;
      }
    }
    __syncwarp();
    if (i + kStages < my_count) issue(i + kStages);
  }
  (void)ok;

  // merge the warps of this CTA, write one partial per head
  __syncthreads();
  const int stride = 2 + RPL * 32;
  float* mb = reinterpret_cast<float*>(smem);  // [warps][G][stride]
#pragma unroll
  for (int hi = 0; hi < G; ++hi) {
    const float lsum = warp_sum(l_run[hi]);
    float* dst = mb + ((size_t)w * G + hi) * stride;
    if (lane == 0) {
      dst[0] = m_run[hi];
      dst[1] = lsum;
    }
#pragma unroll
    for (int u = 0; u < RPL; ++u) dst[2 + u * 32 + lane] = acc[hi][u];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * r; idx += blockDim.x) {
    const int hi = idx / r, dim = idx - hi * r;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kAttnWarps; ++ww) M = fmaxf(M, mb[((size_t)ww * G + hi) * stride]);
    float Ls = 0.f, As = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < kAttnWarps; ++ww) {
        const float* src = mb + ((size_t)ww * G + hi) * stride;
        const float f = exp2f(src[0] - M);  // 0 for a warp that saw nothing of this head
        Ls += src[1] * f;
        As += src[2 + dim] * f;
      }
    }
    float* out = p.part + (((size_t)b * p.Hq + (size_t)g * G + hi) * p.nsplit + split) * (r + 2);
    out[2 + dim] = As;
    if (dim == 0) {
      out[0] = M;
      out[1] = Ls;
    }
  }
}

// ---------------------------------------------------------------------------
// combine splits
// ---------------------------------------------------------------------------


__global__ void __launch_bounds__(128) combine_kernel(CombineParams p) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = p.Hq / p.Hkv;
  const int U = p.ucnt[(size_t)b * p.Hkv + h / G];
  const int ns = min(p.nsplit, (U + p.pps - 1) / p.pps);
  const float* base = p.part + ((size_t)b * p.Hq + h) * p.nsplit * (p.r + 2);
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, base[(size_t)s * (p.r + 2)]);
  float Ls = 0.f;
  if (M != -INFINITY)
    for (int s = 0; s < ns; ++s) {
      const float* ps = base + (size_t)s * (p.r + 2);
      Ls += ps[1] * exp2f(ps[0] - M);
    }
  for (int dim = threadIdx.x; dim < p.r; dim += blockDim.x) {
    float a = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < ns; ++s) {
        const float* ps = base + (size_t)s * (p.r + 2);
        a += ps[2 + dim] * exp2f(ps[0] - M);
      }
    p.o_lat[((size_t)b * p.Hq + h) * p.r + dim] = (Ls > 0.f) ? a / Ls : 0.f;
  }
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
int attn_pages_per_split(int page) { return max(1, kTilesPerSplit / (page / kTile)); }
int attn_nsplit(int umax, int page) {
  const int pps = attn_pages_per_split(page);
  return (umax + pps - 1) / pps;
}
constexpr size_t kSmemLimit = 227 * 1024;

int attn_stages(int d, int r, int esize) {
  const size_t stage = ((size_t)kTile * (d + r) * esize + 127) & ~(size_t)127;
  int n = kMaxStages;
  while (n > 1 && (size_t)kAttnWarps * n * (stage + 8) > kSmemLimit) --n;
  return n;
}

size_t attn_smem_bytes(int d, int r, int esize, int G, int rpl, int nstages) {
  const size_t stage = ((size_t)kTile * (d + r) * esize + 127) & ~(size_t)127;
  size_t ring = (size_t)kAttnWarps * nstages * stage + (size_t)kAttnWarps * nstages * 8;
  const size_t merge = (size_t)kAttnWarps * G * (2 + rpl * 32) * 4;
  return ring > merge ? ring : merge;
}

template <typename T, int D, int G, int RPL>
static cudaError_t launch_attn_t(const AttnParams& p, int batch, cudaStream_t st) {
  const size_t smem = attn_smem_bytes(D, p.r, sizeof(T), G, RPL, p.nstages);
  cudaError_t e = ensure_smem((const void*)attn_kernel<T, D, G, RPL>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, p.Hkv, batch);
  attn_kernel<T, D, G, RPL><<<grid, kAttnWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int G>
static cudaError_t launch_attn_r(AttnParams p, int batch, cudaStream_t st) {
  p.nstages = attn_stages(D, p.r, sizeof(T));
  const int rpl = (p.r + 31) / 32;
  switch (rpl) {
    case 1: return launch_attn_t<T, D, G, 1>(p, batch, st);
    case 2: return launch_attn_t<T, D, G, 2>(p, batch, st);
    case 3: return launch_attn_t<T, D, G, 3>(p, batch, st);
    case 4: return launch_attn_t<T, D, G, 4>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D>
static cudaError_t launch_attn_g(const AttnParams& p, int G, int batch, cudaStream_t st) {
  switch (G) {
    case 1: return launch_attn_r<T, D, 1>(p, batch, st);
    case 2: return launch_attn_r<T, D, 2>(p, batch, st);
    case 4: return launch_attn_r<T, D, 4>(p, batch, st);
    case 8: return launch_attn_r<T, D, 8>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_attn(const UnionParams& up, const AttnParams& ap, const CombineParams& cp,
                               int batch, int d, bool bf16, cudaStream_t st) {
  const size_t usmem = ((size_t)up.max_pages + 3) / 4 * 4;
  cudaError_t e0 = ensure_smem((const void*)union_kernel, usmem);
  if (e0 != cudaSuccess) return e0;
  union_kernel<<<dim3(up.Hkv, batch), 256, usmem, st>>>(up);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int G = ap.Hq / ap.Hkv;
  if (bf16)
    e = (d == 128) ? launch_attn_g<__nv_bfloat16, 128>(ap, G, batch, st)
                   : launch_attn_g<__nv_bfloat16, 64>(ap, G, batch, st);
  else
    e = (d == 128) ? launch_attn_g<float, 128>(ap, G, batch, st)
                   : launch_attn_g<float, 64>(ap, G, batch, st);
  if (e != cudaSuccess) return e;
  combine_kernel<<<dim3(cp.Hq, batch), 128, 0, st>>>(cp);
  return cudaGetLastError();
}

}  // namespace bkv
