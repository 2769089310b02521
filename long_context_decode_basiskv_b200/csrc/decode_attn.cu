// Step 4 of the BasisKV decode step: exact attention on the routed pages.
//
// Only the selected key pages are read back, and the QK scores on them are
// exact (BasisKV abstract; kongchang.com explainer, section
// "用Value潜变量辅助Key路由"); the attention formula is the textbook one
// (machinelearning.ru "KV-кэширование", section "Математическая формализация"),
// restricted to the selected tokens, with the weights applied to the rank-r
// Value latents instead of full-width values.
//
// Two launches:
//  union  one CTA per (sequence, KV head): merges the G query heads'
//         selections into one ascending page list with a G-bit head mask per
//         page (a page chosen by several heads of a group is read once), and
//         zeroes the group's split counter.
//  attn   one CTA per (sequence, KV head, split of the union).  Warp 0 is the
//         producer: its lanes hold the split's union entries (page, mask,
//         physical page, valid tokens) and lane 0 streams 16-token tiles (raw
//         K rows and C rows, each contiguous in the page block) into a ring of
//         shared-memory stages with 1-D bulk copies (cp.async.bulk, mbarrier
//         completion, no multicast), writing each stage's head mask beside it.
//         Warps 1..G are the consumers, one per query head of the group: a warp
//         whose head selected the tile forms its 16 exact scores, updates an
//         online softmax (running max and sum, base 2) and accumulates p * C;
//         every consumer releases the stage.  Each head's split result (max,
//         sum, acc[r]) goes to the workspace; the last CTA of a group to finish
//         (counted with an atomic) merges the group's splits with the
//         log-sum-exp rule and writes o_lat.
// HBM-bound: every byte of the union's pages is read once.
#include "kernels.cuh"

namespace bkv {

constexpr int kTile = 16;           // tokens per tile
constexpr int kStages = 4;          // ring depth per CTA
constexpr int kTargetCtas = 888;    // one wave of attn CTAs on a B200 (148 SMs x 6)

// ---------------------------------------------------------------------------
// plan: tiles per split and scratch layout (independent of the device)
// ---------------------------------------------------------------------------
static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodePlan decode_plan(int Hq, int Hkv, int page, int r, int top_k, int batch, int max_pages) {
  DecodePlan pl{};
  const int G = Hq / Hkv;
  long long um = (long long)G * (top_k + 2);
  if (um > max_pages) um = max_pages;
  pl.umax = (int)um;
  pl.tpp = page / kTile;
  const long long groups = (long long)batch * Hkv;
  const long long tiles = (long long)pl.umax * pl.tpp;
  long long eps = (tiles * groups + kTargetCtas - 1) / kTargetCtas;  // tiles per split, then pages
  eps = (eps + pl.tpp - 1) / pl.tpp;
  if (eps < 1) eps = 1;
  pl.eps = (int)eps;
  pl.nsplit = (pl.umax + pl.eps - 1) / pl.eps;
  size_t off = 0;
  pl.uni_off = off;
  off += up256((size_t)batch * Hkv * pl.umax * 4);
  pl.ucnt_off = off;
  off += up256((size_t)batch * Hkv * 4);
  pl.cnt_off = off;
  off += up256((size_t)batch * Hkv * 4);
  pl.part_off = off;
  off += up256((size_t)batch * Hq * pl.nsplit * (r + 2) * 4);
  pl.bytes = off;
  return pl;
}

// ---------------------------------------------------------------------------
// union of the group's selections
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) union_kernel(UnionParams p) {
  extern __shared__ __align__(16) uint32_t words[];  // [ceil(max_pages / 4)] byte masks
  __shared__ int warp_tot[32];
  __shared__ int s_cnt[8];
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int G = p.Hq / p.Hkv;
  const int row_len = p.top_k + 2;
  const size_t row0 = (size_t)b * p.Hq + (size_t)g * G;
  const int L = p.seq_len[b];
  const int n = min((L + p.page - 1) / p.page, p.max_pages);
  const int nw = (n + 3) / 4;
  if (tid == 0) p.cnt[(size_t)b * p.Hkv + g] = 0;
  if (tid < G) s_cnt[tid] = min(p.sel_cnt[row0 + tid], row_len);
  for (int i = tid; i < nw; i += blockDim.x) words[i] = 0u;
  __syncthreads();
  // the G selection rows are contiguous: one flat pass, every load issued at once
  for (int i = tid; i < G * row_len; i += blockDim.x) {
    const int hi = i / row_len;
    if (i - hi * row_len >= s_cnt[hi]) continue;
    const int pg = p.sel[row0 * row_len + i];
    if (pg < 0 || pg >= n) {
      set_err(p.err, BASISKV_DEVERR_SELECTION);
      continue;
    }
    atomicOr(&words[pg >> 2], (1u << hi) << ((pg & 3) * 8));
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
// split attention with in-kernel merge
// ---------------------------------------------------------------------------
template <typename T, int D>
struct KRow {
  static constexpr int DPL = D / 32;
  // lane's DPL consecutive elements of row j of a [16][D] tile
  static __device__ __forceinline__ void load(const T* tile, int j, int lane, float (&out)[DPL]) {
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

// two consecutive latent dims (dim, dim + 1) of one C row
template <typename T>
__device__ __forceinline__ void load_pair(const T* row, int dim, float& a, float& b) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(row + dim);
    a = bf16lo(w);
    b = bf16hi(w);
  } else {
    const float2 w = *reinterpret_cast<const float2*>(row + dim);
    a = w.x;
    b = w.y;
  }
}

template <typename T, int D, int G, int CU>
__global__ void __launch_bounds__(32 * (G + 1)) attn_kernel(AttnParams p) {
  constexpr int DPL = D / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t meta[kStages];  // head mask | valid tokens << 8 of the tile in each stage
  __shared__ int s_last;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = p.r;
  const size_t bg = (size_t)b * p.Hkv + g;
  const int U = p.ucnt[bg];
  const int e0 = split * p.eps;
  const int nsplit_active = (U + p.eps - 1) / p.eps;
  if (e0 >= U) {
    // no work in this split; split 0 of an empty group still defines its output
    if (split == 0 && U == 0)
      for (int i = threadIdx.x; i < G * r; i += blockDim.x)
        p.o_lat[((size_t)b * p.Hq + (size_t)g * G) * r + i] = 0.f;
    return;
  }
  const int nent = min(U, e0 + p.eps) - e0;
  const int ntiles = nent * p.tpp;

  const uint32_t k_bytes = kTile * D * sizeof(T);
  const uint32_t c_bytes = kTile * r * sizeof(T);
  const uint32_t stage_bytes = (k_bytes + c_bytes + 127u) & ~127u;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * stage_bytes);
  uint64_t* empty = full + kStages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], G);
    }
    fence_mbar_init();
  }
  __syncthreads();

  bool ok = true;
  if (warp == 0) {
    // ---------------- producer ----------------
    const int L = p.seq_len[b];
    const int n = min((L + p.page - 1) / p.page, p.max_pages);
    const int last_valid = L - (n - 1) * p.page;
    const int32_t* uni = p.uni + bg * p.umax;
    const T* kbase = static_cast<const T*>(p.k_raw);
    const T* cbase = static_cast<const T*>(p.c_lat);
    for (int cb = 0; cb < nent && ok; cb += 32) {
      // lane e holds union entry e0 + cb + e
      uint32_t my_mask = 0;
      int my_phys = -1, my_valid = 0;
      if (cb + lane < nent) {
        const uint32_t ent = (uint32_t)uni[e0 + cb + lane];
        const int pg = (int)(ent & 0xffffffu);
        my_mask = ent >> 24;
        if (pg < n) {
          const int ph = p.block_table[(size_t)b * p.max_pages + pg];
          if (ph >= 0 && ph < p.num_phys) {
            my_phys = ph;
            my_valid = (pg == n - 1) ? last_valid : p.page;
          } else {
            set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
          }
        }
      }
      const int t_end = min(nent, cb + 32) * p.tpp;
      for (int t = cb * p.tpp; t < t_end; ++t) {
        const int el = t / p.tpp - cb, sub = t - (t / p.tpp) * p.tpp;
        const int ph = __shfl_sync(kFull, my_phys, el);
        const uint32_t mask = __shfl_sync(kFull, my_mask, el);
        const int pv = __shfl_sync(kFull, my_valid, el);
        const int valid = (ph >= 0) ? min(kTile, max(0, pv - sub * kTile)) : 0;
        const int s = t % kStages;
        if (t >= kStages && !mbar_wait_bounded(&empty[s], (uint32_t)(((t / kStages) - 1) & 1))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          meta[s] = mask | ((uint32_t)valid << 8);
          unsigned char* st = smem + (size_t)s * stage_bytes;
          fence_proxy_async_smem();
          if (valid > 0) {
            const size_t row0 = ((size_t)ph * p.Hkv + g) * p.page + (size_t)sub * kTile;
            mbar_arrive_expect_tx(&full[s], k_bytes + c_bytes);
            bulk_g2s(st, kbase + row0 * D, k_bytes, &full[s]);
            bulk_g2s(st + k_bytes, cbase + row0 * r, c_bytes, &full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], 0);
          }
        }
        __syncwarp();
      }
    }
  } else {
    // ---------------- consumer: one query head ----------------
    const int hi = warp - 1;
    const int h = g * G + hi;
    float qf[DPL];
    {
      const T* qr = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * D + lane * DPL;
#pragma unroll
      for (int u = 0; u < DPL; ++u) qf[u] = Elem<T>::to_f(qr[u]) * p.qscale;
    }
    float m_run = -INFINITY, l_run = 0.f;
    float acc[CU][2];
#pragma unroll
    for (int u = 0; u < CU; ++u) acc[u][0] = acc[u][1] = 0.f;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kStages;
      if (!mbar_wait_bounded(&full[s], (uint32_t)((t / kStages) & 1))) {
        ok = false;
        break;
      }
      const uint32_t mt = meta[s];
      const int valid = (int)(mt >> 8);
      if (((mt >> hi) & 1u) && valid > 0) {
        const T* ks = reinterpret_cast<const T*>(smem + (size_t)s * stage_bytes);
        const T* cs = reinterpret_cast<const T*>(smem + (size_t)s * stage_bytes + k_bytes);
        float sc[kTile];
#pragma unroll
        for (int j = 0; j < kTile; ++j) {
          float kv[DPL];
          KRow<T, D>::load(ks, j, lane, kv);
          float a = 0.f;
#pragma unroll
          for (int u = 0; u < DPL; ++u) a = fmaf(qf[u], kv[u], a);
          sc[j] = a;
        }
        transpose_reduce<kTile>(sc, lane);  // lane holds token (lane >> 1)
        const float sj = ((lane >> 1) < valid) ? sc[0] : -INFINITY;
        float mx = sj;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        const float m_new = fmaxf(m_run, mx);
        const float corr = exp2f(m_run - m_new);
        const float pj = exp2f(sj - m_new);
        l_run = l_run * corr + ((lane & 1) ? 0.f : pj);
#pragma unroll
        for (int u = 0; u < CU; ++u) {
          acc[u][0] *= corr;
          acc[u][1] *= corr;
        }
#pragma unroll
        for (int j = 0; j < kTile; ++j) {
          const float pb = __shfl_sync(kFull, pj, 2 * j);
          if (j < valid) {  // slots past the valid tokens hold stale bits
#pragma unroll
            for (int u = 0; u < CU; ++u) {
              const int dim = 64 * u + 2 * lane;
              if (dim < r) {
                float c0, c1;
                load_pair<T>(cs + j * r, dim, c0, c1);
                acc[u][0] = fmaf(pb, c0, acc[u][0]);
                acc[u][1] = fmaf(pb, c1, acc[u][1]);
              }
            }
          }
        }
        m_run = m_new;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // this head's result for the split
    const float lsum = warp_sum(l_run);
    float* out = p.part + (((size_t)b * p.Hq + h) * p.nsplit + split) * (r + 2);
    if (lane == 0) {
      out[0] = m_run;
      out[1] = lsum;
    }
#pragma unroll
    for (int u = 0; u < CU; ++u) {
      const int dim = 64 * u + 2 * lane;
      if (dim < r) {
        out[2 + dim] = acc[u][0];
        out[3 + dim] = acc[u][1];
      }
    }
  }
  if (!ok) set_err(p.err, BASISKV_DEVERR_TIMEOUT);

  // the last CTA of the group to finish merges every split of its G heads
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&p.cnt[bg], 1) == nsplit_active - 1);
  __syncthreads();
  if (!s_last || warp == 0) return;
  __threadfence();
  const int hi = warp - 1;
  const int h = g * G + hi;
  const float* base = p.part + ((size_t)b * p.Hq + h) * p.nsplit * (r + 2);
  float M = -INFINITY;
  for (int s = lane; s < nsplit_active; s += 32) M = fmaxf(M, __ldcg(base + (size_t)s * (r + 2)));
  M = warp_max(M);
  float Ls = 0.f;
  for (int s = lane; s < nsplit_active; s += 32) {
    const float ms = __ldcg(base + (size_t)s * (r + 2));
    if (ms != -INFINITY) Ls += __ldcg(base + (size_t)s * (r + 2) + 1) * exp2f(ms - M);
  }
  Ls = warp_sum(Ls);
  for (int dim = lane; dim < r; dim += 32) {
    float a = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < nsplit_active; ++s) {
        const float* ps = base + (size_t)s * (r + 2);
        const float ms = __ldcg(ps);
        if (ms != -INFINITY) a += __ldcg(ps + 2 + dim) * exp2f(ms - M);
      }
    p.o_lat[((size_t)b * p.Hq + h) * r + dim] = (Ls > 0.f) ? a / Ls : 0.f;
  }
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
size_t attn_smem_bytes(int d, int r, int esize) {
  const size_t stage = ((size_t)kTile * (d + r) * esize + 127) & ~(size_t)127;
  return (size_t)kStages * stage + 2 * kStages * 8;
}

template <typename T, int D, int G, int CU>
static cudaError_t launch_attn_t(const AttnParams& p, int batch, cudaStream_t st) {
  const size_t smem = attn_smem_bytes(D, p.r, sizeof(T));
  cudaError_t e = ensure_smem((const void*)attn_kernel<T, D, G, CU>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, p.Hkv, batch);
  attn_kernel<T, D, G, CU><<<grid, 32 * (G + 1), smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, int D, int G>
static cudaError_t launch_attn_r(const AttnParams& p, int batch, cudaStream_t st) {
  return (p.r <= 64) ? launch_attn_t<T, D, G, 1>(p, batch, st) : launch_attn_t<T, D, G, 2>(p, batch, st);
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

cudaError_t launch_decode_attn(const DecodePlan& pl, const DecodeArgs& a, void* scratch, int batch,
                               cudaStream_t st) {
  char* base = static_cast<char*>(scratch);
  int32_t* uni = reinterpret_cast<int32_t*>(base + pl.uni_off);
  int32_t* ucnt = reinterpret_cast<int32_t*>(base + pl.ucnt_off);
  int32_t* cnt = reinterpret_cast<int32_t*>(base + pl.cnt_off);
  float* part = reinterpret_cast<float*>(base + pl.part_off);
  UnionParams up{a.sel, a.sel_cnt, a.seq_len, uni, ucnt, cnt, a.err, a.Hq, a.Hkv, a.page, a.max_pages, a.top_k,
                 pl.umax};
  const size_t usmem = ((size_t)a.max_pages + 3) / 4 * 4;
  cudaError_t e = ensure_smem((const void*)union_kernel, usmem);
  if (e != cudaSuccess) return e;
  union_kernel<<<dim3(a.Hkv, batch), 256, usmem, st>>>(up);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  AttnParams ap{a.q, a.k_raw, a.c_lat, a.block_table, a.seq_len, uni, ucnt, cnt, part, a.o_lat, a.err,
                a.Hq, a.Hkv, a.page, a.r, a.max_pages, a.num_phys, pl.umax, pl.tpp, pl.eps, pl.nsplit,
                (float)(1.4426950408889634 / sqrt((double)a.d))};
  const int G = a.Hq / a.Hkv;
  if (a.bf16)
    return (a.d == 128) ? launch_attn_g<__nv_bfloat16, 128>(ap, G, batch, st)
                        : launch_attn_g<__nv_bfloat16, 64>(ap, G, batch, st);
  return (a.d == 128) ? launch_attn_g<float, 128>(ap, G, batch, st) : launch_attn_g<float, 64>(ap, G, batch, st);
}

}  // namespace bkv
