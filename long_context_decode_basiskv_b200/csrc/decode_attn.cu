// Step 4 of the BasisKV decode step: exact attention on the routed pages.
//
// Only the selected key pages are read back, and the QK scores on them are
// exact (BasisKV abstract; kongchang.com explainer, section
// "用Value潜变量辅助Key路由"); the attention formula is the textbook one
// (machinelearning.ru "KV-кэширование", section "Математическая формализация"),
// restricted to the selected tokens, with the weights applied to the rank-r
// Value latents instead of full-width values.
//
// One launch: one CTA per (sequence, KV head, split of the union); the splits
// fill one resident wave (decode_plan).  Each CTA first merges the G query
// heads' selections into the ascending union of pages with a G-bit head mask
// per page (a page chosen by several heads of a group is read once) and keeps
// its split's equal share of it.  Two kernels stream the slice's 16-token
// tiles (raw K rows and C rows, each contiguous in the page block) with 1-D
// bulk copies (cp.async.bulk, mbarrier completion, bounded waits, no
// multicast):
//   * attn_mma_kernel (bf16, the main path): four warps per CTA, each with its
//     own 3-slot ring, run all G heads of the group on the tensor cores
//     (mma.sync m16n8k16: scores with heads as rows, online softmax in base
//     2, P.C accumulated in registers); see the section below.
//   * attn_kernel (fp32 and shapes without the swizzled layout): warp 0
//     produces into a shared ring, warps 1..G consume, one per query head of
//     the group, forming 16 exact scores per tile on the CUDA cores.
// Each head's split result (max, sum, acc[r]) goes to the workspace; the last
// CTA of a group to finish (counted with an atomic) merges the group's splits
// with the log-sum-exp rule and writes o_lat.
// HBM-bound: every byte of the union's pages is read once.
#include "kernels.cuh"

namespace bkv {

constexpr int kTile = 16;           // tokens per tile
constexpr int kStages = 4;          // ring depth per CTA
constexpr int kCoreCtasPerSm = 6;   // resident CTAs per SM of the CUDA-core attention kernel
constexpr int kMmaCtasPerSm = 3;    // ... and of the tensor-core one (registers and shared memory)

// ---------------------------------------------------------------------------
// plan: splits per (sequence, KV head) and the scratch layout
// ---------------------------------------------------------------------------
static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// The splits fill one resident wave of the kernel exactly: with q = slots /
// groups and m = slots % groups, the last m groups get q + 1 splits and the
// others q (at least one each), so every SM holds the same number of CTAs and
// about the same number of tiles (the memory system gives every SM a similar
// share of the bandwidth, so an SM with more work would finish last).  Each
// split takes an equal share of its group's union at run time.  The first
// groups' unused CTAs (split q) exit at once and free their slots.
DecodePlan decode_plan(int Hq, int Hkv, int page, int r, int top_k, int batch, int max_pages, bool bf16, int d,
                       int num_sms) {
  DecodePlan pl{};
  const long long slots = (long long)num_sms * (kc_swizzled(bf16, d, r) ? kMmaCtasPerSm : kCoreCtasPerSm);
  const int G = Hq / Hkv;
  long long um = (long long)G * (top_k + 2);
  if (um > max_pages) um = max_pages;
  pl.umax = (int)um;
  pl.tpp = page / kTile;
  const long long groups = (long long)batch * Hkv;
  long long q = slots / groups, m = slots % groups;
  if (q >= pl.umax) {
    q = pl.umax;
    m = 0;
  }
  if (q < 1) {
    q = 1;
    m = 0;
  }
  pl.nsplit_lo = (int)q;
  pl.nsplit = (int)(m > 0 ? q + 1 : q);
  pl.rich_from = (int)(groups - m);
  pl.eps = (pl.umax + pl.nsplit_lo - 1) / pl.nsplit_lo;
  size_t off = 0;
  pl.cnt_off = off;
  off += up256((size_t)batch * Hkv * 4);
  pl.part_off = off;
  off += up256((size_t)batch * Hq * pl.nsplit * (r + 2) * 4);
  pl.bytes = off;
  return pl;
}

// ---------------------------------------------------------------------------
// union of the group's selections, built by every CTA for its own split
// ---------------------------------------------------------------------------
// All threads of the CTA call this.  It merges the G heads' selections of
// (b, g) into per-page head masks in `words` (shared scratch of at least
// ceil(max_pages / 4) words) and ranks the selected pages in ascending order
// with a block scan.  The union of U pages is cut into nsplit equal slices of
// ceil(U / nsplit) entries; the entries of slice `split` are stored as
// page | mask << 24 in `ent` (shared).  Every load of the selections is issued
// before the first barrier, so their latencies overlap.
struct UnionSlice {
  int U;       // union size of (b, g)
  int e0;      // first union entry of this split
  int cnt;     // entries in this split (0: no work)
  int active;  // splits of (b, g) with work
};
constexpr int kUnionLoads = 8;  // selection entries a thread loads before the first barrier

__device__ UnionSlice union_slice(const AttnParams& p, int b, int g, int G, int split, uint32_t* words,
                                  uint32_t* ent, int* warp_tot, int* s_cnt) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int row_len = p.top_k + 2;
  const size_t row0 = (size_t)b * p.Hq + (size_t)g * G;
  const int total = G * row_len;
  const int32_t* selg = p.sel + row0 * row_len;  // the G rows are contiguous
  const int L = p.seq_len[b];
  if (tid < G) s_cnt[tid] = min(p.sel_cnt[row0 + tid], row_len);
  int v[kUnionLoads];
#pragma unroll
  for (int j = 0; j < kUnionLoads; ++j) {
    const int i = tid + j * nthr;
    v[j] = (i < total) ? selg[i] : -1;
  }
  for (int i = tid; i < (p.max_pages + 3) / 4; i += nthr) words[i] = 0u;
  __syncthreads();
  const int n = max(0, min((L + p.page - 1) / p.page, p.max_pages));
  auto mark = [&](int i, int pg) {
    const int hi = i / row_len;
    if (i - hi * row_len >= s_cnt[hi]) return;
    if (pg < 0 || pg >= n) {
      set_err(p.err, BASISKV_DEVERR_SELECTION);
      return;
    }
    atomicOr(&words[pg >> 2], (1u << hi) << ((pg & 3) * 8));
  };
#pragma unroll
  for (int j = 0; j < kUnionLoads; ++j) {
    const int i = tid + j * nthr;
    if (i < total) mark(i, v[j]);
  }
  for (int i = tid + kUnionLoads * nthr; i < total; i += nthr) mark(i, selg[i]);
  __syncthreads();
  const int per = (n + nthr - 1) / nthr;
  const int lo = tid * per, hi = min(n, lo + per);
  int c = 0;
  for (int pg = lo; pg < hi; ++pg) c += ((words[pg >> 2] >> ((pg & 3) * 8)) & 0xffu) ? 1 : 0;
  int tot;
  int pos = block_exclusive_scan(c, warp_tot, tot);
  UnionSlice sl;
  sl.U = tot;
  const int ns = ((int)(b * p.Hkv + g) >= p.rich_from) ? p.nsplit : p.nsplit_lo;  // splits of this group
  const int eps = (tot + ns - 1) / ns;
  sl.e0 = split * eps;
  sl.cnt = (split < ns) ? max(0, min(tot, sl.e0 + eps) - sl.e0) : 0;
  sl.active = eps > 0 ? (tot + eps - 1) / eps : 0;
  for (int pg = lo; pg < hi && pos < sl.e0 + sl.cnt; ++pg) {
    const uint32_t m = (words[pg >> 2] >> ((pg & 3) * 8)) & 0xffu;
    if (m) {
      if (pos >= sl.e0) ent[pos - sl.e0] = (uint32_t)pg | (m << 24);
      ++pos;
    }
  }
  __syncthreads();
  return sl;
}

// Offset of the split's entry list in dynamic shared memory: after the ring
// (and its barriers), and after the page-mask scratch of union_slice.
__host__ __device__ __forceinline__ size_t attn_ent_offset(size_t ring_bytes, int max_pages) {
  const size_t masks = ((size_t)max_pages + 15) & ~(size_t)15;
  return ((ring_bytes > masks ? ring_bytes : masks) + 15) & ~(size_t)15;
}

// After writing its split results, a CTA counts itself on the group's counter;
// the last one of the group merges.  The merging CTA puts the counter back to
// zero, so counters are zero between calls (the workspace is zero-filled once).
__device__ __forceinline__ bool last_of_group(const AttnParams& p, size_t bg, int nsplit_active, int* s_last) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&p.cnt[bg], 1);
    if (prev >= nsplit_active) set_err(p.err, BASISKV_DEVERR_WORKSPACE);
    *s_last = (prev == nsplit_active - 1);
  }
  __syncthreads();
  if (!*s_last) return false;
  __threadfence();
  return true;
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

// The last CTA of a (sequence, KV head) group merges the group's split
// results: for each of its G heads, log-sum-exp over the splits.  Heads are
// spread over `nw` warps starting at warp index `wi`.
__device__ __forceinline__ void merge_group_splits(const AttnParams& p, int b, int g, int G, int r,
                                                   int nsplit_active, int wi, int nw, int lane) {
  constexpr int kDimIt = 4;  // r <= 128: dims lane + 32 k
  constexpr int kBatch = 8;  // splits whose values are loaded together
  const int stride = r + 2;
  for (int hi = wi; hi < G; hi += nw) {
    const int h = g * G + hi;
    const float* base = p.part + ((size_t)b * p.Hq + h) * p.nsplit * stride;
    float M = -INFINITY;
    for (int s = lane; s < nsplit_active; s += 32) M = fmaxf(M, __ldcg(base + (size_t)s * stride));
    M = warp_max(M);
    float Ls = 0.f;
    float acc[kDimIt] = {0.f, 0.f, 0.f, 0.f};
    for (int c0 = 0; c0 < nsplit_active; c0 += 32) {
      // lane s: the weight of split c0 + s
      const int sl = c0 + lane;
      float wl = 0.f;
      if (sl < nsplit_active) {
        const float ms = __ldcg(base + (size_t)sl * stride);
        if (ms != -INFINITY) {
          wl = exp2f(ms - M);
          Ls += __ldcg(base + (size_t)sl * stride + 1) * wl;
        }
      }
      const int cn = min(32, nsplit_active - c0);
      for (int j0 = 0; j0 < cn; j0 += kBatch) {
        float x[kBatch][kDimIt];
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
#pragma unroll
          for (int k = 0; k < kDimIt; ++k) {
            const int dim = lane + 32 * k;
            x[j][k] = (j0 + j < cn && dim < r) ? __ldcg(base + (size_t)(c0 + j0 + j) * stride + 2 + dim) : 0.f;
          }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const float wt = __shfl_sync(kFull, wl, (j0 + j) & 31);
#pragma unroll
          for (int k = 0; k < kDimIt; ++k) acc[k] = fmaf(x[j][k], wt, acc[k]);
        }
      }
    }
    Ls = warp_sum(Ls);
#pragma unroll
    for (int k = 0; k < kDimIt; ++k) {
      const int dim = lane + 32 * k;
      if (dim < r) p.o_lat[((size_t)b * p.Hq + h) * r + dim] = (Ls > 0.f) ? acc[k] / Ls : 0.f;
    }
  }
}

template <typename T, int D, int G, int CU>
__global__ void __launch_bounds__(32 * (G + 1)) attn_kernel(AttnParams p) {
  constexpr int DPL = D / 32;
  allow_dependents();  // the out-projection may launch and start streaming its weights
  grid_dep_wait();     // the selection is complete (this kernel may launch before it ends)
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t meta[kStages];  // head mask | valid tokens << 8 of the tile in each stage
  __shared__ int s_last;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = p.r;
  const size_t bg = (size_t)b * p.Hkv + g;
  const uint32_t k_bytes = kTile * D * sizeof(T);
  const uint32_t c_bytes = kTile * r * sizeof(T);
  const uint32_t stage_bytes = (k_bytes + c_bytes + 127u) & ~127u;
  // shared memory: [ring | barriers] (page-mask scratch while the union is built) then the split's entries
  uint32_t* ent = reinterpret_cast<uint32_t*>(smem + attn_ent_offset(kStages * stage_bytes + 2 * kStages * 8, p.max_pages));
  __shared__ int warp_tot[32];
  __shared__ int s_cnt[8];
  const UnionSlice sl = union_slice(p, b, g, G, split, reinterpret_cast<uint32_t*>(smem), ent, warp_tot, s_cnt);
  const int U = sl.U, nsplit_active = sl.active;
  if (sl.cnt == 0) {
    // no work in this split; split 0 of an empty group still defines its output
    if (split == 0 && U == 0)
      for (int i = threadIdx.x; i < G * r; i += blockDim.x)
        p.o_lat[((size_t)b * p.Hq + (size_t)g * G) * r + i] = 0.f;
    return;
  }
  const int nent = sl.cnt;
  const int ntiles = nent * p.tpp;
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
    const T* kbase = static_cast<const T*>(p.k_raw);
    const T* cbase = static_cast<const T*>(p.c_lat);
    for (int cb = 0; cb < nent && ok; cb += 32) {
      // lane e holds entry cb + e of this split
      uint32_t my_mask = 0;
      int my_phys = -1, my_valid = 0;
      if (cb + lane < nent) {
        const uint32_t en = ent[cb + lane];
        const int pg = (int)(en & 0xffffffu);
        my_mask = en >> 24;
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
  if (!last_of_group(p, bg, nsplit_active, &s_last)) return;
  if (warp >= 1) merge_group_splits(p, b, g, G, r, nsplit_active, warp - 1, G, lane);
  if (threadIdx.x == 0) p.cnt[bg] = 0;
}

// ---------------------------------------------------------------------------
// bf16 path: one consumer warp per tile, all G heads of the group at once on
// the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate)
//   S^T[16 x 16] = Q[16 (heads, padded) x d] . K_tile^T[d x 16 tokens]
//   O[16 x r]   += P[16 x 16 tokens] . C_tile[16 tokens x r]
// P reuses the S^T accumulator registers as the A operand (the m16n8k16 C and
// A fragments line up), rounded to bf16.  K and C rows are XOR-swizzled in the
// page (see swz()), so ldmatrix reads 8 rows without bank conflicts.
// ---------------------------------------------------------------------------
constexpr int kMmaWarps = 4;       // warps per CTA; each streams and consumes its own tiles
constexpr int kMmaWarpStages = 3;  // ring slots per warp

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int D, int G, int NT>
__global__ void __launch_bounds__(32 * kMmaWarps, 3) attn_mma_kernel(AttnParams p) {
  constexpr int KS = D / 16;
  allow_dependents();  // the out-projection may launch and start streaming its weights
  grid_dep_wait();     // the selection is complete (this kernel may launch before it ends)
  constexpr int SW = kMmaWarpStages;
  constexpr int R = NT * 8;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_last;
  __shared__ uint32_t meta_all[kMmaWarps][kMmaWarpStages];  // head mask | valid << 8 of each slot's tile
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t* meta = meta_all[w];
  const size_t bg = (size_t)b * p.Hkv + g;
  constexpr uint32_t k_bytes = kTile * D * 2;
  constexpr uint32_t c_bytes = kTile * R * 2;
  constexpr uint32_t stage_bytes = (k_bytes + c_bytes + 127u) & ~127u;
  constexpr uint32_t ring_bytes = kMmaWarps * SW * (stage_bytes + 8);
  // shared memory: [rings | barriers] (page-mask scratch while the union is built) then the split's entries
  uint32_t* ent = reinterpret_cast<uint32_t*>(smem + attn_ent_offset(ring_bytes, p.max_pages));
  __shared__ int warp_tot[32];
  __shared__ int s_cnt[8];
  const UnionSlice sl = union_slice(p, b, g, G, split, reinterpret_cast<uint32_t*>(smem), ent, warp_tot, s_cnt);
  const int U = sl.U, nsplit_active = sl.active;
  if (sl.cnt == 0) {
    if (split == 0 && U == 0)
      for (int i = threadIdx.x; i < G * R; i += blockDim.x)
        p.o_lat[((size_t)b * p.Hq + (size_t)g * G) * R + i] = 0.f;
    return;
  }
  const int nent = sl.cnt;
  const int ntiles = nent * p.tpp;

  unsigned char* ring = smem + (size_t)w * SW * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kMmaWarps * SW * stage_bytes) + w * SW;
  if (lane == 0) {
    for (int s = 0; s < SW; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int L = p.seq_len[b];
  const int n = min((L + p.page - 1) / p.page, p.max_pages);
  const int last_valid = L - (n - 1) * p.page;
  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.k_raw);
  const __nv_bfloat16* cbase = static_cast<const __nv_bfloat16*>(p.c_lat);

  // this warp's tiles: t = w + kMmaWarps * i; lane j of a batch of 32 holds tile i = base + j
  const int my_tiles = (ntiles > w) ? (ntiles - w + kMmaWarps - 1) / kMmaWarps : 0;
  int d_phys = -1, d_valid = 0;
  uint32_t d_mask = 0;
  auto load_desc = [&](int base) {  // descriptors of tiles base .. base+31 of this warp
    d_phys = -1;
    d_valid = 0;
    d_mask = 0;
    const int i = base + lane;
    if (i < my_tiles) {
      const int t = w + kMmaWarps * i;
      const int e = t / p.tpp, sub = t - e * p.tpp;
      const uint32_t en = ent[e];
      const int pg = (int)(en & 0xffffffu);
      d_mask = en >> 24;
      if (pg < n) {
        const int ph = p.block_table[(size_t)b * p.max_pages + pg];
        if (ph >= 0 && ph < p.num_phys) {
          d_phys = ph * p.tpp + sub;  // tile index of the head-g page block, in 16-row units
          d_valid = min(kTile, max(0, ((pg == n - 1) ? last_valid : p.page) - sub * kTile));
        } else {
          set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
        }
      }
    }
  };
  const uint64_t stream_pol = l2_evict_first();
  // issue tile i of this warp into slot i % SW (lane 0); all lanes take part in the shuffles
  auto issue = [&](int i) {
    const int j = i & 31;
    const int ph = __shfl_sync(kFull, d_phys, j);
    const int valid = __shfl_sync(kFull, d_valid, j);
    const uint32_t mask = __shfl_sync(kFull, d_mask, j);
    if (lane == 0) {
      meta[i % SW] = mask | ((uint32_t)valid << 8);
      uint64_t* bar = &full[i % SW];
      unsigned char* st = ring + (size_t)(i % SW) * stage_bytes;
      fence_proxy_async_smem();
      if (valid > 0) {
        const int pidx = ph / p.tpp, sub = ph - pidx * p.tpp;
        const size_t row0 = ((size_t)pidx * p.Hkv + g) * p.page + (size_t)sub * kTile;
        mbar_arrive_expect_tx(bar, k_bytes + c_bytes);
        bulk_g2s_hint(st, kbase + row0 * D, k_bytes, bar, stream_pol);  // read once: evict first
        bulk_g2s_hint(st + k_bytes, cbase + row0 * R, c_bytes, bar, stream_pol);
      } else {
        mbar_arrive_expect_tx(bar, 0);
      }
    }
  };

  const int gr = lane >> 2, tq = lane & 3;  // fragment row (head) and column pair
  const bool head_ok = gr < G;
  uint32_t qa[KS][2];
  {
    const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G + gr) * D;
#pragma unroll
    for (int s2 = 0; s2 < KS; ++s2) {
      qa[s2][0] = head_ok ? *reinterpret_cast<const uint32_t*>(qr + 16 * s2 + 2 * tq) : 0u;
      qa[s2][1] = head_ok ? *reinterpret_cast<const uint32_t*>(qr + 16 * s2 + 2 * tq + 8) : 0u;
    }
  }
  float m_run = -INFINITY, l_run = 0.f;
  float oacc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
  constexpr int mk = 7;  // K rows have 8 or 16 chunks
  const int mc = swz_mask(R);
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix mi takes its row rr from this lane
  bool ok = true;

  if (my_tiles > 0) load_desc(0);
  for (int i = 0; i < min(SW, my_tiles); ++i) issue(i);
  for (int i = 0; i < my_tiles; ++i) {
    const int s = i % SW;
    if (!mbar_wait_bounded(&full[s], (uint32_t)((i / SW) & 1))) {
      ok = false;
      break;
    }
    const uint32_t mt = meta[s];
    const int valid = (int)(mt >> 8);
    if (valid > 0) {
      unsigned char* st = ring + (size_t)s * stage_bytes;
      const uint32_t kaddr = smem_u32(st);
      const uint32_t caddr = smem_u32(st + k_bytes);
      if (valid < kTile) {
        // rows past the valid tokens hold stale bits: zero them (0 * NaN would poison O)
        for (int x = lane; x < (kTile - valid) * R / 8; x += 32)
          reinterpret_cast<uint4*>(st + k_bytes)[valid * R / 8 + x] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
      }
      // S^T = Q K^T, k-steps split over two accumulator chains
      float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float sb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int tok = (mi >> 1) * 8 + rr;
        const uint32_t rowaddr = kaddr + (uint32_t)(tok * D * 2);
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          const int chunk = 2 * s2 + (mi & 1);
          uint32_t kb[4];
          ldsm4(kb, rowaddr + (uint32_t)((chunk ^ (tok & mk)) << 4));
          if (s2 & 1) {
            mma16816(sb[0], qa[s2][0], qa[s2][1], kb[0], kb[1]);
            mma16816(sb[1], qa[s2][0], qa[s2][1], kb[2], kb[3]);
          } else {
            mma16816(sa[0], qa[s2][0], qa[s2][1], kb[0], kb[1]);
            mma16816(sa[1], qa[s2][0], qa[s2][1], kb[2], kb[3]);
          }
        }
      }
      // online softmax on row gr (this lane holds tokens 2tq, 2tq+1, 8+2tq, 9+2tq)
      const bool row_on = head_ok && ((mt >> gr) & 1u);
      float sv[4];
      sv[0] = (row_on && 2 * tq < valid) ? (sa[0][0] + sb[0][0]) * p.qscale : -INFINITY;
      sv[1] = (row_on && 2 * tq + 1 < valid) ? (sa[0][1] + sb[0][1]) * p.qscale : -INFINITY;
      sv[2] = (row_on && 8 + 2 * tq < valid) ? (sa[1][0] + sb[1][0]) * p.qscale : -INFINITY;
      sv[3] = (row_on && 9 + 2 * tq < valid) ? (sa[1][1] + sb[1][1]) * p.qscale : -INFINITY;
      float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      float pr[4], corr = 1.f;
      if (m_new == -INFINITY) {
        pr[0] = pr[1] = pr[2] = pr[3] = 0.f;
      } else {
        corr = exp2f(m_run - m_new);
#pragma unroll
        for (int x = 0; x < 4; ++x) pr[x] = exp2f(sv[x] - m_new);
      }
      l_run = l_run * corr + (pr[0] + pr[1] + pr[2] + pr[3]);
      m_run = m_new;
#pragma unroll
      for (int jj = 0; jj < NT; ++jj) {
        oacc[jj][0] *= corr;
        oacc[jj][1] *= corr;
      }
      // O += P C
      const uint32_t pa0 = pack_bf16(pr[0], pr[1]), pa2 = pack_bf16(pr[2], pr[3]);
      {
        const int tok = (mi & 1) * 8 + rr;
        const uint32_t rowaddr = caddr + (uint32_t)(tok * R * 2);
#pragma unroll
        for (int jj = 0; jj < NT / 2; ++jj) {
          const int chunk = 2 * jj + (mi >> 1);
          uint32_t cb4[4];
          ldsm4t(cb4, rowaddr + (uint32_t)((chunk ^ (tok & mc)) << 4));
          mma16816(oacc[2 * jj], pa0, pa2, cb4[0], cb4[1]);
          mma16816(oacc[2 * jj + 1], pa0, pa2, cb4[2], cb4[3]);
        }
      }
    }
    __syncwarp();  // every lane is done with slot s (and read meta[s])
    // refill this slot with tile i + SW; a tile's descriptor is read from the lane
    // registers only when it is issued, so reloading the next 32 here is safe
    const int nx = i + SW;
    if (nx < my_tiles) {
      if ((nx & 31) == 0) load_desc(nx);
      issue(nx);
    }
  }
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  if (!ok) set_err(p.err, BASISKV_DEVERR_TIMEOUT);

  // merge the warps: each warp's (max, sum, acc[R]) per head -> one split result
  constexpr int kOut = 2 + R;
  float* mb = reinterpret_cast<float*>(smem);  // [kMmaWarps][G][kOut], reuses the rings
  __syncthreads();
  if (gr < G) {
    float* dst = mb + ((size_t)w * G + gr) * kOut;
    if (tq == 0) {
      dst[0] = m_run;
      dst[1] = l_run;
    }
#pragma unroll
    for (int jj = 0; jj < NT; ++jj) {
      dst[2 + 8 * jj + 2 * tq] = oacc[jj][0];
      dst[3 + 8 * jj + 2 * tq] = oacc[jj][1];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * R; idx += blockDim.x) {
    const int hi = idx / R, dim = idx - hi * R;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kMmaWarps; ++ww) M = fmaxf(M, mb[((size_t)ww * G + hi) * kOut]);
    float Ls = 0.f, As = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < kMmaWarps; ++ww) {
        const float* src = mb + ((size_t)ww * G + hi) * kOut;
        const float f = exp2f(src[0] - M);  // 0 for a warp that saw nothing of this head
        Ls += src[1] * f;
        As += src[2 + dim] * f;
      }
    }
    float* out = p.part + (((size_t)b * p.Hq + (size_t)g * G + hi) * p.nsplit + split) * (R + 2);
    out[2 + dim] = As;
    if (dim == 0) {
      out[0] = M;
      out[1] = Ls;
    }
  }
  if (!last_of_group(p, bg, nsplit_active, &s_last)) return;
  merge_group_splits(p, b, g, G, R, nsplit_active, w, kMmaWarps, lane);
  if (threadIdx.x == 0) p.cnt[bg] = 0;
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
// The attention kernels launch as programmatic dependents of the selection
// kernel before them on the stream: their CTAs may start while it finishes and
// wait (grid_dep_wait) before reading anything.
template <typename K>
static cudaError_t launch_dependent_of_route(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                            const AttnParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

size_t attn_smem_bytes(int d, int r, int esize, int max_pages, int eps) {
  const size_t stage = ((size_t)kTile * (d + r) * esize + 127) & ~(size_t)127;
  return attn_ent_offset((size_t)kStages * stage + 2 * kStages * 8, max_pages) + (size_t)eps * 4;
}

template <typename T, int D, int G, int CU>
static cudaError_t launch_attn_t(const AttnParams& p, int batch, cudaStream_t st) {
  const size_t smem = attn_smem_bytes(D, p.r, sizeof(T), p.max_pages, p.eps);
  cudaError_t e = ensure_smem((const void*)attn_kernel<T, D, G, CU>, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent_of_route(attn_kernel<T, D, G, CU>, dim3(p.nsplit, p.Hkv, batch), dim3(32 * (G + 1)),
                                   smem, st, p);
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

template <int D, int G, int NT>
static cudaError_t launch_mma_t(const AttnParams& p, int batch, cudaStream_t st) {
  const size_t stage = ((size_t)kTile * (D + NT * 8) * 2 + 127) & ~(size_t)127;
  const size_t smem = attn_ent_offset((size_t)kMmaWarps * kMmaWarpStages * (stage + 8), p.max_pages) + (size_t)p.eps * 4;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem((const void*)attn_mma_kernel<D, G, NT>, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent_of_route(attn_mma_kernel<D, G, NT>, dim3(p.nsplit, p.Hkv, batch), dim3(32 * kMmaWarps),
                                   smem, st, p);
}

template <int D, int G>
static cudaError_t launch_mma_r(const AttnParams& p, int batch, cudaStream_t st) {
  switch (p.r / 8) {
    case 2: return launch_mma_t<D, G, 2>(p, batch, st);
    case 4: return launch_mma_t<D, G, 4>(p, batch, st);
    case 6: return launch_mma_t<D, G, 6>(p, batch, st);
    case 8: return launch_mma_t<D, G, 8>(p, batch, st);
    case 10: return launch_mma_t<D, G, 10>(p, batch, st);
    case 12: return launch_mma_t<D, G, 12>(p, batch, st);
    case 14: return launch_mma_t<D, G, 14>(p, batch, st);
    case 16: return launch_mma_t<D, G, 16>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static cudaError_t launch_mma_g(const AttnParams& p, int G, int batch, cudaStream_t st) {
  switch (G) {
    case 1: return launch_mma_r<D, 1>(p, batch, st);
    case 2: return launch_mma_r<D, 2>(p, batch, st);
    case 4: return launch_mma_r<D, 4>(p, batch, st);
    case 8: return launch_mma_r<D, 8>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_attn(const DecodePlan& pl, const DecodeArgs& a, void* scratch, int batch,
                               cudaStream_t st) {
  char* base = static_cast<char*>(scratch);
  int32_t* cnt = reinterpret_cast<int32_t*>(base + pl.cnt_off);
  float* part = reinterpret_cast<float*>(base + pl.part_off);
  AttnParams ap{a.q, a.k_raw, a.c_lat, a.block_table, a.seq_len, a.sel, a.sel_cnt, cnt, part, a.o_lat, a.err,
                a.Hq, a.Hkv, a.page, a.r, a.max_pages, a.num_phys, a.top_k, pl.umax, pl.tpp, pl.eps, pl.nsplit,
                pl.nsplit_lo, pl.rich_from, (float)(1.4426950408889634 / sqrt((double)a.d))};
  cudaError_t e;
  const int G = a.Hq / a.Hkv;
  (void)e;
  if (kc_swizzled(a.bf16, a.d, a.r))
    return (a.d == 128) ? launch_mma_g<128>(ap, G, batch, st) : launch_mma_g<64>(ap, G, batch, st);
  if (a.bf16)
    return (a.d == 128) ? launch_attn_g<__nv_bfloat16, 128>(ap, G, batch, st)
                        : launch_attn_g<__nv_bfloat16, 64>(ap, G, batch, st);
  return (a.d == 128) ? launch_attn_g<float, 128>(ap, G, batch, st) : launch_attn_g<float, 64>(ap, G, batch, st);
}

}  // namespace bkv
