// Step 4 of the BasisKV decode step: exact attention on the routed pages.
//
// Only the selected key pages are read back, and the QK scores on them are
// exact (BasisKV abstract; kongchang.com explainer, section
// "用Value潜变量辅助Key路由"); the attention formula is the textbook one
// (machinelearning.ru "KV-кэширование", section "Математическая формализация"),
// restricted to the selected tokens, with the weights applied to the rank-r
// Value latents instead of full-width values.
//
// The pages of a (sequence, KV head) group come as a union list (union.cuh):
// every page chosen by any of the group's G query heads, once, with a head
// mask and its physical id resolved.  The routing kernel writes the lists;
// when the caller passes its own selection, union_kernel builds them from it.
// One launch then streams the lists in one resident wave of CTAs: every group
// gets one CTA and the remaining CTAs are shared out in proportion to the
// groups' tiles (assign_cta), so every split holds about the same number of
// tiles; split s of a group takes an equal contiguous share of its list.
// Each split's result per head (max, sum, acc[r]) goes to scratch; the last
// CTA of a group to finish (counted with an atomic) merges the group's splits
// with the log-sum-exp rule and writes o_lat.  Two kernels:
//   * attn_mma_kernel (bf16 with the swizzled K/C layout, the main path): four
//     warps per CTA take the share's 16-token tiles round-robin, each with its
//     own ring of bulk copies (cp.async.bulk, mbarrier completion, bounded
//     waits), and run all G heads of the group on the tensor cores
//     (mma.sync m16n8k16); the warps' states are folded in warp order.
//     The split of the work depends only on the union sizes, so the output is
//     reproducible.
//   * attn_kernel (fp32 and shapes without the swizzled layout): warp 0
//     produces the share's tiles into a shared ring, warps 1..G consume, one
//     per query head, on the CUDA cores.
// HBM-bound: every byte of the union's pages is read once.
#include "kernels.cuh"
#include "union.cuh"

namespace bkv {

constexpr int kTile = 16;           // tokens per tile
constexpr int kStages = 4;          // ring depth per CTA of the CUDA-core kernel
constexpr int kCoreCtasMax = 6;     // resident CTAs per SM of the CUDA-core attention kernel, at most
constexpr int kMmaCtasPerSm = 3;    // ... and of the tensor-core one (registers)
constexpr int kMmaWarps = 4;        // warps per CTA of the tensor-core kernel
constexpr int kMinSplitTiles = 8;   // tiles per split (full unions), at least
constexpr size_t kSmemPerSm = 228 * 1024;
constexpr size_t kSmemPerCtaReserved = 1024;

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// shared memory of the tensor-core kernel: rings, their barriers, the chunk queue's barriers
static size_t mma_smem_bytes(int d, int r, int slots, int G) {
  const size_t stage = ((size_t)kTile * (d + r) * 2 + 127) & ~(size_t)127;
  (void)G;  // the warps' states reuse the first stage of each ring: G (r + 2) floats fit in a 16-row stage
  return (size_t)kMmaWarps * slots * (stage + 8);
}
// ... and of the CUDA-core kernel: ring and full / empty barriers
static size_t core_smem_bytes(int d, int r, int esize) {
  const size_t stage = ((size_t)kTile * (d + r) * esize + 127) & ~(size_t)127;
  return (size_t)kStages * stage + 2 * kStages * 8;
}

// ---------------------------------------------------------------------------
// plan: splits per (sequence, KV head) and the scratch layout
// ---------------------------------------------------------------------------
// Both kernels: one CTA per group at least, up to one resident wave (more
// waves when there are more than half as many groups as resident CTAs); the
// CTAs past one per group are shared out among the groups in proportion to
// their tiles when the kernel runs (assign_cta), each split keeping at least
// kMinSplitTiles tiles of a full union.  Each CTA writes one partial result.
DecodePlan decode_plan(int Hq, int Hkv, int page, int r, int top_k, int batch, int max_pages, bool bf16, int d,
                       int num_sms) {
  DecodePlan pl{};
  const int G = Hq / Hkv;
  long long um = (long long)G * (top_k + 2);
  if (um > max_pages) um = max_pages;
  pl.umax = (int)um;
  pl.tpp = page / kTile;
  pl.ustride = union_stride_words(pl.umax);
  int per_sm;
  if (kc_swizzled(bf16, d, r)) {
    // three slots per warp where three CTAs fit, else two
    pl.ring_slots = 3;
    if (kMmaCtasPerSm * (mma_smem_bytes(d, r, 3, G) + kSmemPerCtaReserved) > kSmemPerSm) pl.ring_slots = 2;
    per_sm = (int)(kSmemPerSm / (mma_smem_bytes(d, r, pl.ring_slots, G) + kSmemPerCtaReserved));
    if (per_sm > kMmaCtasPerSm) per_sm = kMmaCtasPerSm;
  } else {
    pl.ring_slots = 0;
    per_sm = (int)(kSmemPerSm / (core_smem_bytes(d, r, bf16 ? 2 : 4) + kSmemPerCtaReserved));
    if (per_sm > kCoreCtasMax) per_sm = kCoreCtasMax;
  }
  if (per_sm < 1) per_sm = 1;
  const long long slots = (long long)num_sms * per_sm;
  const long long groups = (long long)batch * Hkv;
  long long per_group = ((long long)pl.umax * pl.tpp + kMinSplitTiles - 1) / kMinSplitTiles;
  if (per_group < 1) per_group = 1;
  // one resident wave, or more when there are many groups: with at least two
  // CTAs per group on average the larger groups still get several, and the
  // later waves start wherever an SM frees up
  const long long waves = std::max(1LL, (2 * groups + slots - 1) / slots);
  long long grid = std::min(waves * slots, groups * per_group);
  if (grid < groups) grid = groups;
  pl.grid = (int)grid;
  pl.extra = (int)(grid - groups);
  size_t off = 0;
  pl.list_off = off;
  off += up256((size_t)batch * Hkv * pl.ustride * 4);
  pl.ucount_off = off;
  off += up256((size_t)batch * Hkv * 4);
  pl.cnt_off = off;  // per group: finished splits
  off += up256((size_t)batch * Hkv * 4);
  pl.part_off = off;  // one partial result per CTA
  off += up256((size_t)pl.grid * G * (r + 2) * 4);
  pl.bytes = off;
  return pl;
}

// Which group CTA c works on.  Group g (in b * Hkv + g order) has t_g = U_g *
// tpp tiles, P_g tiles before it and T in all; it gets the CTAs [c_g,
// c_{g+1}) with c_g = g + floor(extra * P_g / T): at least one, the rest in
// proportion to its tiles, grid = groups + extra CTAs in all.  All threads call
// this (each scans a contiguous run of groups, read twice from L2); the result
// lands in s_asg[4] = {group, split, splits, first CTA of the group}.
__device__ __forceinline__ void assign_cta(const AttnParams& p, int c, int* warp_tot, int* s_asg) {
  const int tid = threadIdx.x, nthr = blockDim.x, NG = p.ngroups;
  auto tiles = [&](int g) { return (int)min(__ldcg(p.ucount + g), (uint32_t)p.umax) * p.tpp; };
  const int per = (NG + nthr - 1) / nthr;
  const int g0 = min(NG, tid * per), g1 = min(NG, g0 + per);
  int local = 0;
  for (int g = g0; g < g1; ++g) local += tiles(g);
  int T;
  long long P = block_exclusive_scan(local, warp_tot, T);
  for (int g = g0; g < g1; ++g) {
    const long long pn = P + tiles(g);
    const int cg = g + (int)(T > 0 ? ((long long)p.extra * P) / T : 0);
    const int cn = g + 1 + (int)(T > 0 ? ((long long)p.extra * pn) / T : (g + 1 == NG ? p.extra : 0));
    if (c >= cg && c < cn) {
      s_asg[0] = g;
      s_asg[1] = c - cg;
      s_asg[2] = cn - cg;
      s_asg[3] = cg;
      s_asg[4] = (int)min(__ldcg(p.ucount + g), (uint32_t)p.umax);  // the group's union entries
    }
    P = pn;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// union lists from a given selection
// ---------------------------------------------------------------------------
// One CTA per (KV head, sequence): the G heads' selections are OR-ed into one
// byte of head bits per page (shared memory), then write_union_list stores the
// ascending list.  A selected page outside [0, n) sets
// BASISKV_DEVERR_SELECTION and is dropped.
constexpr int kUnionThreads = 256;

__global__ void __launch_bounds__(kUnionThreads) union_kernel(UnionParams u) {
  extern __shared__ __align__(16) uint32_t masks[];  // ceil(max_pages / 4) words
  __shared__ int warp_tot[32];
  grid_dep_wait();      // the selection may come from the kernel before this one
  allow_dependents();   // the attention kernel may launch; it waits for this grid
  const int g = blockIdx.x, b = blockIdx.y;
  union_from_selection(u.sel, u.sel_cnt, u.block_table, u.seq_len[b], b, g, u.Hq, u.Hkv, u.page, u.max_pages,
                       u.num_phys, u.top_k, u.lists + ((size_t)b * u.Hkv + g) * u.ustride,
                       u.ucount + (size_t)b * u.Hkv + g, u.acnt, (size_t)gridDim.y * u.Hkv, u.err, masks,
                       nullptr, warp_tot);
}

cudaError_t launch_union(const UnionParams& u, int batch, cudaStream_t st) {
  const size_t smem = (size_t)((u.max_pages + 3) / 4) * 4;
  cudaError_t e = ensure_smem((const void*)union_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(u.Hkv, batch);
  cfg.blockDim = dim3(kUnionThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, union_kernel, u);
}

// After writing its split results, a CTA counts itself on the group's counter;
// the last one of the group merges.  The merging CTA puts the counter (and the
// group's tile cursor) back to zero, so both are zero between calls.
// The barrier orders every thread's split results before thread 0's release
// fence and atomic; the last CTA's thread 0 fences again (acquire) before the
// barrier that lets its threads read the other CTAs' results.
__device__ __forceinline__ bool last_of_group(const AttnParams& p, size_t bg, int nsplit_active, int* s_last) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&p.cnt[bg], 1);
    if (prev >= nsplit_active) set_err(p.err, BASISKV_DEVERR_WORKSPACE);
    *s_last = (prev == nsplit_active - 1);
    if (*s_last) __threadfence();
  }
  __syncthreads();
  return *s_last != 0;
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
// results: for each of its G heads, log-sum-exp over the splits, whose
// partials sit in the slots of the group's CTAs (slot0 .. slot0 + ns - 1).
// Heads are spread over `nw` warps starting at warp index `wi`; a warp issues
// the loads of up to eight splits (max, sum and its lanes' dimensions) before
// it uses any.
__device__ __forceinline__ void merge_group_splits(const AttnParams& p, int b, int g, int G, int r, int slot0,
                                                   int ns, int wi, int nw, int lane) {
  constexpr int kDimIt = 4;  // r <= 128: dims lane + 32 k
  constexpr int kBatch = 8;  // splits whose values are loaded together
  const int stride = r + 2;
  for (int hi = wi; hi < G; hi += nw) {
    const int h = g * G + hi;
    const float* base = p.part + ((size_t)slot0 * G + hi) * stride;
    const size_t sstride = (size_t)G * stride;  // between consecutive CTAs' slots
    float M = -INFINITY, Ls = 0.f;
    float acc[kDimIt] = {0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < ns; s0 += kBatch) {
      const int cn = min(kBatch, ns - s0);
      // lane j < cn: max and sum of split s0 + j; every lane: its dims of every split
      float mj = -INFINITY, lj = 0.f;
      if (lane < cn) {
        mj = __ldcg(base + (size_t)(s0 + lane) * sstride);
        lj = __ldcg(base + (size_t)(s0 + lane) * sstride + 1);
      }
      float x[kBatch][kDimIt];
#pragma unroll
      for (int j = 0; j < kBatch; ++j)
#pragma unroll
        for (int k = 0; k < kDimIt; ++k) {
          const int dim = lane + 32 * k;
          x[j][k] = (j < cn && dim < r) ? __ldcg(base + (size_t)(s0 + j) * sstride + 2 + dim) : 0.f;
        }
      const float Mn = fmaxf(M, warp_max(mj));
      if (Mn != -INFINITY) {
        const float cf = (M == -INFINITY) ? 0.f : exp2f(M - Mn);  // rescale what the earlier batches summed
        Ls *= cf;
#pragma unroll
        for (int k = 0; k < kDimIt; ++k) acc[k] *= cf;
        const float wl = (mj == -INFINITY) ? 0.f : exp2f(mj - Mn);
        Ls += warp_sum(lj * wl);
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const float wt = __shfl_sync(kFull, wl, j);
#pragma unroll
          for (int k = 0; k < kDimIt; ++k) acc[k] = fmaf(x[j][k], wt, acc[k]);
        }
        M = Mn;
      }
    }
#pragma unroll
    for (int k = 0; k < kDimIt; ++k) {
      const int dim = lane + 32 * k;
      if (dim < r) p.o_lat[((size_t)b * p.Hq + h) * r + dim] = (Ls > 0.f) ? acc[k] / Ls : 0.f;
    }
  }
}

// Wait (bounded) for the bulk copies a timed-out ring may still have in flight:
// the full barrier of every tile in [from, to) in a ring of `slots` stages.
// Returns false if one of them also gives up.
__device__ __forceinline__ bool drain_ring(uint64_t* full, int slots, int from, int to) {
  bool ok = true;
  for (int t = from; t < to; ++t) ok = mbar_wait_bounded(&full[t % slots], (uint32_t)((t / slots) & 1)) && ok;
  return ok;
}

template <typename T, int D, int G, int CU>
__global__ void __launch_bounds__(32 * (G + 1)) attn_kernel(AttnParams p) {
  constexpr int DPL = D / 32;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t meta[kStages];  // head mask | valid tokens << 8 of the tile in each stage
  __shared__ int s_last, s_fail, s_issued, s_consumed;
  __shared__ int warp_tot[32];
  __shared__ int s_asg[5];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = p.r;
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
    s_fail = 0;
    s_issued = 0;
    s_consumed = 0;
  }
  __syncthreads();
  grid_dep_wait();     // the union lists are complete (this kernel may launch before their writer ends)
  allow_dependents();  // the out-projection may launch and start streaming its weights
  assign_cta(p, blockIdx.x, warp_tot, s_asg);
  const int bg = s_asg[0], split = s_asg[1], ns = s_asg[2], slot0 = s_asg[3];
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  // the query row of a consumer warp
  float qf[DPL];
  if (warp >= 1) {
    const T* qr = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G + warp - 1) * D + lane * DPL;
#pragma unroll
    for (int u = 0; u < DPL; ++u) qf[u] = Elem<T>::to_f(qr[u]) * p.qscale;
  }

  const uint32_t* list = p.lists + (size_t)bg * p.ustride;
  const int U = s_asg[4];  // list[0], as the compact count array holds it
  const int eps = (U + ns - 1) / ns;
  const int e0 = split * eps;
  const int nent = max(0, min(U, e0 + eps) - e0);
  const int ntiles = nent * p.tpp;

  bool ok = true;
  if (warp == 0) {
    // ---------------- producer ----------------
    const T* kbase = static_cast<const T*>(p.k_raw);
    const T* cbase = static_cast<const T*>(p.c_lat);
    int t = 0;
    for (int cb = 0; cb < nent && ok; cb += 32) {
      // lane e holds entry e0 + cb + e of the list
      uint32_t my_en = kNoPage;
      int my_valid = 0;
      if (cb + lane < nent) {
        const int e = e0 + cb + lane;
        my_en = __ldcg(list + 4 + e);
        my_valid = (e == U - 1) ? (int)__ldcg(list + 1) : p.page;
      }
      const int t_end = min(nent, cb + 32) * p.tpp;
      for (; t < t_end; ++t) {
        const int el = t / p.tpp - cb, sub = t - (t / p.tpp) * p.tpp;
        const uint32_t en = __shfl_sync(kFull, my_en, el);
        const int pv = __shfl_sync(kFull, my_valid, el);
        const uint32_t id = en & kNoPage;
        if (lane == 0 && id != kNoPage && id >= (uint32_t)p.num_phys) set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
        const int valid = (id < (uint32_t)p.num_phys) ? min(kTile, max(0, pv - sub * kTile)) : 0;
        const int s = t % kStages;
        // every lane waits; the warp gives up together if any lane's wait expired
        if (t >= kStages && !__all_sync(kFull, mbar_wait_bounded(&empty[s], (uint32_t)(((t / kStages) - 1) & 1)))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          meta[s] = (en >> 24) | ((uint32_t)valid << 8);
          unsigned char* st = smem + (size_t)s * stage_bytes;
          fence_proxy_async_smem();
          if (valid > 0) {
            const size_t row0 = ((size_t)id * p.Hkv + g) * p.page + (size_t)sub * kTile;
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
    if (lane == 0) s_issued = t;
  } else {
    // ---------------- consumer: one query head ----------------
    const int hi = warp - 1;
    const int h = g * G + hi;
    float m_run = -INFINITY, l_run = 0.f;
    float acc[CU][2];
#pragma unroll
    for (int u = 0; u < CU; ++u) acc[u][0] = acc[u][1] = 0.f;
    int t = 0;
    for (; t < ntiles; ++t) {
      const int s = t % kStages;
      if (!__all_sync(kFull, mbar_wait_bounded(&full[s], (uint32_t)((t / kStages) & 1)))) {
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
    if (lane == 0) atomicMax(&s_consumed, t);
    // this head's result for the split
    const float lsum = warp_sum(l_run);
    float* out = p.part + ((size_t)blockIdx.x * G + hi) * (r + 2);
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
  if (!ok) s_fail = 1;
  __syncthreads();
  if (s_fail) {
    // a wait gave up: let the copies still in flight land before the CTA's
    // shared memory is released, and mark the split's result
    if (threadIdx.x == 0) {
      set_err(p.err, BASISKV_DEVERR_TIMEOUT);
      drain_ring(full, kStages, s_consumed, s_issued);
    }
    if (warp >= 1 && lane == 0) {
      float* out = p.part + ((size_t)blockIdx.x * G + warp - 1) * (r + 2);
      out[0] = 0.f;                          // the merge weighs this split's sum ...
      out[1] = __int_as_float(0x7fc00000);   // ... which is NaN: the head's output becomes NaN
    }
  }

  // the last CTA of the group to finish merges every split of its G heads
  if (!last_of_group(p, bg, ns, &s_last)) return;
  if (warp >= 1) merge_group_splits(p, b, g, G, r, slot0, ns, warp - 1, G, lane);
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

// Work of the tensor-core kernel: one resident wave of CTAs, each on one
// group.  Every group gets one CTA and the remaining CTAs are shared out in
// proportion to the groups' tiles (assign_cta, the same rule as the CUDA-core
// kernel), so the splits of all groups hold about the same number of tiles;
// split s of a group's ns takes an equal contiguous share of the group's
// union list.  The four warps take the share's tiles round-robin, each with
// its own ring of 1-D bulk copies (mbarrier completion, bounded waits), and
// run all G heads of the group on the tensor cores
// (mma.sync m16n8k16).  At the end the warps' states are folded in warp order
// into the CTA's partial result; the last CTA of the group merges the
// group's partials into o_lat.  The split of the work depends only on the
// union sizes, so the output is reproducible.
template <int D, int G, int NT, int SW>
__global__ void __launch_bounds__(32 * kMmaWarps, kMmaCtasPerSm) attn_mma_kernel(AttnParams p) {
  constexpr int KS = D / 16;
  constexpr int R = NT * 8;
  constexpr int kOut = 2 + R;
  constexpr uint32_t k_bytes = kTile * D * 2;
  constexpr uint32_t c_bytes = kTile * R * 2;
  constexpr uint32_t stage_bytes = (k_bytes + c_bytes + 127u) & ~127u;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t meta_all[kMmaWarps][SW];  // head mask | valid tokens << 8 of each slot's tile
  __shared__ int warp_tot[32];
  __shared__ int s_asg[5];
  __shared__ int s_last, s_fail;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t* meta = meta_all[w];
  // shared memory: [rings | ring barriers]
  unsigned char* ring = smem + (size_t)w * SW * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kMmaWarps * SW * stage_bytes) + w * SW;
  if (lane == 0) {
    for (int s = 0; s < SW; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) s_fail = 0;
  __syncthreads();
  grid_dep_wait();     // the union lists are complete (this kernel may launch before their writer ends)
  allow_dependents();  // the out-projection may launch and start streaming its weights
  assign_cta(p, blockIdx.x, warp_tot, s_asg);
  const int bg = s_asg[0], split = s_asg[1], ns = s_asg[2], slot0 = s_asg[3];
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  const uint32_t* list = p.lists + (size_t)bg * p.ustride;
  const int U = s_asg[4];  // list[0], as the compact count array holds it
  const int T = U * p.tpp;
  const int per = (T + ns - 1) / ns;
  const int lo = min(T, split * per), hi = min(T, lo + per);
  const int my_tiles = (hi - lo > w) ? (hi - lo - w + kMmaWarps - 1) / kMmaWarps : 0;  // tiles lo + w + 4k

  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.k_raw);
  const __nv_bfloat16* cbase = static_cast<const __nv_bfloat16*>(p.c_lat);
  const uint64_t stream_pol = l2_evict_first();

  // descriptors of this warp's tiles, 32 at a time (lane j: the batch's tile j):
  // the physical page (kNoPage: nothing to read), head mask | valid tokens << 8 | 16-row block << 16
  uint32_t d_id = kNoPage, d_meta = 0;
  auto load_desc = [&](int k0) {
    const int k = k0 + lane;
    d_id = kNoPage;
    d_meta = 0;
    if (k < my_tiles) {
      const int t = lo + w + kMmaWarps * k;
      const int e = t / p.tpp, sub = t - e * p.tpp;
      const uint32_t en = __ldcg(list + 4 + e);
      const int pv = (e == U - 1) ? (int)__ldcg(list + 1) : p.page;
      const uint32_t id = en & kNoPage;
      if (id != kNoPage && id >= (uint32_t)p.num_phys) set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
      const int valid = (id < (uint32_t)p.num_phys) ? min(kTile, max(0, pv - sub * kTile)) : 0;
      d_id = valid > 0 ? id : kNoPage;
      d_meta = (en >> 24) | ((uint32_t)valid << 8) | ((uint32_t)sub << 16);
    }
  };
  // issue the warp's tile i into slot i % SW (lane 0 copies; all lanes shuffle)
  auto issue = [&](int i) {
    const int j = i & 31;
    const uint32_t id = __shfl_sync(kFull, d_id, j);
    const uint32_t mt = __shfl_sync(kFull, d_meta, j);
    if (lane == 0) {
      meta[i % SW] = (id == kNoPage) ? (mt & 0xffu) : (mt & 0xffffu);
      uint64_t* bar = &full[i % SW];
      unsigned char* st = ring + (size_t)(i % SW) * stage_bytes;
      fence_proxy_async_smem();
      if (id != kNoPage) {
        const int sub = (int)(mt >> 16);
        const size_t row0 = ((size_t)id * p.Hkv + (size_t)g) * p.page + (size_t)sub * kTile;
        mbar_arrive_expect_tx(bar, k_bytes + c_bytes);
        bulk_g2s_hint(st, kbase + row0 * D, k_bytes, bar, stream_pol);  // read once: evict first
        bulk_g2s_hint(st + k_bytes, cbase + row0 * R, c_bytes, bar, stream_pol);
      } else {
        mbar_arrive_expect_tx(bar, 0);
      }
    }
  };

  // the warp's running state (heads as fragment rows) and the group's query
  const int gr = lane >> 2, tq = lane & 3;  // fragment row (head) and column pair
  const bool head_ok = gr < G;
  float m_run = -INFINITY, l_run = 0.f;
  float oacc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
  uint32_t qa[KS][2];
  {
    const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G + gr) * D;
#pragma unroll
    for (int s2 = 0; s2 < KS; ++s2) {
      qa[s2][0] = head_ok ? *reinterpret_cast<const uint32_t*>(qr + 16 * s2 + 2 * tq) : 0u;
      qa[s2][1] = head_ok ? *reinterpret_cast<const uint32_t*>(qr + 16 * s2 + 2 * tq + 8) : 0u;
    }
  }

  constexpr int mk = 7;  // K rows have 8 or 16 chunks
  const int mc = swz_mask(R);
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix mi takes its row rr from this lane
  bool ok = true;
  int issued = 0, consumed = 0;
  if (my_tiles > 0) load_desc(0);
  while (issued < SW && issued < my_tiles) {
    issue(issued);
    ++issued;
  }
  while (consumed < my_tiles) {
    const int s = consumed % SW;
    if (!__all_sync(kFull, mbar_wait_bounded(&full[s], (uint32_t)((consumed / SW) & 1)))) {
      ok = false;  // the whole warp gives up together
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
    __syncwarp();  // every lane is done with slot s (and has read meta[s])
    ++consumed;
    // refill the slot just consumed (the next batch of descriptors replaces the
    // lane registers only once every tile of this batch has been issued)
    if (issued < my_tiles) {
      if ((issued & 31) == 0) load_desc(issued);
      issue(issued);
      ++issued;
    }
  }
  if (!ok) {
    // a wait gave up: let this warp's copies still in flight land before its
    // ring is released, and mark the CTA's result
    if (lane == 0) {
      s_fail = 1;
      set_err(p.err, BASISKV_DEVERR_TIMEOUT);
      drain_ring(full, SW, consumed, issued);
    }
    __syncwarp();
  }
  // The warps' states, each [G][kOut] = (max, sum, o) per head, go to the
  // first stage of the warp's own ring (free once its loop is done); then
  // every thread combines the four warps' values of its elements in warp
  // order (a fixed order, so the result does not depend on timing) into the
  // CTA's slot.  After a timed-out wait a ring may still be receiving copies:
  // it is not touched and the slot marks the heads' outputs NaN.
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  __syncthreads();  // s_fail is final
  const bool failed = s_fail != 0;
  if (!failed && head_ok) {
    float* row = reinterpret_cast<float*>(ring) + gr * kOut;
    if (tq == 0) {
      row[0] = m_run;
      row[1] = l_run;
    }
#pragma unroll
    for (int jj = 0; jj < NT; ++jj) {
      row[2 + 8 * jj + 2 * tq] = oacc[jj][0];
      row[3 + 8 * jj + 2 * tq] = oacc[jj][1];
    }
  }
  __syncthreads();
  float* slot = p.part + (size_t)blockIdx.x * G * kOut;  // the group's CTAs, and slots, are consecutive
  for (int i = threadIdx.x; i < G * kOut; i += blockDim.x) {
    const int hh = i / kOut, col = i - hh * kOut;
    float v = (col == 1) ? __int_as_float(0x7fc00000) : 0.f;  // a wait gave up: the head's output is NaN
    if (!failed) {
      float mw[kMmaWarps], M = -INFINITY;
#pragma unroll
      for (int ww = 0; ww < kMmaWarps; ++ww) {
        mw[ww] = reinterpret_cast<const float*>(smem + (size_t)ww * SW * stage_bytes)[hh * kOut];
        M = fmaxf(M, mw[ww]);
      }
      if (col == 0) {
        v = M;
      } else {
        v = 0.f;
#pragma unroll
        for (int ww = 0; ww < kMmaWarps; ++ww) {
          const float s = (mw[ww] == -INFINITY) ? 0.f : exp2f(mw[ww] - M);
          v = fmaf(reinterpret_cast<const float*>(smem + (size_t)ww * SW * stage_bytes)[i], s, v);
        }
      }
    }
    slot[i] = v;
  }
  // the last CTA of the group to finish merges every split of its G heads
  if (!last_of_group(p, (size_t)bg, ns, &s_last)) return;
  merge_group_splits(p, b, g, G, R, slot0, ns, w, kMmaWarps, lane);
  if (threadIdx.x == 0) p.cnt[bg] = 0;
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
// The attention kernels launch as programmatic dependents of the kernel that
// writes the union lists: their CTAs may start while it finishes and wait
// (grid_dep_wait) before reading them.
template <typename K>
static cudaError_t launch_dependent(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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

template <typename T, int D, int G, int CU>
static cudaError_t launch_attn_t(const AttnParams& p, int grid, cudaStream_t st) {
  const size_t smem = core_smem_bytes(D, p.r, sizeof(T));
  cudaError_t e = ensure_smem((const void*)attn_kernel<T, D, G, CU>, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(attn_kernel<T, D, G, CU>, dim3(grid), dim3(32 * (G + 1)), smem, st, p);
}

template <typename T, int D, int G>
static cudaError_t launch_attn_r(const AttnParams& p, int grid, cudaStream_t st) {
  return (p.r <= 64) ? launch_attn_t<T, D, G, 1>(p, grid, st) : launch_attn_t<T, D, G, 2>(p, grid, st);
}

template <typename T, int D>
static cudaError_t launch_attn_g(const AttnParams& p, int G, int grid, cudaStream_t st) {
  switch (G) {
    case 1: return launch_attn_r<T, D, 1>(p, grid, st);
    case 2: return launch_attn_r<T, D, 2>(p, grid, st);
    case 4: return launch_attn_r<T, D, 4>(p, grid, st);
    case 8: return launch_attn_r<T, D, 8>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int G, int NT, int SW>
static cudaError_t launch_mma_t(const AttnParams& p, int grid, cudaStream_t st) {
  const size_t smem = mma_smem_bytes(D, NT * 8, SW, G);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem((const void*)attn_mma_kernel<D, G, NT, SW>, smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(attn_mma_kernel<D, G, NT, SW>, dim3(grid), dim3(32 * kMmaWarps), smem,
                          st, p);
}

template <int D, int G, int NT>
static cudaError_t launch_mma_s(const AttnParams& p, int slots, int grid, cudaStream_t st) {
  return (slots == 2) ? launch_mma_t<D, G, NT, 2>(p, grid, st) : launch_mma_t<D, G, NT, 3>(p, grid, st);
}

template <int D, int G>
static cudaError_t launch_mma_r(const AttnParams& p, int slots, int grid, cudaStream_t st) {
  switch (p.r / 8) {
    case 2: return launch_mma_s<D, G, 2>(p, slots, grid, st);
    case 4: return launch_mma_s<D, G, 4>(p, slots, grid, st);
    case 6: return launch_mma_s<D, G, 6>(p, slots, grid, st);
    case 8: return launch_mma_s<D, G, 8>(p, slots, grid, st);
    case 10: return launch_mma_s<D, G, 10>(p, slots, grid, st);
    case 12: return launch_mma_s<D, G, 12>(p, slots, grid, st);
    case 14: return launch_mma_s<D, G, 14>(p, slots, grid, st);
    case 16: return launch_mma_s<D, G, 16>(p, slots, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static cudaError_t launch_mma_g(const AttnParams& p, int G, int slots, int grid, cudaStream_t st) {
  switch (G) {
    case 1: return launch_mma_r<D, 1>(p, slots, grid, st);
    case 2: return launch_mma_r<D, 2>(p, slots, grid, st);
    case 4: return launch_mma_r<D, 4>(p, slots, grid, st);
    case 8: return launch_mma_r<D, 8>(p, slots, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_attn(const DecodePlan& pl, const DecodeArgs& a, void* scratch, int batch,
                               cudaStream_t st) {
  char* base = static_cast<char*>(scratch);
  AttnParams ap{a.q, a.k_raw, a.c_lat, reinterpret_cast<const uint32_t*>(base + pl.list_off),
                reinterpret_cast<const uint32_t*>(base + pl.ucount_off), reinterpret_cast<int32_t*>(base + pl.cnt_off),
                reinterpret_cast<float*>(base + pl.part_off), a.o_lat, a.err, a.Hq, a.Hkv, a.page, a.r,
                a.num_phys, pl.tpp, batch * a.Hkv, pl.extra, pl.ustride, pl.umax,
                (float)(1.4426950408889634 / sqrt((double)a.d))};
  const int G = a.Hq / a.Hkv;
  if (kc_swizzled(a.bf16, a.d, a.r))
    return (a.d == 128) ? launch_mma_g<128>(ap, G, pl.ring_slots, pl.grid, st)
                        : launch_mma_g<64>(ap, G, pl.ring_slots, pl.grid, st);
  if (a.bf16)
    return (a.d == 128) ? launch_attn_g<__nv_bfloat16, 128>(ap, G, pl.grid, st)
                        : launch_attn_g<__nv_bfloat16, 64>(ap, G, pl.grid, st);
  return (a.d == 128) ? launch_attn_g<float, 128>(ap, G, pl.grid, st)
                      : launch_attn_g<float, 64>(ap, G, pl.grid, st);
}

}  // namespace bkv
