// Step 3 of the BasisKV decode step: key-page routing.
//
// The compressed cache predicts which key pages matter (kongchang.com
// explainer, section "用Value潜变量辅助Key路由"; BasisKV abstract): every page
// keeps its mean predicted key S_p, each query head scores all pages with
// q_h . S_p and keeps the top-k, plus the sink page 0 and the recent page.
//
// Kernel 1 (score) streams the fp32 summaries once; HBM-bound.  Grid (chunk,
// KV head g, sequence b): CTA c scores pages [c * 256, c * 256 + 256) of
// (b, g) for the G query heads of the group, warp w the 32 pages starting at
// c * 256 + w * 32 in four 8-page items: one coalesced block-table load per
// warp; per item one 16-byte summary load per lane and page, the G partial dot
// products against the query rows (held in registers), and one
// transpose-reduction that leaves one (page, head) score per lane.  The
// summary of a page is read once for the whole GQA group.  The grid is one
// resident wave (<= 64 registers, 4 CTAs per SM).
//
// Kernel 2 (select), one CTA per (sequence, query head), exact:
//   * each thread holds the scores of up to KPT consecutive pages as
//     order-preserving 32-bit keys (NaN lowest, -0 == +0) in registers;
//   * T, the k-th largest key of pages 1..n-2, is found bit by bit from the
//     top: a bit is set when at least k keys are >= the prefix with it set (a
//     block-wide count per bit); when exactly k keys are >= the prefix, those
//     k are the answer and there are no ties to break;
//   * pages with key > T are kept, and of the keys equal to T the ones with
//     the lowest page indices; two block scans (ties, kept pages) give every
//     thread its output positions, so sel is written in ascending page order.
// The result is the same as sorting by (score descending, page ascending).
// The G selection CTAs of a KV group run as one thread-block cluster; each
// ORs its kept pages, with its head's bit, into a head mask per page held in
// the shared memory of the cluster's first CTA (distributed shared memory),
// which then writes the group's union list for the attention kernel
// (union.cuh).  Block tables wider than 8192 pages take a histogram selection
// whose last CTA per group (an arrival counter) builds the list instead.
//
// Per-group routing (group_mode 1 / 2): the score kernel folds the G head
// scores of a page, which sit on neighbouring lanes after the transpose
// reduction, into their sum or maximum and writes one row per (sequence, KV
// group); one selection CTA per group ranks it and writes its pages to the
// sel rows of all G heads, so the attention kernel reads k + 2 pages per
// group.
#include "kernels.cuh"
#include "union.cuh"

namespace bkv {

constexpr int kPagesPerWarp = 8;   // pages per warp item of the score kernel
constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kScoreWarpPages = 32;
constexpr int kScoreCtaPages = kScoreWarps * kScoreWarpPages;

// sum (mode 1) or maximum (mode 2) of two head scores; the maximum keeps a NaN
__device__ __forceinline__ float group_fold(float a, float b, int mode) {
  if (mode == 1) return a + b;
  return (a > b || a != a) ? a : b;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kScoreThreads, (G >= 8) ? 2 : 4) route_score_kernel(RouteParams p) {
  constexpr int DPL = D / 32;
  constexpr int N = kPagesPerWarp * G;
  __shared__ __align__(16) float sq[G * D];
  // D = 128: each warp's next item of summary rows lands here (cp.async) while
  // the current item is scored; lane l's 16 bytes of page i at [warp][i][l]
  __shared__ __align__(16) float4 s_next[(DPL == 4) ? kScoreWarps : 1][kPagesPerWarp][32];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Launched as a programmatic dependent of the step's append (see
  // launch_route), this kernel runs beside it: it reads no page the append
  // writes, except with all_pages (the recent page's summary), when it waits
  // for the append first.  The first CTA waits for the append before it ends,
  // so the grid completes after the append and the kernels after it see the
  // append's writes; the other CTAs leave as soon as they are done (a grid of
  // more than one wave keeps its slots turning over).  In an ordinary launch
  // both waits return at once.
  if (p.all_pages) grid_dep_wait();
  // the length, this lane's block-table entry and the query rows are loaded
  // together (the entry is validated once the length is known)
  const int pw0 = c * kScoreCtaPages + warp * kScoreWarpPages;
  const int pl = pw0 + lane;
  const int raw_phys = (pl < p.max_pages) ? p.block_table[(size_t)b * p.max_pages + pl] : -1;
  const int L = p.seq_len[b];
  int n = (L + p.page - 1) / p.page;
  if (n > p.max_pages) {
    if (c == 0 && tid == 0) set_err(p.err, BASISKV_DEVERR_SEQ_LEN);
    n = p.max_pages;
  }
  if (c * kScoreCtaPages >= n) return;  // the whole CTA is past the last page (never the first CTA)
  const size_t qrow = (size_t)b * p.Hq + (size_t)g * G;
  const T* qb = static_cast<const T*>(p.q) + qrow * D;
  for (int i = tid; i < G * D; i += kScoreThreads) sq[i] = Elem<T>::to_f(qb[i]);

  int my_phys = -1;  // -1: not scored, -2: bad block-table entry
  if (pl < n && (p.all_pages || (pl != 0 && pl != n - 1))) {
    my_phys = raw_phys;
    if (my_phys < 0 || my_phys >= p.num_phys) {
      set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
      my_phys = -2;
    }
  }
  __syncthreads();  // sq
  float qf[G][DPL];  // this lane's dimensions of the G query rows
#pragma unroll
  for (int hi = 0; hi < G; ++hi)
#pragma unroll
    for (int u = 0; u < DPL; ++u) qf[hi][u] = sq[hi * D + lane * DPL + u];
  float* outb = p.scores + qrow * p.max_pages;
  float* outg = p.scores + ((size_t)b * p.Hkv + g) * p.max_pages;  // the group's row (group modes)
  // item i0's rows into this warp's s_next slot (zeros for a page not scored)
  auto issue_next = [&](int i0) {
#pragma unroll
    for (int i = 0; i < kPagesPerWarp; ++i) {
      const int ph = __shfl_sync(kFull, my_phys, i0 + i);
      const float* rowp = (ph >= 0) ? p.summary + ((size_t)ph * p.Hkv + g) * D + lane * DPL : p.summary;
      cp_async16_zfill(&s_next[(DPL == 4) ? warp : 0][i][lane], rowp, ph >= 0);
    }
    cp_async_commit_group();
  };
#pragma unroll 1
  for (int i0 = 0; i0 < kScoreWarpPages; i0 += kPagesPerWarp) {
    const int p0 = pw0 + i0;
    if (p0 >= n) break;
    const bool staged = DPL == 4 && i0 > 0;  // this item was prefetched into s_next
    float sv[kPagesPerWarp][DPL];
    if (staged) {
      cp_async_wait_group<0>();
#pragma unroll
      for (int i = 0; i < kPagesPerWarp; ++i) {
        const float4 v = s_next[(DPL == 4) ? warp : 0][i][lane];
        sv[i][0] = v.x; sv[i][1] = v.y;
        if constexpr (DPL == 4) { sv[i][2] = v.z; sv[i][3] = v.w; }
      }
    }
#pragma unroll
    for (int i = 0; i < kPagesPerWarp && !staged; ++i) {
      const int ph = __shfl_sync(kFull, my_phys, i0 + i);
      if (ph >= 0) {
        const float* rowp = p.summary + ((size_t)ph * p.Hkv + g) * D + lane * DPL;
        if constexpr (DPL == 4) {
          const float4 v = __ldcs(reinterpret_cast<const float4*>(rowp));  // read once: evict first
          sv[i][0] = v.x; sv[i][1] = v.y; sv[i][2] = v.z; sv[i][3] = v.w;
        } else {
          const float2 v = __ldcs(reinterpret_cast<const float2*>(rowp));
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
    // the next item's rows start coming in now: the reads of the slot above fed the
    // products just issued, so they are done before the slot is written again
    if (DPL == 4 && i0 + kPagesPerWarp < kScoreWarpPages && p0 + kPagesPerWarp < n) issue_next(i0 + kPagesPerWarp);
    transpose_reduce<N>(part, lane);
    float* out = outb + p0;
    if (p.group_mode != 0) {
      // the G head scores of page i: N <= 32, lanes [i G kDup, (i + 1) G kDup)
      // hold one each (kDup copies); N = 64, lanes [i G / 2, (i + 1) G / 2) two each
      float v;
      int i;
      bool writer;
      if constexpr (N <= 32) {
        constexpr int kDup = 32 / N;
        v = part[0];
#pragma unroll
        for (int o = kDup; o < kDup * G; o <<= 1) v = group_fold(v, __shfl_xor_sync(kFull, v, o), p.group_mode);
        i = lane / (kDup * G);
        writer = lane % (kDup * G) == 0;
      } else {
        v = group_fold(part[0], part[1], p.group_mode);
#pragma unroll
        for (int o = 1; o < G / 2; o <<= 1) v = group_fold(v, __shfl_xor_sync(kFull, v, o), p.group_mode);
        i = lane / (G / 2);
        writer = lane % (G / 2) == 0;
      }
      const int ph = __shfl_sync(kFull, my_phys, i0 + i);
      if (writer && p0 + i < n && ph != -1) outg[p0 + i] = (ph == -2) ? -INFINITY : v;
    } else if constexpr (N <= 32) {
      constexpr int kDup = 32 / N;
      const int idx = lane / kDup;
      const int i = idx / G, hi = idx % G;
      const int ph = __shfl_sync(kFull, my_phys, i0 + i);
      if ((lane % kDup) == 0 && p0 + i < n && ph != -1)
        out[(size_t)hi * p.max_pages + i] = (ph == -2) ? -INFINITY : part[0];
    } else {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = 2 * lane + j;
        const int i = idx / G, hi = idx % G;
        const int ph = __shfl_sync(kFull, my_phys, i0 + i);
        if (p0 + i < n && ph != -1) out[(size_t)hi * p.max_pages + i] = (ph == -2) ? -INFINITY : part[j];
      }
    }
  }
  cp_async_wait_group<0>();  // no copy still landing in shared memory when the CTA ends
  if (c == 0 && g == 0 && b == 0) grid_dep_wait();
}

// ---------------------------------------------------------------------------
// selection with the keys in registers
// ---------------------------------------------------------------------------
constexpr int kSelectThreads = 256;
constexpr int kSelectWarps = kSelectThreads / 32;

// Sum of one int per thread over the block.  `red` is shared scratch of
// 2 * kSelectWarps ints used alternately (`phase` flips it), so one barrier
// per call suffices.
__device__ __forceinline__ int block_total(int v, int* red, int& phase) {
  v = (int)__reduce_add_sync(kFull, (unsigned)v);
  int* slot = red + (phase & 1) * kSelectWarps;
  ++phase;
  if ((threadIdx.x & 31) == 0) slot[threadIdx.x >> 5] = v;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int w = 0; w < kSelectWarps; ++w) t += slot[w];
  return t;
}

// The score row a selection CTA (x = blockIdx.x) ranks and the sel rows it
// writes: its own head's, or the G heads' of its group (contiguous rows).
struct SelRows {
  size_t in, out;
  int copies;
};
__device__ __forceinline__ SelRows sel_rows(const RouteParams& p, int x, int b) {
  if (p.group_mode == 0) {
    const size_t r = (size_t)b * p.Hq + x;
    return {r, r, 1};
  }
  const int G = p.Hq / p.Hkv;
  return {(size_t)b * p.Hkv + x, (size_t)b * p.Hq + (size_t)x * G, G};
}

// sel entry i of every output row of the CTA
__device__ __forceinline__ void put_sel(const RouteParams& p, const SelRows& r, int i, int32_t v) {
  int32_t* out = p.sel + r.out * (p.top_k + 2) + i;
  for (int c = 0; c < r.copies; ++c) out[(size_t)c * (p.top_k + 2)] = v;
}

__device__ __forceinline__ void put_cnt(const RouteParams& p, const SelRows& r, int v) {
  for (int c = 0; c < r.copies; ++c) p.sel_cnt[r.out + c] = v;
}

// After its rows are written, a selection CTA counts itself on its KV group's
// counter; the last of the group's G CTAs (the only one in the per-group
// modes) builds the group's union list for the attention kernel and returns
// the counter to zero.  All threads call this.
__device__ __forceinline__ void select_union_tail(const RouteParams& p, int b, int x, uint32_t* masks,
                                                  int32_t* bt_smem, int* warp_tot, int* s_flag) {
  const int G = p.Hq / p.Hkv;
  const int g = p.group_mode ? x : x / G;
  const int need = p.group_mode ? 1 : G;
  const size_t bg = (size_t)b * p.Hkv + g;
  __syncthreads();  // orders this CTA's sel stores before thread 0's release
  if (threadIdx.x == 0) {
    int last = 1;
    if (need > 1) {
      __threadfence();
      const int prev = atomicAdd(&p.ucnt[bg], 1);
      if (prev >= need) set_err(p.err, BASISKV_DEVERR_WORKSPACE);
      last = prev == need - 1;
      if (last) {
        p.ucnt[bg] = 0;
        __threadfence();  // acquire: the other heads' rows are visible from here on
      }
    }
    *s_flag = last;
  }
  __syncthreads();
  if (!*s_flag) return;
  union_from_selection(p.sel, p.sel_cnt, p.block_table, p.seq_len[b], b, g, p.Hq, p.Hkv, p.page, p.max_pages,
                       p.num_phys, p.top_k, p.lists + bg * p.ustride, p.ucount + bg, p.acnt,
                       (size_t)p.batch * p.Hkv, p.err, masks, bt_smem, warp_tot);
}

// The selection proper of route_select_kernel (n > top_k + 2 pages): returns
// this thread's kept pages as bits (bit j: page tid KPT + j), the sel row
// position of its first one and the row's count (put_kept writes them).
template <int KPT>
__device__ __forceinline__ uint32_t select_rows_reg(const RouteParams& p, const SelRows& rows, int n, int* red,
                                                    int* warp_tot, int& first_pos, int& total) {
  const int tid = threadIdx.x;
  const int kk = p.top_k;
  // thread t holds pages [t * KPT, t * KPT + KPT)
  const float* sc = p.scores + rows.in * p.max_pages;
  const int p0 = tid * KPT;
  uint32_t key[KPT];
  if ((p.max_pages & 3) == 0) {
    // 16-byte rows: the thread's scores four at a time (every load inside the row:
    // p0 + j + 4 <= n <= max_pages whenever p0 + j < n)
#pragma unroll
    for (int j = 0; j < KPT; j += 4) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p0 + j < n) v = *reinterpret_cast<const float4*>(sc + p0 + j);
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pg = p0 + j + u;
        key[j + u] = (pg >= 1 && pg <= n - 2) ? order_key(vv[u]) : 0u;  // 0: not a candidate
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
      const int pg = p0 + j;
      key[j] = (pg >= 1 && pg <= n - 2) ? order_key(sc[pg]) : 0u;  // 0: not a candidate
    }
  }
  auto count_ge = [&](uint32_t t) {
    int c = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) c += key[j] >= t;
    return c;
  };
  // T: the largest key with at least k candidate keys >= T, bit by bit
  int phase = 0;
  uint32_t T = 0;
  bool exact = false;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    const int c = block_total(count_ge(cand), red, phase);
    if (c >= kk) {
      T = cand;
      if (c == kk) {
        exact = true;
        break;
      }
    }
  }
  // Kept: pages 0 and n - 1, keys above Tk, and the first keep_eq keys equal
  // to Tk in page order.  Exactly k keys are >= T when `exact`: keep those
  // (Tk = T - 1, no key equal to Tk is kept).  Otherwise T is the k-th largest
  // key and the keys equal to it fill what the larger ones leave.  One scan
  // counts both classes (above | equal << 16) before each thread.
  const uint32_t Tk = exact ? T - 1 : T;
  int above = 0, equal = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int pg = p0 + j;
    above += (pg == 0 || pg == n - 1 || key[j] > Tk) && pg < n;
    equal += key[j] != 0u && key[j] == Tk;
  }
  int tot;
  const int before = block_exclusive_scan(above | (equal << 16), warp_tot, tot);
  const int above_tot = tot & 0xffff, equal_tot = tot >> 16;
  const int keep_eq = exact ? 0 : kk - (above_tot - 2);  // pages 0 and n - 1 are counted in above_tot
  const int eq_before = before >> 16;
  int pos = (before & 0xffff) + min(eq_before, keep_eq);
  int tie = eq_before;
  uint32_t bits = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int pg = p0 + j;
    bool take = (pg == 0 || pg == n - 1 || key[j] > Tk) && pg < n;
    if (key[j] != 0u && key[j] == Tk) take = tie++ < keep_eq;
    if (take) bits |= 1u << j;
  }
  first_pos = pos;
  total = above_tot + min(equal_tot, keep_eq);
  return bits;
}

// The sel row entries of this thread's kept pages (bits from select_rows_reg,
// positions from first_pos on), the row's unused tail (-1) and its count.
template <int KPT>
__device__ __forceinline__ void put_kept(const RouteParams& p, const SelRows& rows, uint32_t bits, int first_pos,
                                         int total) {
  const int tid = threadIdx.x, p0 = tid * KPT;
  int pos = first_pos;
#pragma unroll
  for (int j = 0; j < KPT; ++j)
    if ((bits >> j) & 1u) put_sel(p, rows, pos++, p0 + j);
  for (int i = total + tid; i < p.top_k + 2; i += kSelectThreads) put_sel(p, rows, i, -1);
  if (tid == 0) put_cnt(p, rows, total);
}

// One CTA per (sequence, query head), or per (sequence, KV group) in the group
// modes.  The G CTAs of a KV group run as one thread-block cluster: each keeps
// its head's kept pages as bits in its own shared memory, and after a cluster
// barrier the first CTA reads the others' bits (distributed shared memory),
// forms the head mask of every page and writes the group's union list.  Each
// CTA writes its sel row between its cluster arrive and wait, beside the
// cluster's other heads still ranking (nothing in the cluster reads it).
template <int KPT>
__global__ void __launch_bounds__(kSelectThreads) route_select_kernel(RouteParams p) {
  __shared__ int red[2 * kSelectWarps];
  __shared__ int warp_tot[32];
  __shared__ uint32_t s_take[kSelectThreads];               // this CTA's kept pages, KPT bits per thread
  __shared__ uint32_t s_masks[kSelectThreads * KPT / 4];    // the group's head masks (first CTA)
  __shared__ int32_t s_bt[kSelectThreads * KPT];            // the sequence's block-table row (first CTA)
  allow_dependents();  // the union lists' reader may launch; it waits for this grid
  const int b = blockIdx.y, tid = threadIdx.x;
  const int L = p.seq_len[b];
  const int n = max(1, min((L + p.page - 1) / p.page, p.max_pages));
  const int nu = (L <= 0) ? 0 : n;  // pages of the union list
  const int kk = p.top_k;
  const int G = p.Hq / p.Hkv;
  const int g = p.group_mode ? (int)blockIdx.x : (int)blockIdx.x / G;
  const size_t bg = (size_t)b * p.Hkv + g;
  const uint32_t crank = cluster_ctarank();  // the head within the group (per-head mode)
  const int csize = p.group_mode ? 1 : G;
  const SelRows rows = sel_rows(p, blockIdx.x, b);
  const int p0 = tid * KPT;
  if (crank == 0) {
    // this thread's block-table entries come in while the rows are ranked
    const int32_t* bt_row = p.block_table + (size_t)b * p.max_pages;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (p0 + j < nu) cp_async4(&s_bt[p0 + j], bt_row + p0 + j);
    cp_async_commit_group();
  }
  uint32_t take;
  int first_pos = 0, total = 0;
  const bool ranked = n > kk + 2;
  if (!ranked) {
    for (int i = tid; i < kk + 2; i += kSelectThreads) put_sel(p, rows, i, (i < n) ? i : -1);
    if (tid == 0) put_cnt(p, rows, n);
    const int m = min(KPT, max(0, n - p0));  // every page is kept
    take = (m >= 32) ? 0xffffffffu : ((1u << m) - 1u);
  } else {
    take = select_rows_reg<KPT>(p, rows, n, red, warp_tot, first_pos, total);
  }
  s_take[tid] = take;
  cluster_arrive_release();  // this CTA's kept pages are in its shared memory
  // the sel rows are written while the cluster's other heads finish (nothing in
  // the cluster reads them)
  if (ranked) put_kept<KPT>(p, rows, take, first_pos, total);
  cluster_wait_acquire();
  if (crank != 0) {
    cluster_arrive_relaxed();  // the first CTA arrives here once it has read s_take: stay until then
    cluster_wait_acquire();
    return;
  }
  // head masks of this thread's pages: bit r from cluster CTA r (head g G + r)
  uint32_t tk[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) tk[r] = (r == 0) ? take : (r < csize ? ld_shared_cluster(&s_take[tid], r) : 0u);
  const uint32_t all_heads = (G >= 8) ? 0xffu : ((1u << G) - 1u);
#pragma unroll
  for (int w = 0; w < KPT / 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = 4 * w + q;
      uint32_t m = 0;
      if (p.group_mode) {
        m = ((take >> j) & 1u) ? all_heads : 0u;
      } else {
#pragma unroll
        for (int r = 0; r < 8; ++r) m |= ((tk[r] >> j) & 1u) << r;
      }
      word |= m << (8 * q);
    }
    s_masks[p0 / 4 + w] = word;
  }
  cluster_arrive_relaxed();  // the other CTAs' bits are read: they may exit
  cp_async_wait_group<0>();  // this thread's block-table entries
  if (tid == 0) zero_group_counters(p.acnt, bg, (size_t)p.batch * p.Hkv);  // the attention kernel's counters
  // each thread lists its own pages (masks and block-table entries it wrote itself)
  write_union_list_range(s_masks, min(nu, p0), min(nu, p0 + KPT), nu, s_bt, L, p.page, p.num_phys,
                         p.lists + bg * p.ustride, p.ucount + bg, p.err, warp_tot);
  cluster_wait_acquire();
}

// ---------------------------------------------------------------------------
// selection for block tables wider than the register-key kernel handles
// ---------------------------------------------------------------------------
constexpr int kCandCap = 512;  // boundary candidates ranked exactly in shared memory
constexpr int kLevels = 3;     // histogram refinements of the boundary bucket

// Monotone map of a score to one of 256 linear buckets over [lo, lo + 255.99/inv]:
// s1 <= s2 implies bucket(s1) <= bucket(s2) (fp subtraction, scaling and the
// clamps are all monotone), so every score in a higher bucket is larger.
__device__ __forceinline__ int lin_bucket(float s, float lo, float inv) {
  const float x = fminf(fmaxf((s - lo) * inv, 0.f), 255.f);  // fmaxf maps NaN to 0
  return (int)x;
}

__device__ __forceinline__ void block_minmax(float& mn, float& mx, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  mn = -warp_max(-mn);
  mx = warp_max(mx);
  if (lane == 0) {
    red[w] = mn;
    red[32 + w] = mx;
  }
  __syncthreads();
  float a = (lane < nw) ? red[lane] : INFINITY, c = (lane < nw) ? red[32 + lane] : -INFINITY;
  mn = -warp_max(-a);
  mx = warp_max(c);
  __syncthreads();
}

__device__ __forceinline__ int block_sum(int v, int* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  if (lane == 0) red[w] = v;
  __syncthreads();
  int t = (lane < nw) ? red[lane] : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
  __syncthreads();
  return t;
}

// One CTA per (sequence, query head), scores staged in shared memory.  A
// 256-bucket histogram over the linear score range (a monotone map, so whole
// buckets above the boundary bucket are kept) narrows the search to the
// boundary bucket, refined up to three times; its few scores are ranked
// exactly.  Finds T, the k-th largest score of pages 1..n-2, and how many pages
// scoring exactly T are kept (the lowest indices), then writes the kept pages
// plus 0 and n-1 in ascending order.
// The selection proper of route_select_hist_kernel (n > top_k + 2 pages).
__device__ __forceinline__ void select_rows_hist(const RouteParams& p, const SelRows& rows, int b, int n,
                                                 const float* sc, float* ssc, int* hist, int* warp_tot, float* redf,
                                                 float* cand, int* ps_ncand, int* ps_D, int* ps_above, int* ps_rem,
                                                 float* ps_T) {
  const int tid = threadIdx.x;
  const int kk = p.top_k;
  int& s_ncand = *ps_ncand;
  int& s_D = *ps_D;
  int& s_above = *ps_above;
  int& s_rem = *ps_rem;
  float& s_T = *ps_T;
  const int ncand = n - 2;  // pages 1 .. n-2 compete

  float mn = INFINITY, mx = -INFINITY;
  for (int i = tid; i < ncand; i += blockDim.x) {
    float v = sc[1 + i];
    if (v == 0.f) v = 0.f;  // -0 == +0
    ssc[1 + i] = v;
    if (isfinite(v)) {
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
  }
  block_minmax(mn, mx, redf);  // also orders the stores to ssc before the reads below
  float lo = (mn <= mx) ? mn : 0.f, hi = (mn <= mx) ? mx : 0.f;
  int rem = kk;   // how many of the still-undecided candidates are kept
  int D = 0;      // boundary bucket of the last level
  float inv = 0.f;
  int level = 0;
  for (;; ++level) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    inv = (hi > lo) ? 255.99f / (hi - lo) : 0.f;
    if (!isfinite(inv)) inv = 0.f;
    for (int i = tid; i < ncand; i += blockDim.x) {
      const float v = ssc[1 + i];
      if (level == 0 || (v >= lo && v <= hi)) atomicAdd(&hist[lin_bucket(v, lo, inv)], 1);
    }
    __syncthreads();
    if (tid < 32) {
      int loc[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        loc[j] = hist[8 * tid + j];
        sum += loc[j];
      }
      int x = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(kFull, x, o);
        if (tid + o < 32) x += y;
      }
      int above = x - sum;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (above < rem && rem <= above + loc[j]) {
          s_D = 8 * tid + j;
          s_above = above;
        }
        above += loc[j];
      }
    }
    __syncthreads();
    D = s_D;
    rem -= s_above;
    const int c = hist[D];
    if (c <= kCandCap || inv == 0.f || level + 1 >= kLevels) break;
    // refine: the scores of bucket D form an interval; histogram it again
    float bmn = INFINITY, bmx = -INFINITY;
    for (int i = tid; i < ncand; i += blockDim.x) {
      const float v = ssc[1 + i];
      if ((level == 0 || (v >= lo && v <= hi)) && lin_bucket(v, lo, inv) == D) {
        bmn = fminf(bmn, v);
        bmx = fmaxf(bmx, v);
      }
    }
    block_minmax(bmn, bmx, redf);
    if (!(isfinite(bmn) && isfinite(bmx))) break;  // an infinite score in the bucket: rank it exactly
    lo = bmn;
    hi = bmx;
  }

  // the boundary candidates: the level's active scores in bucket D
  auto in_boundary = [&](float v) {
    return (level == 0 || (v >= lo && v <= hi)) && lin_bucket(v, lo, inv) == D;
  };
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  const int c = hist[D];
  if (c <= kCandCap) {
    for (int i = tid; i < ncand; i += blockDim.x) {
      const float v = ssc[1 + i];
      if (in_boundary(v)) cand[atomicAdd(&s_ncand, 1)] = v;
    }
    __syncthreads();
    for (int i = tid; i < c; i += blockDim.x) {
      const float v = cand[i];
      int gt = 0, eq = 0;
      for (int j = 0; j < c; ++j) {
        gt += cand[j] > v;
        eq += cand[j] == v;
      }
      if (gt < rem && rem <= gt + eq) {
        s_T = v;
        s_rem = rem - gt;
      }
    }
  } else {
    // many equal (or infinite) scores in one bucket: rank against every boundary score
    for (int i = tid; i < ncand; i += blockDim.x) {
      const float v = ssc[1 + i];
      if (!in_boundary(v)) continue;
      int gt = 0, eq = 0;
      for (int j = 0; j < ncand; ++j) {
        const float w = ssc[1 + j];
        if (in_boundary(w)) {
          gt += w > v;
          eq += w == v;
        }
      }
      if (gt < rem && rem <= gt + eq) {
        s_T = v;
        s_rem = rem - gt;
      }
    }
  }
  __syncthreads();
  const float T = s_T;
  const int keep_eq = s_rem;  // candidates scoring exactly T that are kept

  // ties at T: the lowest page indices win
  const int per = (n + kSelectThreads - 1) / kSelectThreads;
  const int plo = tid * per, phi = min(n, plo + per);
  int eq_local = 0;
  for (int pg = plo; pg < phi; ++pg)
    if (pg >= 1 && pg <= n - 2 && ssc[pg] == T) ++eq_local;
  const int eq_total = block_sum(eq_local, warp_tot);
  int eq_rank = 0, tot = 0;
  if (eq_total > keep_eq) eq_rank = block_exclusive_scan(eq_local, warp_tot, tot);
  int take_local = 0;
  {
    int er = eq_rank;
    for (int pg = plo; pg < phi; ++pg) {
      bool take = (pg == 0 || pg == n - 1);
      if (!take) {
        const float v = ssc[pg];
        take = v > T || (v == T && er < keep_eq);
        if (v == T) ++er;
      }
      take_local += take;
    }
  }
  int pos = block_exclusive_scan(take_local, warp_tot, tot);
  {
    int er = eq_rank;
    for (int pg = plo; pg < phi; ++pg) {
      bool take = (pg == 0 || pg == n - 1);
      if (!take) {
        const float v = ssc[pg];
        take = v > T || (v == T && er < keep_eq);
        if (v == T) ++er;
      }
      if (take) put_sel(p, rows, pos++, pg);
    }
  }
  for (int i = tot + tid; i < kk + 2; i += blockDim.x) put_sel(p, rows, i, -1);
  if (tid == 0) put_cnt(p, rows, tot);
}


__global__ void __launch_bounds__(kSelectThreads) route_select_hist_kernel(RouteParams p) {
  extern __shared__ __align__(16) float ssc[];  // [max_pages] scores of this head
  __shared__ int hist[256];
  __shared__ int warp_tot[32];
  __shared__ float redf[64];
  __shared__ float cand[kCandCap];
  __shared__ int s_ncand, s_D, s_above, s_rem;
  __shared__ float s_T;
  __shared__ int s_flag;
  allow_dependents();

  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  const int L = p.seq_len[b];
  const int n = max(1, min((L + p.page - 1) / p.page, p.max_pages));
  const int kk = p.top_k;
  const SelRows rows = sel_rows(p, blockIdx.x, b);
  const float* sc = p.scores + rows.in * p.max_pages;

  if (n <= kk + 2) {
    for (int i = tid; i < kk + 2; i += blockDim.x) put_sel(p, rows, i, (i < n) ? i : -1);
    if (tid == 0) put_cnt(p, rows, n);
  } else {
    select_rows_hist(p, rows, b, n, sc, ssc, hist, warp_tot, redf, cand, &s_ncand, &s_D, &s_above, &s_rem, &s_T);
  }
  // the scores are no longer needed: their shared memory holds the union's page masks
  select_union_tail(p, b, blockIdx.x, reinterpret_cast<uint32_t*>(ssc), nullptr, warp_tot, &s_flag);
}

// ---------------------------------------------------------------------------
// launch
// ---------------------------------------------------------------------------
template <typename T, int D>
static cudaError_t launch_score_g(const RouteParams& p, int G, bool beside_append, cudaStream_t st) {
  const int nchunk = (p.max_pages + kScoreCtaPages - 1) / kScoreCtaPages;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunk, p.Hkv, p.batch);
  cfg.blockDim = dim3(kScoreThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may start while the append runs
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = beside_append ? 1 : 0;
  switch (G) {
    case 1: return cudaLaunchKernelEx(&cfg, route_score_kernel<T, D, 1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, route_score_kernel<T, D, 2>, p);
    case 4: return cudaLaunchKernelEx(&cfg, route_score_kernel<T, D, 4>, p);
    case 8: return cudaLaunchKernelEx(&cfg, route_score_kernel<T, D, 8>, p);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_route(const RouteParams& p, int d, bool bf16, int num_sms, cudaStream_t st, bool beside_append) {
  (void)num_sms;
  const int G = p.Hq / p.Hkv;
  cudaError_t e;
  const bool pa = beside_append;
  if (bf16)
    e = (d == 128) ? launch_score_g<__nv_bfloat16, 128>(p, G, pa, st) : launch_score_g<__nv_bfloat16, 64>(p, G, pa, st);
  else
    e = (d == 128) ? launch_score_g<float, 128>(p, G, pa, st) : launch_score_g<float, 64>(p, G, pa, st);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.group_mode ? p.Hkv : p.Hq, p.batch);
  if (p.max_pages <= kSelectThreads * 32) {
    // the G heads of a KV group as one cluster (one CTA per group in the group modes)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kSelectThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.group_mode ? 1 : G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (p.max_pages <= kSelectThreads * 8) return cudaLaunchKernelEx(&cfg, route_select_kernel<8>, p);
    if (p.max_pages <= kSelectThreads * 16) return cudaLaunchKernelEx(&cfg, route_select_kernel<16>, p);
    return cudaLaunchKernelEx(&cfg, route_select_kernel<32>, p);
  } else {
    const size_t smem = (size_t)p.max_pages * sizeof(float);
    if ((e = ensure_smem((const void*)route_select_hist_kernel, smem)) != cudaSuccess) return e;
    route_select_hist_kernel<<<grid, kSelectThreads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace bkv
