// Per-group union lists: the pages a KV group's attention reads.
//
// Under grouped-query attention the G query heads of a KV group share one key
// head, so the sparse-attention kernel reads every page selected by any head
// of the group once and applies it to the heads that selected it.  The routing
// step (or, when the caller passes its own selection, a small kernel) stores,
// per (sequence, KV head), the ascending list of those pages with what the
// attention kernel needs to fetch a page without further lookups:
//
//   uint32 list[4 + umax]:  list[0] = U (entries), list[1] = valid tokens of
//   the last entry (the page size unless that entry is the sequence's partial
//   last page), list[2..3] unused;
//   entry i at list[4 + i]:  physical page id (bits 0-23; kNoPage: unusable,
//   skipped) | head mask << 24 (bit hi: head g G + hi reads the page).
//
// Pages are ascending, so only the last entry can be the partial last page.
// The list stride is a multiple of 4 words, so every list starts on 16 bytes
// and the attention kernel copies it with one bulk copy.
#pragma once

#include "common.cuh"

namespace bkv {

constexpr uint32_t kNoPage = 0xffffffu;      // entry id of a page whose block-table entry is out of range
// The attention kernels keep kGroupCounters int counters per group (the
// finished splits), in planes of B Hkv ints; whoever writes a group's list
// sets them to zero.
constexpr int kGroupCounters = 1;
__device__ __forceinline__ void zero_group_counters(int32_t* cnt, size_t bg, size_t ngroups) {
#pragma unroll
  for (int i = 0; i < kGroupCounters; ++i) cnt[(size_t)i * ngroups + bg] = 0;
}
constexpr int kMaxPhysPages = 0xffffff;      // physical page ids must fit the 24 id bits

__host__ __device__ __forceinline__ int union_stride_words(int umax) { return (4 + umax + 3) & ~3; }

// All threads of the block call this, each for its pages [lo, hi) (the
// threads' ranges ascend with the thread index and cover 0 .. n-1).  `mask8`
// holds one byte per logical page of the sequence (packed four to a word;
// nonzero = selected by the heads whose bits are set).  Writes the group's
// list in ascending page order.  `bt_row` is the sequence's block-table row
// (shared or global memory); a page whose entry is outside [0, num_phys) is
// stored as kNoPage and sets the error flag.  `L` is the sequence length (the
// last page may be partial).  The entry count also goes to *ucount, the
// group's slot of a compact [B][Hkv] array from which the attention kernel
// shares its CTAs out among the groups.  A thread's own mask bytes and
// block-table entries need no barrier before the call; thread 0 reads page
// n-1's byte after the call's first barrier.
__device__ __forceinline__ void write_union_list_range(const uint32_t* mask8, int lo, int hi, int n,
                                                       const int32_t* bt_row, int L, int page, int num_phys,
                                                       uint32_t* list, uint32_t* ucount, int32_t* err,
                                                       int* warp_tot) {
  const int tid = threadIdx.x;
  int c = 0;
  for (int pg = lo; pg < hi; ++pg) c += ((mask8[pg >> 2] >> ((pg & 3) * 8)) & 0xffu) ? 1 : 0;
  int tot;
  int pos = block_exclusive_scan(c, warp_tot, tot);
  bool has_last = false;
  for (int pg = lo; pg < hi; ++pg) {
    const uint32_t m = (mask8[pg >> 2] >> ((pg & 3) * 8)) & 0xffu;
    if (!m) continue;
    const int ph = bt_row[pg];
    uint32_t id = (uint32_t)ph;
    if (ph < 0 || ph >= num_phys) {
      set_err(err, BASISKV_DEVERR_BLOCK_TABLE);
      id = kNoPage;
    }
    list[4 + pos] = id | (m << 24);
    ++pos;
    has_last = has_last || pg == n - 1;
  }
  if (has_last) list[1] = (uint32_t)(L - (n - 1) * page);  // the thread holding page n - 1
  if (tid == 0) {
    list[0] = (uint32_t)tot;
    *ucount = (uint32_t)tot;  // the same count, in the compact per-group array
    if (n < 1 || !((mask8[(n - 1) >> 2] >> (((n - 1) & 3) * 8)) & 0xffu)) list[1] = (uint32_t)page;
  }
}

// write_union_list_range with the pages split evenly over the block's threads.
__device__ __forceinline__ void write_union_list(const uint32_t* mask8, int n, const int32_t* bt_row, int L,
                                                 int page, int num_phys, uint32_t* list, uint32_t* ucount,
                                                 int32_t* err, int* warp_tot) {
  const int nthr = blockDim.x;
  const int per = (n + nthr - 1) / nthr;
  const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
  write_union_list_range(mask8, lo, hi, n, bt_row, L, page, num_phys, list, ucount, err, warp_tot);
}

// The union list of group (b, g) from the G heads' selection rows: sel
// [B][Hq][top_k + 2] / sel_cnt [B][Hq] as basiskv_route writes them (rows
// written by other CTAs of the grid are read from L2).  All threads of the block
// call this; `masks` is shared scratch of (max_pages + 3) / 4 words; `bt_smem`
// (may be NULL) shared scratch of max_pages words that receives the sequence's
// block-table row while the selections load.  A selected page outside [0, n)
// sets BASISKV_DEVERR_SELECTION and is dropped.  Also zeroes the group's
// attention counters (acnt) for the attention launch that reads the list, whatever the scratch held before (`ngroups` = B Hkv).
__device__ __forceinline__ void union_from_selection(const int32_t* sel, const int32_t* sel_cnt,
                                                     const int32_t* block_table, int L, int b, int g, int Hq,
                                                     int Hkv, int page, int max_pages, int num_phys, int top_k,
                                                     uint32_t* list, uint32_t* ucount, int32_t* acnt,
                                                     size_t ngroups, int32_t* err, uint32_t* masks,
                                                     int32_t* bt_smem, int* warp_tot) {
  const int tid = threadIdx.x;
  const int G = Hq / Hkv;
  const int row_len = top_k + 2;
  int n = (L + page - 1) / page;
  if (L < 0) n = 0;
  if (n > max_pages) n = max_pages;
  const size_t row0 = (size_t)b * Hq + (size_t)g * G;
  const int32_t* bt_row = block_table + (size_t)b * max_pages;
  if (tid == 0) zero_group_counters(acnt, (size_t)b * Hkv + g, ngroups);
  const int words = (max_pages + 3) / 4;
  for (int i = tid; i < words; i += blockDim.x) masks[i] = 0u;
  if (bt_smem)
    for (int i = tid; i < n; i += blockDim.x) bt_smem[i] = bt_row[i];
  __syncthreads();
  for (int i = tid; i < G * row_len; i += blockDim.x) {
    const int hi = i / row_len, j = i - hi * row_len;
    if (j >= min(__ldcg(sel_cnt + row0 + hi), row_len)) continue;
    const int pg = __ldcg(sel + row0 * row_len + i);
    if (pg < 0 || pg >= n) {
      set_err(err, BASISKV_DEVERR_SELECTION);
      continue;
    }
    atomicOr(&masks[pg >> 2], (1u << hi) << ((pg & 3) * 8));
  }
  __syncthreads();
  write_union_list(masks, n, bt_smem ? bt_smem : bt_row, L, page, num_phys, list, ucount, err, warp_tot);
}

}  // namespace bkv
