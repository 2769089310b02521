// Steps 1-2 of the BasisKV decode step: latent/residual append and page summary.
//
// Per new token and KV head g (BasisKV abstract; kongchang.com explainer,
// section on Value latents assisting key routing):
//   C = v A_g                       Value latent, rank r
//   R = (k - C P_g) E_g             key-specific residual, rank s (from the unrounded C)
// the raw key, C and R are written to the token's slot of its page.  Then the
// page's summary, the mean predicted key over its valid tokens, is recomputed:
//   S = mean(C) P_g + mean(R) E_g^T                       (fp32)
//
// One CTA owns one (sequence, KV head, touched page), so the summary of a page
// is written by exactly one CTA after all of that page's new tokens are stored.
// All sums are fp64: the bf16/fp32 value stored for C, R and S is the correctly
// rounded value of the exact result, which is what the fp64 reference rounds.
// The work is tiny per decode step (one token per (b, g)); it is latency-bound.
#include "kernels.cuh"

namespace bkv {



constexpr int kAppendThreads = 256;
constexpr int kAppendChunkMax = 16;  // new tokens processed together (fewer when fewer are appended)

// 16-byte vector copy global -> shared of `bytes` (multiple of 16).
__device__ __forceinline__ void copy16(void* dst, const void* src, int bytes, int tid, int nthr) {
  const int4* s = reinterpret_cast<const int4*>(src);
  int4* t = reinterpret_cast<int4*>(dst);
  for (int i = tid; i < bytes / 16; i += nthr) t[i] = s[i];
}

template <typename T>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(AppendParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int b = blockIdx.z, g = blockIdx.y;
  const int tid = threadIdx.x;
  const int d = p.d, r = p.r, s = p.s, P = p.page;

  const int kAppendChunk = min(kAppendChunkMax, p.n_new);
  const int L = p.seq_len[b];
  if (L < p.n_new || L > p.max_pages * P || p.n_new <= 0) {
    if (tid == 0 && blockIdx.x == 0) set_err(p.err, BASISKV_DEVERR_SEQ_LEN);
    return;
  }
  const int first_new = L - p.n_new;
  const int page = first_new / P + blockIdx.x;
  if (page * P >= L) return;  // this CTA has no page (grid sized for the longest range)
  const int phys = p.block_table[(size_t)b * p.max_pages + page];
  if (phys < 0 || phys >= p.num_phys) {
    if (tid == 0) set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
    return;
  }

  // shared memory: factors of head g (storage dtype), token rows, fp64 scratch
  T* sA = reinterpret_cast<T*>(smem);                 // [d][r]
  T* sP = sA + d * r;                                  // [r][d]
  T* sE = sP + r * d;                                  // [d][s]
  float* sk = reinterpret_cast<float*>(sE + d * s);    // [chunk][d]
  float* sv = sk + kAppendChunk * d;                   // [chunk][d]
  double* sC = reinterpret_cast<double*>(sv + kAppendChunk * d);  // [chunk][r]
  double* sU = sC + kAppendChunk * r;                  // [chunk][d]  k - C P
  double* sMean = sU + kAppendChunk * d;               // [r + s]

  copy16(sA, static_cast<const T*>(p.A) + (size_t)g * d * r, d * r * (int)sizeof(T), tid, blockDim.x);
  copy16(sP, static_cast<const T*>(p.P) + (size_t)g * r * d, r * d * (int)sizeof(T), tid, blockDim.x);
  copy16(sE, static_cast<const T*>(p.E) + (size_t)g * d * s, d * s * (int)sizeof(T), tid, blockDim.x);

  const size_t blk = (size_t)phys * p.Hkv + g;  // page block of head g
  T* kdst = static_cast<T*>(p.k_raw) + blk * P * d;
  T* cdst = static_cast<T*>(p.c_lat) + blk * P * r;
  T* rdst = static_cast<T*>(p.r_res) + blk * P * s;

  // bf16 K and C rows are stored swizzled for the tensor-core attention path
  const bool swz_on = kc_swizzled(sizeof(T) == 2, d, r);
  const int mk = swz_on ? swz_mask(d) : 0, mc = swz_on ? swz_mask(r) : 0;
  const int t_lo = max(first_new, page * P);
  const int t_hi = min(L, (page + 1) * P);
  const T* kin = static_cast<const T*>(p.k_new);
  const T* vin = static_cast<const T*>(p.v_new);

  for (int c0 = t_lo; c0 < t_hi; c0 += kAppendChunk) {
    const int nt = min(kAppendChunk, t_hi - c0);
    __syncthreads();  // factors loaded / previous chunk finished with sk, sv, sC, sU
    for (int i = tid; i < nt * d; i += blockDim.x) {
      const int t = i / d, x = i - t * d;
      const size_t row = ((size_t)b * p.n_new + (c0 + t - first_new)) * p.Hkv + g;
      const T kv = kin[row * d + x];
      sk[t * d + x] = Elem<T>::to_f(kv);
      sv[t * d + x] = Elem<T>::to_f(vin[row * d + x]);
      const int slot = c0 + t - page * P;
      kdst[(size_t)slot * d + swz(x, slot, mk)] = kv;  // raw key stored as given
    }
    __syncthreads();
    // C = v A
    for (int i = tid; i < nt * r; i += blockDim.x) {
      const int t = i / r, j = i - t * r;
      double acc = 0.0;
      for (int x = 0; x < d; ++x) acc = fma((double)sv[t * d + x], Elem<T>::to_d(sA[x * r + j]), acc);
      sC[t * r + j] = acc;
      const int slot = c0 + t - page * P;
      cdst[(size_t)slot * r + swz(j, slot, mc)] = Elem<T>::from_d(acc);
    }
    __syncthreads();
    // U = k - C P   (C unrounded)
    for (int i = tid; i < nt * d; i += blockDim.x) {
      const int t = i / d, x = i - t * d;
      double acc = 0.0;
      for (int j = 0; j < r; ++j) acc = fma(sC[t * r + j], Elem<T>::to_d(sP[j * d + x]), acc);
      sU[t * d + x] = (double)sk[t * d + x] - acc;
    }
    __syncthreads();
    // R = U E
    for (int i = tid; i < nt * s; i += blockDim.x) {
      const int t = i / s, m = i - t * s;
      double acc = 0.0;
      for (int x = 0; x < d; ++x) acc = fma(sU[t * d + x], Elem<T>::to_d(sE[x * s + m]), acc);
      rdst[(size_t)(c0 + t - page * P) * s + m] = Elem<T>::from_d(acc);
    }
  }
  __syncthreads();  // this CTA's stores of C and R are visible to the whole CTA

  // page summary over the valid tokens 0 .. m-1 of this page (old and new)
  const int m = min(L, (page + 1) * P) - page * P;
  for (int j = tid; j < r + s; j += blockDim.x) {
    double acc = 0.0;
    if (j < r) {
      for (int t = 0; t < m; ++t) acc += Elem<T>::to_d(cdst[(size_t)t * r + swz(j, t, mc)]);
    } else {
      for (int t = 0; t < m; ++t) acc += Elem<T>::to_d(rdst[(size_t)t * s + (j - r)]);
    }
    sMean[j] = acc / (double)m;
  }
  __syncthreads();
  for (int x = tid; x < d; x += blockDim.x) {
    double acc = 0.0;
    for (int j = 0; j < r; ++j) acc = fma(sMean[j], Elem<T>::to_d(sP[j * d + x]), acc);
    double acc2 = 0.0;
    for (int q = 0; q < s; ++q) acc2 = fma(sMean[r + q], Elem<T>::to_d(sE[x * s + q]), acc2);
    p.summary[blk * d + x] = __double2float_rn(acc + acc2);
  }
}

// ---------------------------------------------------------------------------
// decode step (one new token per sequence): one CTA per (KV head, sequence).
// Every load is issued up front (factors, the new k and v, the page's earlier
// latents and residuals), then each output of C = v A, U = k - C P, R = U E and
// S = mean(C) P + mean(R) E^T is a dot product split over a few threads of a
// warp and summed with shuffles, all in fp64 with one rounding per stored value.
// ---------------------------------------------------------------------------
constexpr int kDecThreads = 256;

// sum of `len` fp64 products a[i * sa] * b[i * sb], split over `tpo` adjacent
// lanes (tpo a power of two <= 32); every lane of the group returns the total
__device__ __forceinline__ double as_d(double x) { return x; }
__device__ __forceinline__ double as_d(float x) { return (double)x; }
__device__ __forceinline__ double as_d(__nv_bfloat16 x) { return (double)__bfloat162float(x); }

template <typename TA, typename TB>
__device__ __forceinline__ double split_dot(const TA* a, int sa, const TB* b, int sb, int len, int tpo,
                                           int part) {
  double acc = 0.0;
  for (int i = part; i < len; i += tpo) acc = fma(as_d(a[i * sa]), as_d(b[i * sb]), acc);
  for (int o = tpo >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
  return acc;
}

__host__ __device__ __forceinline__ int pow2_floor(int x) {
  int v = 1;
  while (v * 2 <= x) v *= 2;
  return v;
}

// Shared memory of the decode append; every region starts on 16 bytes.
// Storage type T: A [d][r], P [r][d], E [d][s], the page's C block [page][r] and
// R block [page][s] as stored (C rows swizzled when K/C swizzling is on), k and v.
// fp64: C [r] (unrounded), U = k - C P [d], the stored C [r] and R [s] of the new
// token, the page means [r + s]; then one mbarrier.
struct DecLayout {
  size_t a, p, e, cb, rb, k, v, c, u, cs, rs, mean, bar, total;
};

__host__ __device__ __forceinline__ size_t round16(size_t x) { return (x + 15) & ~(size_t)15; }

__host__ __device__ __forceinline__ DecLayout dec_layout(int d, int r, int s, int P, int es) {
  DecLayout L;
  size_t o = 0;
  L.a = o;    o = round16(o + (size_t)d * r * es);
  L.p = o;    o = round16(o + (size_t)r * d * es);
  L.e = o;    o = round16(o + (size_t)d * s * es);
  L.cb = o;   o = round16(o + (size_t)P * r * es);
  L.rb = o;   o = round16(o + (size_t)P * s * es);
  L.k = o;    o = round16(o + (size_t)d * es);
  L.v = o;    o = round16(o + (size_t)d * es);
  L.c = o;    o += (size_t)r * 8;
  L.u = o;    o += (size_t)d * 8;
  L.cs = o;   o += (size_t)r * 8;
  L.rs = o;   o += (size_t)s * 8;
  L.mean = o; o += (size_t)(r + s) * 8;
  L.bar = o;  o += 8;
  L.total = o;
  return L;
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads) append_decode_kernel(AppendParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int s_ok;
  // A kernel launched as this one's programmatic dependent (the route's scoring
  // in basiskv_append_route) may start now: it reads nothing this kernel writes
  // and waits for it before it ends.
  allow_dependents();
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int d = p.d, r = p.r, s = p.s, P = p.page;
  const int L = p.seq_len[b];
  if (L < 1 || L > p.max_pages * P) {
    if (tid == 0) set_err(p.err, BASISKV_DEVERR_SEQ_LEN);
    return;
  }
  const int page = (L - 1) / P, slot = (L - 1) - page * P;
  const int phys = p.block_table[(size_t)b * p.max_pages + page];
  if (phys < 0 || phys >= p.num_phys) {
    if (tid == 0) set_err(p.err, BASISKV_DEVERR_BLOCK_TABLE);
    return;
  }
  const bool swz_on = kc_swizzled(sizeof(T) == 2, d, r);
  const int mk = swz_on ? swz_mask(d) : 0, mc = swz_on ? swz_mask(r) : 0;
  const DecLayout ly = dec_layout(d, r, s, P, (int)sizeof(T));
  T* sA = reinterpret_cast<T*>(smem + ly.a);
  T* sP = reinterpret_cast<T*>(smem + ly.p);
  T* sE = reinterpret_cast<T*>(smem + ly.e);
  T* sCb = reinterpret_cast<T*>(smem + ly.cb);
  T* sRb = reinterpret_cast<T*>(smem + ly.rb);
  T* skT = reinterpret_cast<T*>(smem + ly.k);
  T* svT = reinterpret_cast<T*>(smem + ly.v);
  double* sC = reinterpret_cast<double*>(smem + ly.c);
  double* sU = reinterpret_cast<double*>(smem + ly.u);
  double* sCs = reinterpret_cast<double*>(smem + ly.cs);
  double* sRs = reinterpret_cast<double*>(smem + ly.rs);
  double* sMean = reinterpret_cast<double*>(smem + ly.mean);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + ly.bar);

  const size_t blk = (size_t)phys * p.Hkv + g;
  const size_t row = (size_t)b * p.Hkv + g;  // n_new == 1
  T* kdst = static_cast<T*>(p.k_raw) + blk * P * d;
  T* cdst = static_cast<T*>(p.c_lat) + blk * P * r;
  T* rdst = static_cast<T*>(p.r_res) + blk * P * s;

  // Stage everything at once: the factors of head g, the page's stored C and R
  // blocks (only the first `slot` rows are read) and the new k and v.  Pieces
  // that are 16-byte aligned in global memory travel as bulk copies on one
  // mbarrier; any other piece is copied element-wise by all threads.
  constexpr int kPieces = 7;
  const T* src[kPieces] = {static_cast<const T*>(p.A) + (size_t)g * d * r,
                           static_cast<const T*>(p.P) + (size_t)g * r * d,
                           static_cast<const T*>(p.E) + (size_t)g * d * s,
                           cdst, rdst,
                           static_cast<const T*>(p.k_new) + row * d,
                           static_cast<const T*>(p.v_new) + row * d};
  T* dst[kPieces] = {sA, sP, sE, sCb, sRb, skT, svT};
  const int len[kPieces] = {d * r, r * d, d * s, P * r, P * s, d, d};
  auto bulk_able = [&](int i) {
    return ((reinterpret_cast<uintptr_t>(src[i]) | ((size_t)len[i] * sizeof(T))) & 15u) == 0;
  };
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    uint32_t tx = 0;
#pragma unroll
    for (int i = 0; i < kPieces; ++i)
      if (bulk_able(i)) tx += (uint32_t)(len[i] * sizeof(T));
    mbar_arrive_expect_tx(bar, tx);
#pragma unroll
    for (int i = 0; i < kPieces; ++i)
      if (bulk_able(i)) bulk_g2s(dst[i], src[i], (uint32_t)(len[i] * sizeof(T)), bar);
  }
#pragma unroll
  for (int i = 0; i < kPieces; ++i)
    if (!bulk_able(i))
      for (int j = tid; j < len[i]; j += kDecThreads) dst[i][j] = src[i][j];
  if (tid == 0) s_ok = mbar_wait_bounded(bar, 0) ? 1 : 0;
  __syncthreads();
  if (!s_ok) {
    if (tid == 0) set_err(p.err, BASISKV_DEVERR_TIMEOUT);
    return;
  }

  for (int i = tid; i < d; i += kDecThreads) kdst[(size_t)slot * d + swz(i, slot, mk)] = skT[i];  // raw key as given
  const int lane = tid & 31;
  // Each phase runs the same number of rounds on every lane (the shuffles need
  // the whole warp); lanes past the last output use an empty sum.
  // C = v A
  {
    const int tpo = min(32, pow2_floor(max(1, kDecThreads / r)));
    const int part = lane & (tpo - 1), per = kDecThreads / tpo;
    for (int rd = 0; rd < (r + per - 1) / per; ++rd) {
      const int base = rd * per + tid / tpo;
      const bool on = base < r;
      const double c = split_dot(svT, 1, sA + (on ? base : 0), r, on ? d : 0, tpo, part);
      if (on && part == 0) {
        const T cq = Elem<T>::from_d(c);
        sC[base] = c;
        sCs[base] = Elem<T>::to_d(cq);  // the stored value, for the page mean
        cdst[(size_t)slot * r + swz(base, slot, mc)] = cq;
      }
    }
  }
  __syncthreads();
  // U = k - C P   (C unrounded)
  {
    const int tpo = min(32, pow2_floor(max(1, kDecThreads / d)));
    const int part = lane & (tpo - 1), per = kDecThreads / tpo;
    for (int rd = 0; rd < (d + per - 1) / per; ++rd) {
      const int base = rd * per + tid / tpo;
      const bool on = base < d;
      const double cp = split_dot(sC, 1, sP + (on ? base : 0), d, on ? r : 0, tpo, part);
      if (on && part == 0) sU[base] = Elem<T>::to_d(skT[base]) - cp;
    }
  }
  __syncthreads();
  // R = U E
  {
    const int tpo = min(32, pow2_floor(max(1, kDecThreads / s)));
    const int part = lane & (tpo - 1), per = kDecThreads / tpo;
    for (int rd = 0; rd < (s + per - 1) / per; ++rd) {
      const int base = rd * per + tid / tpo;
      const bool on = base < s;
      const double rv = split_dot(sU, 1, sE + (on ? base : 0), s, on ? d : 0, tpo, part);
      if (on && part == 0) {
        const T rq = Elem<T>::from_d(rv);
        rdst[(size_t)slot * s + base] = rq;
        sRs[base] = Elem<T>::to_d(rq);
      }
    }
  }
  __syncthreads();
  // page means over the slot + 1 valid tokens, in token order
  for (int j = tid; j < r + s; j += kDecThreads) {
    double acc = 0.0;
    if (j < r) {
      for (int t = 0; t < slot; ++t) acc += Elem<T>::to_d(sCb[t * r + swz(j, t, mc)]);
      acc += sCs[j];
    } else {
      for (int t = 0; t < slot; ++t) acc += Elem<T>::to_d(sRb[t * s + (j - r)]);
      acc += sRs[j - r];
    }
    sMean[j] = acc / (double)(slot + 1);
  }
  __syncthreads();
  // S = mean(C) P + mean(R) E^T
  {
    const int tpo = min(32, pow2_floor(max(1, kDecThreads / d)));
    const int part = lane & (tpo - 1), per = kDecThreads / tpo;
    for (int rd = 0; rd < (d + per - 1) / per; ++rd) {
      const int base = rd * per + tid / tpo;
      const bool on = base < d;
      const double a1 = split_dot(sMean, 1, sP + (on ? base : 0), d, on ? r : 0, tpo, part);
      const double a2 = split_dot(sMean + r, 1, sE + (size_t)(on ? base : 0) * s, 1, on ? s : 0, tpo, part);
      if (on && part == 0) p.summary[blk * d + base] = __double2float_rn(a1 + a2);
    }
  }
}

static size_t append_decode_smem_bytes(int d, int r, int s, int P, int esize) {
  return dec_layout(d, r, s, P, esize).total;
}

size_t append_smem_bytes(int d, int r, int s, int esize, int n_new) {
  const int chunk = n_new < kAppendChunkMax ? n_new : kAppendChunkMax;
  size_t f = (size_t)(d * r * 2 + d * s) * esize;
  f = (f + 15) & ~(size_t)15;
  return f + (size_t)chunk * d * 4 * 2 + (size_t)chunk * (r + d) * 8 + (size_t)(r + s) * 8;
}

cudaError_t launch_append(const AppendParams& p, bool bf16, cudaStream_t st) {
  const size_t dsm = append_decode_smem_bytes(p.d, p.r, p.s, p.page, bf16 ? 2 : 4);
  if (p.n_new == 1 && dsm <= 227 * 1024) {
    dim3 grid(p.Hkv, p.batch);
    if (bf16) {
      if (cudaError_t e = ensure_smem((const void*)append_decode_kernel<__nv_bfloat16>, dsm); e != cudaSuccess) return e;
      append_decode_kernel<__nv_bfloat16><<<grid, kDecThreads, dsm, st>>>(p);
    } else {
      if (cudaError_t e = ensure_smem((const void*)append_decode_kernel<float>, dsm); e != cudaSuccess) return e;
      append_decode_kernel<float><<<grid, kDecThreads, dsm, st>>>(p);
    }
    return cudaGetLastError();
  }
  const int max_touched = (p.n_new + p.page - 1) / p.page + 1;
  dim3 grid(max_touched, p.Hkv, p.batch);
  const size_t smem = append_smem_bytes(p.d, p.r, p.s, bf16 ? 2 : 4, p.n_new);
  if (bf16) {
    if (cudaError_t e = ensure_smem((const void*)append_kernel<__nv_bfloat16>, smem); e != cudaSuccess) return e;
    append_kernel<__nv_bfloat16><<<grid, kAppendThreads, smem, st>>>(p);
  } else {
    if (cudaError_t e = ensure_smem((const void*)append_kernel<float>, smem); e != cudaSuccess) return e;
    append_kernel<float><<<grid, kAppendThreads, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace bkv
