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
constexpr int kAppendChunk = 16;  // new tokens processed together

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

size_t append_smem_bytes(int d, int r, int s, int esize) {
  size_t f = (size_t)(d * r * 2 + d * s) * esize;
  f = (f + 15) & ~(size_t)15;
  return f + (size_t)kAppendChunk * d * 4 * 2 + (size_t)kAppendChunk * (r + d) * 8 + (size_t)(r + s) * 8;
}

cudaError_t launch_append(const AppendParams& p, bool bf16, cudaStream_t st) {
  const int max_touched = (p.n_new + p.page - 1) / p.page + 1;
  dim3 grid(max_touched, p.Hkv, p.batch);
  const size_t smem = append_smem_bytes(p.d, p.r, p.s, bf16 ? 2 : 4);
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
