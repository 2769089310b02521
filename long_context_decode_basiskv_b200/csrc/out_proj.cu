// Step 5 of the BasisKV decode step: out-projection through the bound factor.
//
// The Value latent is tied to the output projection (kongchang.com explainer,
// opening section; BasisKV abstract): with V ~ C B_g, the layer output
//   y = sum_h softmax(...) (C B_g) W_O,h = sum_h o_h (B_g W_O,h) = sum_h o_h G_h
// so the rank-r attention output of each head is multiplied by the fused
// factor G_h and the full Value width is never formed.
//
// Gt holds row c = output column c for every (head, latent dim), so y[b][c]
// is one dot product of length Hq*r per batch row.  This file holds the
// CUDA-core kernels: the GEMV for fp32 (and for bf16 when Gt is not in the
// tensor-core tile layout), and the fp64 fusion that writes Gt, tiled for the
// tensor-core kernels when the shape allows.
#include "kernels.cuh"

namespace bkv {



constexpr int kOpWarps = 8;
constexpr int kOpRows = 8;  // batch rows per CTA

// one warp per output column, kOpRows batch rows per CTA
template <typename T>
__global__ void __launch_bounds__(kOpWarps * 32) out_proj_gemv_kernel(OutProjParams p) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * kOpWarps + w;
  const int b0 = blockIdx.y * kOpRows;
  if (c >= p.hidden) return;
  const int nb = min(kOpRows, p.batch - b0);
  const T* grow = static_cast<const T*>(p.Gt) + (size_t)c * p.K;
  float acc[kOpRows];
#pragma unroll
  for (int i = 0; i < kOpRows; ++i) acc[i] = 0.f;
  for (int k = lane; k < p.K; k += 32) {
    const float gv = Elem<T>::to_f(grow[k]);
#pragma unroll
    for (int i = 0; i < kOpRows; ++i)
      if (i < nb) acc[i] = fmaf(gv, p.o[(size_t)(b0 + i) * p.K + k], acc[i]);
  }
#pragma unroll
  for (int i = 0; i < kOpRows; ++i) {
    const float v = warp_sum(acc[i]);
    if (lane == 0 && i < nb) p.y[(size_t)(b0 + i) * p.hidden + c] = v;
  }
}

cudaError_t launch_out_proj_gemv(const OutProjParams& p, bool bf16, cudaStream_t st) {
  dim3 grid((p.hidden + kOpWarps - 1) / kOpWarps, (p.batch + kOpRows - 1) / kOpRows);
  if (bf16)
    out_proj_gemv_kernel<__nv_bfloat16><<<grid, kOpWarps * 32, 0, st>>>(p);
  else
    out_proj_gemv_kernel<float><<<grid, kOpWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// fusion: Gt[c][h][i] = sum_j Bf[g(h)][i][j] W_O[h d + j][c]   (fp64, rounded once)
// ---------------------------------------------------------------------------


constexpr int kFuseCols = 32;

template <typename T>
__global__ void __launch_bounds__(128) fuse_kernel(FuseParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int h = blockIdx.y, c0 = blockIdx.x * kFuseCols;
  const int g = h / (p.Hq / p.Hkv);
  const int d = p.d, r = p.r;
  const int ld = d + 1;                                  // padded row of Bf
  float* sB = reinterpret_cast<float*>(smem);            // [r][d + 1]
  double* sW = reinterpret_cast<double*>(sB + ((r * ld + 1) & ~1));  // [d][kFuseCols]
  const T* B = static_cast<const T*>(p.Bf) + (size_t)g * r * d;
  for (int i = threadIdx.x; i < r * d; i += blockDim.x) sB[(i / d) * ld + (i % d)] = Elem<T>::to_f(B[i]);
  const T* W = static_cast<const T*>(p.W_O) + (size_t)h * d * p.hidden;
  for (int i = threadIdx.x; i < d * kFuseCols; i += blockDim.x) {
    const int j = i / kFuseCols, c = i % kFuseCols;
    sW[i] = (c0 + c < p.hidden) ? Elem<T>::to_d(W[(size_t)j * p.hidden + c0 + c]) : 0.0;
  }
  __syncthreads();
  T* out = static_cast<T*>(p.Gt);
  for (int i = threadIdx.x; i < r; i += blockDim.x) {
    for (int c = 0; c < kFuseCols && c0 + c < p.hidden; ++c) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc = fma((double)sB[i * ld + j], sW[j * kFuseCols + c], acc);
      const int col = c0 + c, k = h * r + i;
      size_t idx;
      if (p.blocked) {
        // tile (col / 128, k / 64); row col % 128 holds 8 chunks of 8, chunk j at j ^ (row % 8)
        const int KC = p.Hq * r / 64, m = col & 127, kk = k & 63;
        idx = (((size_t)(col >> 7) * KC + (k >> 6)) * 128 + m) * 64 + ((((kk >> 3) ^ (m & 7)) << 3) | (kk & 7));
      } else {
        idx = (size_t)col * p.Hq * r + k;
      }
      out[idx] = Elem<T>::from_d(acc);
    }
  }
}

cudaError_t launch_fuse(const FuseParams& p, bool bf16, cudaStream_t st) {
  const size_t smem = (((size_t)p.r * (p.d + 1) + 1) & ~(size_t)1) * 4 + (size_t)p.d * kFuseCols * 8;
  dim3 grid((p.hidden + kFuseCols - 1) / kFuseCols, p.Hq);
  if (bf16) {
    if (cudaError_t e = ensure_smem((const void*)fuse_kernel<__nv_bfloat16>, smem); e != cudaSuccess) return e;
    fuse_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(p);
  } else {
    if (cudaError_t e = ensure_smem((const void*)fuse_kernel<float>, smem); e != cudaSuccess) return e;
    fuse_kernel<float><<<grid, 128, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace bkv
