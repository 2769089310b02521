// Step 5 for small batches: y[b][c] = sum_k o[b][k] Gt[c][k] with mma.sync.
//
// At decode batch sizes (B <= 8) the out-projection is a matrix-vector
// product: 2 * B flops per byte of the fused factor, far below the tensor
// ridge, so its cost is streaming Gt (hidden x Hq*r bf16) once plus fixed
// latencies.  This kernel keeps those latencies small: no cluster, no tensor
// memory, no distributed shared memory.
//
// One CTA per 32 output columns (128 CTAs for hidden = 4096), 16 warps.
// Before it waits for the attention kernel (it is launched as a programmatic
// dependent of it), thread 0 copies the CTA's 32 x K slice of the pre-tiled Gt
// into shared memory: one 4 KB bulk copy per 64-wide K chunk (the tile layout
// keeps 32 consecutive rows of a chunk contiguous, 128-byte rows with their
// 16-byte chunks XOR-swizzled by row).  After griddepcontrol.wait, warp w takes
// K range [w K/16, (w+1) K/16): it loads its o values straight into the
// m16n8k16 B-fragment layout, splits each fp32 value into bf16 hi + lo
// (o ~ hi + lo to ~2^-16 relative), and accumulates Gt.hi + Gt.lo for the
// two 16-row tiles of the CTA in fp32; ldmatrix reads the swizzled Gt rows
// without bank conflicts.  The 16 warps' partial tiles are summed in shared
// memory in warp order and written to y.
#include "kernels.cuh"

namespace bkv {

constexpr int kOpCols = 32;          // output columns per CTA
constexpr int kOpWarps = 16;
constexpr int kOpThreads = 32 * kOpWarps;
constexpr int kOpBatch = 8;          // batch rows (one n8 tile)
constexpr int kOpKGroup = 8;         // K steps of 16 whose o values a lane loads at once

__device__ __forceinline__ void op_ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void op_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 pair {x0, x1} (x0 in the low half) and the pair of their remainders
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
  const __nv_bfloat16 l0 = __float2bfloat16_rn(x0 - __bfloat162float(h0));
  const __nv_bfloat16 l1 = __float2bfloat16_rn(x1 - __bfloat162float(h1));
  hi = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
  lo = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
}

struct OutProjMmaParams {
  const __nv_bfloat16* Gt;  // pre-tiled: [hidden/128][K/64] tiles of 128 x 64, rows' 16-byte chunks swizzled
  const float* o;           // [B][K]
  float* y;                 // [B][hidden]
  int batch, K, hidden;
};

__global__ void __launch_bounds__(kOpThreads, 1) out_proj_mma_kernel(OutProjMmaParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_ok;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = blockIdx.x * kOpCols;
  const int KC = p.K / 64;  // 64-wide chunks; the CTA's slice of chunk kc sits at smem + kc * 4096
  float* red = reinterpret_cast<float*>(smem + (size_t)KC * 4096);  // [warps][32 rows][8 batch]

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    const int mt = c0 / 128, r0 = c0 % 128;
    const __nv_bfloat16* src = p.Gt + ((size_t)mt * KC * 128 + r0) * 64;  // chunk 0, row r0
    mbar_arrive_expect_tx(&bar, (uint32_t)KC * 4096u);
    for (int kc = 0; kc < KC; ++kc) bulk_g2s(smem + (size_t)kc * 4096, src + (size_t)kc * 128 * 64, 4096u, &bar);
  }
  grid_dep_wait();  // o is written by the kernel this one follows

  // this warp's K range, in steps of 16
  const int ksteps = p.K / 16 / kOpWarps;
  const int kbeg = warp * ksteps * 16;
  const int g = lane >> 2, t = lane & 3;  // fragment row / column pair
  const bool brow = g < p.batch;
  const float* orow = p.o + (size_t)(brow ? g : 0) * p.K;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix mi gets its row rr from this lane

  if (tid == 0) s_ok = mbar_wait_bounded(&bar, 0) ? 1 : 0;
  __syncthreads();
  const bool ok = s_ok != 0;
  for (int s0 = 0; s0 < ksteps && ok; s0 += kOpKGroup) {
    float2 x[kOpKGroup][2];
#pragma unroll
    for (int j = 0; j < kOpKGroup; ++j) {
      const int k = kbeg + (s0 + j) * 16 + 2 * t;
      const bool on = brow && s0 + j < ksteps;
      x[j][0] = on ? *reinterpret_cast<const float2*>(orow + k) : make_float2(0.f, 0.f);
      x[j][1] = on ? *reinterpret_cast<const float2*>(orow + k + 8) : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kOpKGroup; ++j) {
      if (s0 + j >= ksteps) break;
      uint32_t bh0, bl0, bh1, bl1;
      split_pair(x[j][0].x, x[j][0].y, bh0, bl0);
      split_pair(x[j][1].x, x[j][1].y, bh1, bl1);
      const int kk = kbeg + (s0 + j) * 16;
      const int kc = kk >> 6, cbase = (kk & 63) >> 3;  // chunk, first 16-byte column of this K step
      const uint32_t chunk = smem_u32(smem + (size_t)kc * 4096);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const int row = mt * 16 + (mi & 1) * 8 + rr;
        const int col = cbase + (mi >> 1);
        uint32_t a[4];
        op_ldsm4(a, chunk + (uint32_t)(row * 128 + ((col ^ (row & 7)) << 4)));
        op_mma(acc[mt], a, bh0, bh1);
        op_mma(acc[mt], a, bl0, bl1);
      }
    }
  }
  // acc[mt]: rows mt*16 + g (+8), batch columns 2t, 2t+1
  float* mine = red + (size_t)warp * kOpCols * kOpBatch;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    mine[(mt * 16 + g) * kOpBatch + 2 * t] = acc[mt][0];
    mine[(mt * 16 + g) * kOpBatch + 2 * t + 1] = acc[mt][1];
    mine[(mt * 16 + g + 8) * kOpBatch + 2 * t] = acc[mt][2];
    mine[(mt * 16 + g + 8) * kOpBatch + 2 * t + 1] = acc[mt][3];
  }
  __syncthreads();
  if (tid < kOpCols * kOpBatch) {
    const int r = tid % kOpCols, b = tid / kOpCols;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kOpWarps; ++w) v += red[((size_t)w * kOpCols + r) * kOpBatch + b];
    if (!ok) v = __int_as_float(0x7fc00000);  // the Gt copy did not arrive: mark the result
    if (b < p.batch) p.y[(size_t)b * p.hidden + c0 + r] = v;
  }
}

bool out_proj_mma_fits(int batch, int K, int hidden) {
  return batch >= 1 && batch <= kOpBatch && gt_blocked(K, hidden) && K % (16 * kOpWarps) == 0 &&
         (size_t)K / 64 * 4096 + (size_t)kOpWarps * kOpCols * kOpBatch * 4 <= 200 * 1024;
}

cudaError_t launch_out_proj_mma(const float* o, const void* Gt, float* y, int batch, int K, int hidden,
                                cudaStream_t st) {
  const OutProjMmaParams p{static_cast<const __nv_bfloat16*>(Gt), o, y, batch, K, hidden};
  const size_t smem = (size_t)K / 64 * 4096 + (size_t)kOpWarps * kOpCols * kOpBatch * 4;
  cudaError_t e = ensure_smem((const void*)out_proj_mma_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(hidden / kOpCols);
  cfg.blockDim = dim3(kOpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may start before the o producer ends
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, out_proj_mma_kernel, p);
}

}  // namespace bkv
