// Step 5 on the tensor cores: y^T = Gt . o^T with tcgen05 (sm_100a).
//
// The fused factor Gt [hidden][K] (K = Hq*r, K-major rows) is the A operand
// (M = 128 output columns per CTA), the rank-r attention outputs o [B][K] are
// the B operand (N = batch rows, padded to a multiple of 16).  o is fp32; it
// is split on the fly into bf16 hi + lo (o ~ hi + lo to ~2^-16 relative) and
// both halves are multiplied into the same fp32 TMEM accumulator, so the
// product keeps fp32-level accuracy with bf16 operands.
//
// Gt is stored pre-tiled for this kernel (basiskv_fuse_out_factor writes it):
// tile (m-tile, k-chunk) of 128 output columns x 64 latent dims is one
// contiguous 16 KB block holding exactly the 128-byte-swizzled shared-memory
// image the MMA reads, and the k-chunks of an m-tile are consecutive, so each
// CTA streams one contiguous region with 1-D bulk copies.
//
// Per CTA: warp 0 streams the 16 KB tiles of Gt (cp.async.bulk into this CTA only)
// into a ring of 4-8 stages and one of its threads issues the
// tcgen05.mma instructions, refilling each stage one iteration after its MMAs
// were committed; warps 1-4 prefetch the matching slices of o with cp.async,
// write them as swizzled bf16 hi/lo tiles into a matching ring and, at the
// end, read the accumulator out of TMEM.
// The K dimension is split over the CTAs of a thread-block cluster.  Each CTA
// stores its partial rows straight into the shared memory of the CTA that
// owns them (distributed shared memory stores); after one cluster barrier
// every CTA sums its slice of rows in rank order (deterministic) and writes y.
// HBM-bound: Gt is read once (16.8 MB for the 32K Llama-3-8B shape).
//
// The kernel is launched as a programmatic dependent of the attention kernel
// that produces o: the Gt stream starts as soon as SMs free up, and only the
// threads that read o wait (griddepcontrol.wait) for the producer to finish.
#include <stdio.h>

#include "kernels.cuh"
#include "tcgen05.cuh"

namespace bkv {

constexpr int kTcM = 128;        // output columns (rows of Gt) per CTA
constexpr int kTcK = 64;         // K per stage: one 128-byte swizzle atom of bf16
constexpr int kTcThreads = 160;  // warp 0: TMA + MMA; warps 1-4: o producers + epilogue
constexpr uint32_t kTcABytes = kTcM * kTcK * 2;

struct OutProjTcParams {
  const __nv_bfloat16* Gt;  // blocked: [hidden/128][K/64] tiles of 128x64, each a swizzled 16 KB image
  const float* o;           // [B][K]
  float* y;                 // [B][hidden]
  int32_t* err;
  int batch, K, hidden, chunks_per_cta, ksplit;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16-byte store into the shared memory of CTA `rank` of the cluster, at the
// address that `local` has in this CTA
__device__ __forceinline__ void st_dsmem_v4(const float* local, uint32_t rank, float4 v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(remote), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}


__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(pred ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ring depth per batch tile width (shared memory: A 16 KB, B 2*NB*128 B, o staging NB*256 B per stage;
// plus the 128 x NB fp32 receive buffer of the cluster reduction)
template <int NB>
struct TcStages {
  static constexpr int S = NB <= 16 ? 8 : NB <= 32 ? 6 : 4;
};

// The MMAs of one accumulator execute one after another; spreading the K-steps
// over kTcAcc accumulators (one per K = 16 slice of a stage and per hi / lo
// half) keeps the tensor core busy with independent chains.  The epilogue sums
// the accumulators.
constexpr int kTcAcc = 8;
template <int NB>
struct TcCols {  // TMEM columns: kTcAcc accumulators of NB fp32 columns, a power of two >= 32
  static constexpr uint32_t n = kTcAcc * NB <= 128 ? 128u : kTcAcc * NB <= 256 ? 256u : 512u;
};

template <int NB>
__global__ void __launch_bounds__(kTcThreads, 1)
    out_proj_tc_kernel(OutProjTcParams p) {
  constexpr int S = TcStages<NB>::S;
  constexpr uint32_t kBBytes = NB * kTcK * 2;       // one of hi / lo per stage
  constexpr uint32_t kStageF32 = NB * kTcK * 4;     // fp32 staging of o per stage
  constexpr int kChunks = NB * 8 / 128;            // 8-float chunks per producer thread per stage
  constexpr uint32_t kCols = TcCols<NB>::n;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  unsigned char* sB = smem + S * kTcABytes;
  unsigned char* sO = sB + S * 2 * kBBytes;
  float* recv = reinterpret_cast<float*>(sO + S * kStageF32);  // [ksplit][rows][NB]: partial rows from every rank
  uint64_t* afull = reinterpret_cast<uint64_t*>(recv + kTcM * NB);
  uint64_t* bfull = afull + S;
  uint64_t* empty = bfull + S;
  uint64_t* done = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  __shared__ int s_fail;  // a bounded wait gave up: the outputs of this cluster become NaN

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int c0 = blockIdx.y * kTcM;
  const int b0 = blockIdx.z * NB;
  const int KC = p.K / kTcK;
  const int ch0 = (int)rank * p.chunks_per_cta;
  const int nst = max(0, min(KC, ch0 + p.chunks_per_cta) - ch0);

  if (threadIdx.x == 0) s_fail = 0;
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(&afull[s], 1);
        mbar_init(&bfull[s], 128);
        mbar_init(&empty[s], 1);
      }
      mbar_init(done, 1);
      fence_mbar_init();
    }
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // this CTA has started; the matching wait comes before the first store into a peer's shared memory
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0 && nst > 0) {
      constexpr uint32_t idesc = idesc_bf16(kTcM, NB);
      // this CTA's tiles of Gt are one contiguous run of 16 KB images
      const __nv_bfloat16* gsrc = p.Gt + ((size_t)blockIdx.y * KC + ch0) * (kTcM * kTcK);
      for (int i = 0; i < min(S, nst); ++i) {
        mbar_arrive_expect_tx(&afull[i], kTcABytes);
        bulk_g2s(sA + i * kTcABytes, gsrc + (size_t)i * (kTcM * kTcK), kTcABytes, &afull[i]);
      }
      for (int i = 0; i < nst; ++i) {
        const int s = i % S;
        const uint32_t ph = (uint32_t)((i / S) & 1);
        if (!mbar_wait_bounded(&afull[s], ph) || !mbar_wait_bounded(&bfull[s], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = smem_desc_sw128(sA + s * kTcABytes);
        const uint64_t bh = smem_desc_sw128(sB + s * 2 * kBBytes);
        const uint64_t bl = smem_desc_sw128(sB + s * 2 * kBBytes + kBBytes);
#pragma unroll
        for (int j = 0; j < kTcK / 16; ++j) {
          const uint64_t step = (uint64_t)(j * 32) >> 4;  // 32 bytes per K = 16 slice
          const uint32_t acc_h = tmem + (uint32_t)(2 * j) * NB, acc_l = acc_h + NB;
          tc_mma(acc_h, ad + step, bh + step, idesc, i > 0 ? 1u : 0u);
          tc_mma(acc_l, ad + step, bl + step, idesc, i > 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        // refill the stage of the previous iteration (its MMAs have had a whole iteration to finish)
        const int ip = i - 1;
        if (ip >= 0 && ip + S < nst) {
          const int sp = ip % S;
          if (!mbar_wait_bounded(&empty[sp], (uint32_t)((ip / S) & 1))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&afull[sp], kTcABytes);
          bulk_g2s(sA + sp * kTcABytes, gsrc + (size_t)(ip + S) * (kTcM * kTcK), kTcABytes, &afull[sp]);
        }
      }
      tc_commit(done);  // arrives when every MMA issued above has completed
    }
    __syncwarp();
  } else {
    // o producers: each of the 128 threads owns kChunks 8-float chunks of every
    // stage; they are prefetched S stages ahead with cp.async into fp32 staging,
    // then split into bf16 hi / lo and written in the operand's swizzled layout
    const int t = threadIdx.x - 32;
    grid_dep_wait();  // o is written by the kernel this one follows
    auto issue = [&](int i) {
      unsigned char* stg = sO + (i % S) * kStageF32;
#pragma unroll
      for (int m = 0; m < kChunks; ++m) {
        const int idx = t + 128 * m;
        const int n = idx >> 3, c = idx & 7;
        const bool in = b0 + n < p.batch;
        const float* src = p.o + (in ? (size_t)(b0 + n) * p.K + (size_t)(ch0 + i) * kTcK + c * 8 : 0);
        cp_async16(stg + n * 256 + c * 32, src, in);
        cp_async16(stg + n * 256 + c * 32 + 16, src + 4, in);
      }
    };
    for (int i = 0; i < S; ++i) {
      if (i < nst) issue(i);
      cp_async_commit();
    }
    for (int i = 0; i < nst; ++i) {
      const int s = i % S;
      cp_async_wait<S - 1>();  // this thread's chunks of stage i have landed
      if (i >= S && !mbar_wait_bounded(&empty[s], (uint32_t)(((i / S) - 1) & 1))) {
        ok = false;
        break;
      }
      const unsigned char* stg = sO + s * kStageF32;
      unsigned char* hi_t = sB + s * 2 * kBBytes;
      unsigned char* lo_t = hi_t + kBBytes;
#pragma unroll
      for (int m = 0; m < kChunks; ++m) {
        const int idx = t + 128 * m;
        const int n = idx >> 3, c = idx & 7;
        const float4 x0 = *reinterpret_cast<const float4*>(stg + n * 256 + c * 32);
        const float4 x1 = *reinterpret_cast<const float4*>(stg + n * 256 + c * 32 + 16);
        const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * j]), h1 = __float2bfloat16_rn(v[2 * j + 1]);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * j] - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * j + 1] - __bfloat162float(h1));
          hw[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
          lw[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int off = n * 128 + ((c ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(hi_t + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lo_t + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bfull[s]);
      if (i + S < nst) issue(i + S);  // the staging slot of stage i is free again
      cp_async_commit();
    }
    cp_async_wait<0>();
  }

  // accumulator complete
  if (nst > 0 && !mbar_wait_bounded(done, 0)) ok = false;
  if (!ok) {
    s_fail = 1;
    set_err(p.err, BASISKV_DEVERR_TIMEOUT);
  }
  tc_fence_after();
  __syncthreads();
  // accumulator row m goes to the CTA that owns it: rank m / rows, slot [rank][m % rows]
  const int rows = kTcM / p.ksplit;
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every CTA of the cluster is running
  if (warp >= 1) {
    const int q = warp & 3;
    const int m = q * 32 + lane;
    const uint32_t owner = (uint32_t)(m / rows);
    float* slot = recv + ((size_t)rank * rows + (m % rows)) * NB;
#pragma unroll
    for (int cc = 0; cc < NB; cc += 16) {
      float v[16];
      tc_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)cc, v);
#pragma unroll
      for (int a = 1; a < kTcAcc; ++a) {
        float u[16];
        tc_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * NB + cc), u);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += u[j];
      }
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        const float4 x = (nst > 0) ? make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
        st_dsmem_v4(slot + cc + j, owner, x);
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // every partial row has landed in its owner's receive buffer
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
  }
  // this CTA's rows r0 .. r0 + rows - 1, summed over the ranks in order
  const int r0 = (int)rank * rows;
  for (int idx = threadIdx.x; idx < rows * NB; idx += blockDim.x) {
    const int n = idx / rows, mm = idx % rows;
    float acc = 0.f;
    for (int q = 0; q < p.ksplit; ++q) acc += recv[((size_t)q * rows + mm) * NB + n];
    if (s_fail) acc = __int_as_float(0x7fc00000);  // NaN marks a result that cannot be trusted
    if (b0 + n < p.batch) p.y[(size_t)(b0 + n) * p.hidden + c0 + r0 + mm] = acc;
  }
}

// ---------------------------------------------------------------------------
// host side: tensor map (cached per pointer/shape/device) and launch
// ---------------------------------------------------------------------------
bool gt_blocked(int K, int hidden) { return K % kTcK == 0 && hidden % kTcM == 0; }

template <int NB>
static size_t tc_smem_bytes() {
  constexpr int S = TcStages<NB>::S;
  return 1024 + (size_t)S * kTcABytes + (size_t)S * 2 * NB * kTcK * 2 + (size_t)S * NB * kTcK * 4 +
         (size_t)kTcM * NB * 4 + (3 * S + 1) * 8 + 16;
}

template <int NB>
static cudaError_t launch_tc_nb(OutProjTcParams p, int num_sms, cudaStream_t st) {
  const int mtiles = p.hidden / kTcM;
  const int bchunks = (p.batch + NB - 1) / NB;
  const int KC = p.K / kTcK;
  int ks = 1;
  while (ks * 2 <= 8 && ks * 2 <= KC && (long long)mtiles * bchunks * ks * 2 <= num_sms) ks *= 2;
  p.ksplit = ks;
  p.chunks_per_cta = (KC + ks - 1) / ks;
  const size_t smem = tc_smem_bytes<NB>();
  cudaError_t e = ensure_smem((const void*)out_proj_tc_kernel<NB>, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ks, mtiles, bchunks);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may start before the o producer ends
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, out_proj_tc_kernel<NB>, p);
}

cudaError_t launch_out_proj_tc(const float* o, const void* Gt, float* y, int32_t* err, int batch, int K, int hidden,
                               int num_sms, cudaStream_t st) {
  OutProjTcParams p{static_cast<const __nv_bfloat16*>(Gt), o, y, err, batch, K, hidden, 0, 1};
  const int nb = batch <= 16 ? 16 : batch <= 32 ? 32 : batch <= 48 ? 48 : 64;
  switch (nb) {
    case 16: return launch_tc_nb<16>(p, num_sms, st);
    case 32: return launch_tc_nb<32>(p, num_sms, st);
    case 48: return launch_tc_nb<48>(p, num_sms, st);
    default: return launch_tc_nb<64>(p, num_sms, st);
  }
}

}  // namespace bkv
