// Moving a decode step's inputs and outputs between page-locked host memory
// and the device with the SMs' own loads and stores.
//
// A decode step reads about a hundred kilobytes from the host (q, k_new,
// v_new) and returns about as much (y).  Inside a CUDA graph a copy-engine
// transfer of that size costs several times its wire time (the copy node's
// start and completion handshakes sit on the step's critical path), whereas
// one load or store per thread, all in flight at once, costs one round trip to
// host memory plus the bytes.  Page-locked host memory allocated or registered
// with the runtime is mapped into the device's address space (unified
// addressing), so a kernel reads it like device memory; stores to it are
// posted writes that the kernel's completion makes visible to the host.
#include "kernels.cuh"

namespace bkv {

constexpr int kCopyThreads = 256;

// dst[i] = src[i] for i < n16 (16-byte words), then the last `tail` (< 16)
// bytes one by one.  Either side may be device memory or mapped host memory.
__global__ void __launch_bounds__(kCopyThreads) copy16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                              size_t n16, const unsigned char* __restrict__ src_tail,
                                                              unsigned char* __restrict__ dst_tail, int tail) {
  const size_t stride = (size_t)gridDim.x * kCopyThreads;
  for (size_t i = (size_t)blockIdx.x * kCopyThreads + threadIdx.x; i < n16; i += stride) dst[i] = src[i];
  if (blockIdx.x == 0 && (int)threadIdx.x < tail) dst_tail[threadIdx.x] = src_tail[threadIdx.x];
}

cudaError_t launch_copy(void* dst, const void* src, size_t bytes, int num_sms, cudaStream_t st) {
  if (bytes == 0) return cudaSuccess;
  const size_t n16 = bytes / 16;
  const int tail = (int)(bytes - n16 * 16);
  // one word per thread up to 8 CTAs per SM (every load issued at once), then a grid-stride loop
  const size_t want = (n16 + kCopyThreads - 1) / kCopyThreads;
  const int grid = (int)(want < 1 ? 1 : (want > (size_t)num_sms * 8 ? (size_t)num_sms * 8 : want));
  copy16_kernel<<<grid, kCopyThreads, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16,
                                               static_cast<const unsigned char*>(src) + n16 * 16,
                                               static_cast<unsigned char*>(dst) + n16 * 16, tail);
  return cudaGetLastError();
}

}  // namespace bkv
